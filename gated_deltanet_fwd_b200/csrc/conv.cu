// conv.cu -- depthwise causal conv1d over time + SiLU + per-head L2 normalisation of q and k.
//
// Source: "Qwen3.5 Gated DeltaNet 核心机制解析", conv-layer section and flowchart: the q|k|v mix
// passes a depthwise causal conv (local context) before it is split into q, k and v.
//
//   pre[t,c] = bias[c] + sum_{i<K} w[c,i] * x[t-(K-1)+i, c]        y = silu(pre)
//   each group of `group` channels among the first n_l2 channels:  y[t,G] /= sqrt(|y[t,G]|^2 + eps)
//
// HBM-bound stencil: x is read once (plus a K-1 token halo per tile, served by L2) and y written
// once.  Each thread owns 8 consecutive channels (one 16-byte bf16 transaction per token) and walks
// a tile of TT tokens, keeping the last K-1 inputs in registers; a warp covers 256 contiguous
// channels, so every token row is read as 512-byte coalesced segments.  The L2 norm of a head is a
// shuffle reduction over the group's group/8 lanes.
#include "gdn_internal.cuh"

namespace gdn {

constexpr int CONV_TT = 32;       // tokens per tile
constexpr int CONV_THREADS = 128; // threads per block -> 1024 channels per block
constexpr int CONV_U = 8;         // tokens loaded ahead per batch

__device__ __forceinline__ void seq_range(const int32_t* cu, int64_t T, int n, int64_t& s,
                                          int64_t& e) {
  if (cu) {
    s = cu[n];
    e = cu[n + 1];
  } else {
    s = (int64_t)n * T;
    e = s + T;
  }
}

template <typename T, int K>
__global__ void __launch_bounds__(CONV_THREADS, 4) conv_silu_kernel(
    const T* __restrict__ x, const float* __restrict__ w, const float* __restrict__ bias,
    int64_t n_tok, int64_t Tlen, int C, const int32_t* __restrict__ cu, int N, int n_l2,
    int group, float l2_eps, const float* __restrict__ cs_in, float* __restrict__ cs_out,
    T* __restrict__ y) {
  const int cc = blockIdx.y * CONV_THREADS + threadIdx.x;
  const int c0 = cc * 8;
  const bool chan_ok = c0 < C;
  const bool do_norm = chan_ok && c0 < n_l2;

  float wt[8][K];
  float bs[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    bs[e] = (chan_ok && bias) ? __ldg(bias + c0 + e) : 0.0f;
#pragma unroll
    for (int i = 0; i < K; ++i) wt[e][i] = chan_ok ? __ldg(w + (int64_t)(c0 + e) * K + i) : 0.0f;
  }

  // Zero-length sequences still produce a conv state (copied through); tile 0 handles them.
  if (blockIdx.x == 0 && cs_out && chan_ok && cu) {
    for (int n = 0; n < N; ++n) {
      if (cu[n + 1] != cu[n]) continue;
      for (int e = 0; e < 8; ++e)
        for (int j = 0; j < K - 1; ++j) {
          const int64_t o = ((int64_t)n * C + c0 + e) * (K - 1) + j;
          cs_out[o] = cs_in ? cs_in[o] : 0.0f;
        }
    }
  }

  const int64_t t_begin = (int64_t)blockIdx.x * CONV_TT;
  if (t_begin >= n_tok) return;
  const int64_t t_end = min(t_begin + (int64_t)CONV_TT, n_tok);

  int n = seq_of_token(cu, N, Tlen, t_begin);
  int64_t s_beg, s_end;
  seq_range(cu, Tlen, n, s_beg, s_end);

  // win[j][e]: input at position t-(K-1)+j for the next token t (oldest first).
  float win[K > 1 ? K - 1 : 1][8];
  auto fill_window = [&](int64_t t) {
#pragma unroll
    for (int j = 0; j < K - 1; ++j) {
      const int64_t p = t - (K - 1) + j;
      if (!chan_ok) {
#pragma unroll
        for (int e = 0; e < 8; ++e) win[j][e] = 0.0f;
      } else if (p >= s_beg && p >= 0 && p < n_tok) {
        load8(x + p * C + c0, win[j]);
      } else {
        // before the sequence start: carried conv state (or zero).  The range check only
        // matters for a malformed cu_seqlens, which must not cause out-of-bounds reads.
        const int64_t r = (K - 1) + (p - s_beg);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          win[j][e] = (cs_in && r >= 0 && r < K - 1)
                          ? cs_in[((int64_t)n * C + c0 + e) * (K - 1) + r]
                          : 0.0f;
      }
    }
  };
  fill_window(t_begin);

  const int lanes_per_group = group >> 3;  // 0 when no normalisation
  for (int64_t tb = t_begin; tb < t_end; tb += CONV_U) {
    Raw8<T> xs[CONV_U];
#pragma unroll
    for (int u = 0; u < CONV_U; ++u) {
      if (chan_ok && tb + u < t_end)
        xs[u].load(x + (tb + u) * C + c0);
      else
        xs[u].zero();
    }
#pragma unroll
    for (int u = 0; u < CONV_U; ++u) {
      const int64_t t = tb + u;
      if (t >= t_end) break;  // uniform across the block
      if (t >= s_end) {       // entered the next non-empty sequence
        if (cu) {
          while (n + 1 < N && (int64_t)cu[n + 1] <= t) ++n;
        } else {
          n = (int)(t / Tlen);
        }
        seq_range(cu, Tlen, n, s_beg, s_end);
        fill_window(t);
      }
      // false only when cu_seqlens is malformed (token outside every sequence): skip writes
      const bool tok_ok = t >= s_beg && t < s_end;
      float xt[8];
      xs[u].to_float(xt);
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float a = bs[e];
#pragma unroll
        for (int j = 0; j < K - 1; ++j) a = fmaf(wt[e][j], win[j][e], a);
        acc[e] = silu_fast(fmaf(wt[e][K - 1], xt[e], a));
      }
#pragma unroll
      for (int j = 0; j + 1 < K - 1; ++j)
#pragma unroll
        for (int e = 0; e < 8; ++e) win[j][e] = win[j + 1][e];
      if (K > 1) {
#pragma unroll
        for (int e = 0; e < 8; ++e) win[K > 1 ? K - 2 : 0][e] = xt[e];
      }
      if (lanes_per_group) {
        float ss = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(acc[e], acc[e], ss);
        for (int o = lanes_per_group >> 1; o > 0; o >>= 1)
          ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (do_norm) {
          const float inv = rsqrtf(ss + l2_eps);
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] *= inv;
        }
      }
      if (chan_ok && tok_ok) store8(y + t * C + c0, acc);
      if (cs_out && chan_ok && tok_ok && t == s_end - 1) {
        // last token of sequence n: the window now holds its last K-1 inputs
#pragma unroll
        for (int e = 0; e < 8; ++e)
#pragma unroll
          for (int j = 0; j < K - 1; ++j)
            cs_out[((int64_t)n * C + c0 + e) * (K - 1) + j] = win[j][e];
      }
    }
  }
}

template <typename T>
static cudaError_t launch_conv_t(const T* x, const float* w, const float* bias, int B, int64_t T_,
                                 int C, int K, const int32_t* cu, int N, int n_l2, int group,
                                 float l2_eps, const float* cs_in, float* cs_out, T* y,
                                 cudaStream_t s) {
  const int64_t n_tok = (int64_t)B * T_;
  const int64_t tiles = n_tok > 0 ? (n_tok + CONV_TT - 1) / CONV_TT : 1;
  const int chunks = C / 8;
  dim3 grid((unsigned)tiles, (unsigned)((chunks + CONV_THREADS - 1) / CONV_THREADS));
  if (grid.y > 65535u) return cudaErrorInvalidConfiguration;
  switch (K) {
#define GDN_CONV_CASE(KK)                                                                     \
  case KK:                                                                                    \
    conv_silu_kernel<T, KK><<<grid, CONV_THREADS, 0, s>>>(x, w, bias, n_tok, T_, C, cu, N,    \
                                                          n_l2, group, l2_eps, cs_in, cs_out, \
                                                          y);                                 \
    break;
    GDN_CONV_CASE(1)
    GDN_CONV_CASE(2)
    GDN_CONV_CASE(3)
    GDN_CONV_CASE(4)
    GDN_CONV_CASE(5)
    GDN_CONV_CASE(6)
    GDN_CONV_CASE(7)
    GDN_CONV_CASE(8)
#undef GDN_CONV_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_conv(const void* x, gdn_dtype dt, const float* w, const float* bias, int B,
                        int64_t T, int C, int K, const int32_t* cu, int N, int n_l2, int group,
                        float l2_eps, const float* cs_in, float* cs_out, void* y,
                        cudaStream_t s) {
  if (dt == GDN_BF16)
    return launch_conv_t((const __nv_bfloat16*)x, w, bias, B, T, C, K, cu, N, n_l2, group, l2_eps,
                         cs_in, cs_out, (__nv_bfloat16*)y, s);
  return launch_conv_t((const float*)x, w, bias, B, T, C, K, cu, N, n_l2, group, l2_eps, cs_in,
                       cs_out, (float*)y, s);
}

}  // namespace gdn
