// conv.cu -- depthwise causal conv1d over time + SiLU + per-head L2 normalisation of q and k.
//
// Source: "Qwen3.5 Gated DeltaNet 核心机制解析", conv-layer section and flowchart: the q|k|v mix
// passes a depthwise causal conv (local context) before it is split into q, k and v.
//
//   pre[t,c] = bias[c] + sum_{i<K} w[c,i] * x[t-(K-1)+i, c]        y = silu(pre)
//   each group of `group` channels among the first n_l2 channels:  y[t,G] /= sqrt(|y[t,G]|^2 + eps)
//
// HBM-bound stencil: x is read once (plus a K-1 token halo per block) and y written once.  Each
// thread owns 8 consecutive channels (one 16-byte bf16 vector per token) and streams a long,
// contiguous token range of them; a warp covers 256 contiguous channels, so every token row is
// read and written as 512-byte coalesced segments.
//
// Memory-level parallelism comes from a private per-thread ring in shared memory: each thread
// keeps DEPTH-NT tokens of its own channels in flight with cp.async (16-byte, L1-bypassing), and
// waits only for the oldest ones.  Because a thread reads back only the slots it filled itself,
// no block-wide synchronisation is needed.  The last K-1 inputs live in registers as a circular
// window whose rotation is unrolled, so no register moves are spent on shifting it, and tokens
// are computed two or three at a time in packed fp32 (two lanes per instruction) so that the
// latency chains of conv -> SiLU -> norm overlap.  The grid is one wave (two blocks per SM for
// K <= 4), each block taking an equal share of the tokens of one 2048-channel slab.  The L2 norm
// of a head is a shuffle reduction over the group's group/8 lanes, skipped by warps that hold
// only v channels.
#include <type_traits>

#include "gdn_internal.cuh"

namespace gdn {

constexpr int CONV_THREADS = 256;     // 8 channels per thread -> 2048 channels per block
// blocks per SM: two while weights + window fit the 128 registers that allows (K <= 4), else one
__host__ __device__ constexpr int conv_blocks_per_sm(int K) { return K <= 4 ? 2 : 1; }
constexpr int CONV_RING_BYTES = 256;  // per-thread ring: 16 bf16 tokens or 8 fp32 tokens
constexpr int CONV_MIN_TOKENS = 64;   // fewest tokens per block

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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a)
               : "memory");
  return v;
}

// 8 channels of one token, as stored in the ring (V 16-byte parts, CONV_THREADS*16 apart), as
// four channel pairs
__device__ __forceinline__ void ring_to_float2(uint32_t a, const __nv_bfloat16*, float2 (&f)[4]) {
  const uint4 u = lds128(a);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    f[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
}
__device__ __forceinline__ void ring_to_float2(uint32_t a, const float*, float2 (&f)[4]) {
  const uint4 u = lds128(a);
  const uint4 v = lds128(a + CONV_THREADS * 16);
  f[0] = make_float2(__uint_as_float(u.x), __uint_as_float(u.y));
  f[1] = make_float2(__uint_as_float(u.z), __uint_as_float(u.w));
  f[2] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
  f[3] = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
}
__device__ __forceinline__ void store8x2(__nv_bfloat16* p, const float2 (&f)[4]) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __float22bfloat162_rn(f[i]);
  *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void store8x2(float* p, const float2 (&f)[4]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(f[0].x, f[0].y, f[1].x, f[1].y);
  reinterpret_cast<float4*>(p)[1] = make_float4(f[2].x, f[2].y, f[3].x, f[3].y);
}
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// silu on two channel pairs (four channels): x / (1 + 2^(-x log2 e)).  The four exponentials are
// special-function ops; the four reciprocals share one: with d_i = 1 + 2^(-x_i log2 e) and
// r = 1 / (d1 d2 d3 d4), 1/d1 = r d2 d3 d4 and so on (products formed pairwise), so the element
// costs 1.25 special-function ops instead of 2, at the price of a few packed multiplies.  Each
// exponent is clamped at 31 so that the product of four d_i stays below 2^124 and its reciprocal
// a normal number: for x < -21.5 the sigmoid factor then reads 2^-31 instead of e^x, an absolute
// error below 5e-10 |x| in the result.  The products and the reciprocal add about three roundings
// (< 4e-7 relative), far below bf16's 2^-8.
__device__ __forceinline__ void silu4(float2& a, float2& b) {
  const float2 l2e = make_float2(-1.4426950408889634f, -1.4426950408889634f);
  const float2 ma = __fmul2_rn(a, l2e), mb = __fmul2_rn(b, l2e);
  const float2 one = make_float2(1.f, 1.f);
  const float2 da = __fadd2_rn(make_float2(ex2_approx(fminf(ma.x, 31.f)),
                                           ex2_approx(fminf(ma.y, 31.f))), one);
  const float2 db = __fadd2_rn(make_float2(ex2_approx(fminf(mb.x, 31.f)),
                                           ex2_approx(fminf(mb.y, 31.f))), one);
  // p = (da.x db.x, da.y db.y); then the reciprocal of the full product
  const float2 p = __fmul2_rn(da, db);
  const float r = rcp_approx(p.x * p.y);
  const float2 rp = __fmul2_rn(make_float2(r, r), make_float2(p.y, p.x));  // 1/(da.x db.x), ...
  // 1/da = rp * db, 1/db = rp * da (component-wise)
  const float2 ia = __fmul2_rn(rp, db), ib = __fmul2_rn(rp, da);
  a = __fmul2_rn(a, ia);
  b = __fmul2_rn(b, ib);
}

template <typename T, int K>
__global__ void __launch_bounds__(CONV_THREADS, conv_blocks_per_sm(K)) conv_silu_kernel(
    const T* __restrict__ x, const float* __restrict__ w, const float* __restrict__ bias,
    int64_t n_tok, int64_t Tlen, int C, const int32_t* __restrict__ cu, int N, int n_l2,
    int group, float l2_eps, const float* __restrict__ cs_in, float* __restrict__ cs_out,
    T* __restrict__ y) {
  constexpr int V = (int)sizeof(T) / 2;              // 16-byte parts per 8-channel vector
  constexpr int DEPTH = CONV_RING_BYTES / (16 * V);  // ring slots per thread
  constexpr uint32_t SLOT = V * CONV_THREADS * 16;   // bytes per ring slot (whole block)
  constexpr int W = K > 1 ? K - 1 : 1;               // window length
  // tokens computed side by side: three where the window length allows a group of two triples
  // (and the registers allow: bf16), else two
  constexpr int NT = (W % 3 == 0 && sizeof(T) == 2) ? 3 : 2;
  // tokens per unrolled group: a multiple of W (the window returns to phase 0) and of NT
  constexpr int U = NT == 3 ? 6 : (W >= 4 ? (W % 2 ? 2 * W : W) : W * (8 / W));
  static_assert(U % W == 0 && U % NT == 0, "group must hold whole windows and whole steps");
  static_assert((DEPTH & (DEPTH - 1)) == 0, "ring depth must be a power of two");
  extern __shared__ __align__(16) uint4 conv_ring[];

  const int cc = blockIdx.y * CONV_THREADS + threadIdx.x;
  const int c0 = cc * 8;
  const int warp_c0 = (blockIdx.y * CONV_THREADS + (threadIdx.x & ~31)) * 8;
  if (warp_c0 >= C) return;  // whole warp past the last channel (warp-uniform)
  const bool chan_ok = c0 < C;
  const bool do_norm = chan_ok && c0 < n_l2;
  const int lanes_per_group = group >> 3;  // 0 when no normalisation
  const bool warp_norm = lanes_per_group > 0 && warp_c0 < n_l2;

  // weights and bias of the thread's 8 channels, as channel pairs (p: channels 2p, 2p+1)
  float2 wt[4][K];
  float2 bs[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    bs[p] = (chan_ok && bias) ? make_float2(__ldg(bias + c0 + 2 * p), __ldg(bias + c0 + 2 * p + 1))
                              : make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < K; ++i)
      wt[p][i] = chan_ok ? make_float2(__ldg(w + (int64_t)(c0 + 2 * p) * K + i),
                                       __ldg(w + (int64_t)(c0 + 2 * p + 1) * K + i))
                         : make_float2(0.f, 0.f);
  }

  // Zero-length sequences still produce a conv state (copied through); blocks of column 0 do it.
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

  const int64_t t_begin = n_tok * blockIdx.x / gridDim.x;
  const int64_t t_end = n_tok * (blockIdx.x + 1) / gridDim.x;
  if (t_begin >= t_end) return;  // block-uniform

  // ---- per-thread cp.async ring: token t_begin + i lives in slot i % DEPTH
  const uint32_t ring = (uint32_t)__cvta_generic_to_shared(conv_ring) + threadIdx.x * 16u;
  const T* xsrc = x + c0;
  auto issue = [&](int64_t i) {  // start loading token t_begin + i; one commit group per token
    const int64_t t = t_begin + i;
    if (chan_ok && t < t_end) {
      const uint32_t dst = ring + (uint32_t)(i & (DEPTH - 1)) * SLOT;
      const char* src = reinterpret_cast<const char*>(xsrc + t * C);
#pragma unroll
      for (int v = 0; v < V; ++v) cp_async16(dst + v * CONV_THREADS * 16, src + 16 * v);
    }
    cp_async_commit();
  };
  // Before token t_begin + i is taken, tokens up to i + DEPTH - NT - 1 have been issued.
  // Taking m <= NT tokens refills m of the NT slots before token i, all consumed by earlier
  // steps (their values are already in registers and used), then waits until token i + m - 1
  // has landed: DEPTH - NT newer groups may still be in flight.
  auto take = [&](auto nt, int64_t i, float2 (*xt)[4]) {
    constexpr int M = decltype(nt)::value;
    static_assert(M <= NT, "a step takes at most NT tokens");
#pragma unroll
    for (int k = 0; k < M; ++k) issue(i + k + DEPTH - NT);
    cp_async_wait<DEPTH - NT>();
#pragma unroll
    for (int k = 0; k < M; ++k) {
      if (chan_ok) {
        ring_to_float2(ring + (uint32_t)((i + k) & (DEPTH - 1)) * SLOT, x, xt[k]);
      } else {
#pragma unroll
        for (int p = 0; p < 4; ++p) xt[k][p] = make_float2(0.f, 0.f);
      }
    }
  };
#pragma unroll 1
  for (int i = 0; i < DEPTH - NT; ++i) issue(i);

  int n = seq_of_token(cu, N, Tlen, t_begin);
  int64_t s_beg, s_end;
  seq_range(cu, Tlen, n, s_beg, s_end);

  // win[j][q], j = 0..K-2, in "phase 0" order: oldest input first; q = channel pair.
  float2 win[W][4];
#pragma unroll
  for (int j = 0; j < W; ++j)
#pragma unroll
    for (int q = 0; q < 4; ++q) win[j][q] = make_float2(0.f, 0.f);
  auto fill_window = [&](int64_t t) {
#pragma unroll
    for (int j = 0; j < K - 1; ++j) {
      const int64_t p = t - (K - 1) + j;
      float f[8];
      if (!chan_ok) {
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = 0.0f;
      } else if (p >= s_beg && p >= 0 && p < n_tok) {
        load8(x + p * C + c0, f);
      } else {
        // before the sequence start: carried conv state (or zero).  The range check only
        // matters for a malformed cu_seqlens, which must not cause out-of-bounds reads.
        const int64_t r = (K - 1) + (p - s_beg);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          f[e] = (cs_in && r >= 0 && r < K - 1) ? cs_in[((int64_t)n * C + c0 + e) * (K - 1) + r]
                                                : 0.0f;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) win[j][q] = make_float2(f[2 * q], f[2 * q + 1]);
    }
  };

  // conv + SiLU + (optional) head L2 norm + store of M (NT or one) consecutive tokens from t.
  // The window order is rotated by `ph` (token t's oldest input sits in win[ph]); each token
  // overwrites its oldest slot with its own input, which the next token then sees as its newest.
  // The tokens of a step are computed side by side, so their dependency chains overlap.
  auto tokens = [&](auto nt, int64_t t, const float2 (*xt)[4], int ph) {
    constexpr int M = decltype(nt)::value;
    float2 acc[M][4];
#pragma unroll
    for (int k = 0; k < M; ++k) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float2 a = bs[q];
#pragma unroll
        for (int j = 0; j < K - 1; ++j) a = __ffma2_rn(wt[q][j], win[(ph + k + j) % W][q], a);
        acc[k][q] = __ffma2_rn(wt[q][K - 1], xt[k][q], a);
      }
      if (K > 1) {
#pragma unroll
        for (int q = 0; q < 4; ++q) win[(ph + k) % W][q] = xt[k][q];
      }
    }
#pragma unroll
    for (int k = 0; k < M; ++k) {
      silu4(acc[k][0], acc[k][1]);
      silu4(acc[k][2], acc[k][3]);
    }
    if (warp_norm) {
      float ss[M];
#pragma unroll
      for (int k = 0; k < M; ++k) {
        float2 s2 = __fmul2_rn(acc[k][0], acc[k][0]);
#pragma unroll
        for (int q = 1; q < 4; ++q) s2 = __ffma2_rn(acc[k][q], acc[k][q], s2);
        ss[k] = s2.x + s2.y;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
        if (o < lanes_per_group) {
#pragma unroll
          for (int k = 0; k < M; ++k) ss[k] += __shfl_xor_sync(0xffffffffu, ss[k], o);
        }
#pragma unroll
      for (int k = 0; k < M; ++k) {
        const float inv = do_norm ? rsqrtf(ss[k] + l2_eps) : 1.0f;
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[k][q] = __fmul2_rn(acc[k][q], make_float2(inv, inv));
      }
    }
    if (chan_ok) {
#pragma unroll
      for (int k = 0; k < M; ++k) store8x2(y + (t + k) * C + c0, acc[k]);
    }
  };
  using One = std::integral_constant<int, 1>;
  using Step = std::integral_constant<int, NT>;

  int64_t t = t_begin;
  if (t >= s_beg && t < s_end) fill_window(t);
  while (t < t_end) {
    if (t >= s_end) {  // entered the next non-empty sequence
      if (cu) {
        while (n + 1 < N && (int64_t)cu[n + 1] <= t) ++n;
      } else {
        n = (int)(t / Tlen);
      }
      seq_range(cu, Tlen, n, s_beg, s_end);
      if (t >= s_beg && t < s_end) fill_window(t);
    }
    if (t < s_beg || t >= s_end) {
      // token outside every sequence (only a malformed cu_seqlens): consume it, write nothing
      const int64_t stop = t < s_beg ? min(s_beg, t_end) : t_end;
      for (; t < stop; ++t) {
        float2 xt[1][4];
        take(One{}, t - t_begin, xt);
      }
      continue;
    }
    const int64_t seg_end = min(s_end, t_end);
    // groups of U tokens: the window rotates through all W phases and returns to phase 0
    while (t + U <= seg_end) {
#pragma unroll
      for (int u = 0; u < U; u += NT) {
        float2 xt[NT][4];
        take(Step{}, t + u - t_begin, xt);
        tokens(Step{}, t + u, xt, u % W);
      }
      t += U;
    }
    // tail: phase 0 every token, window shifted in registers
    for (; t < seg_end; ++t) {
      float2 xt[1][4];
      take(One{}, t - t_begin, xt);
      tokens(One{}, t, xt, 0);  // overwrote win[0] (the oldest) with xt: rotate back to phase 0
      if (K > 2) {
        float2 tmp[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmp[q] = win[0][q];
#pragma unroll
        for (int j = 0; j + 1 < K - 1; ++j)
#pragma unroll
          for (int q = 0; q < 4; ++q) win[j][q] = win[j + 1][q];
#pragma unroll
        for (int q = 0; q < 4; ++q) win[W - 1][q] = tmp[q];
      }
    }
    if (t == s_end && cs_out && chan_ok) {
      // last token of sequence n was t-1: the window holds its last K-1 inputs, oldest first
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int j = 0; j < K - 1; ++j) {
          cs_out[((int64_t)n * C + c0 + 2 * q) * (K - 1) + j] = win[j][q].x;
          cs_out[((int64_t)n * C + c0 + 2 * q + 1) * (K - 1) + j] = win[j][q].y;
        }
    }
  }
  cp_async_wait<0>();  // leave no copy in flight into shared memory
}

template <typename T, int K>
static cudaError_t launch_conv_k(int sms, int64_t n_tok, int slabs, const T* x, const float* w,
                                 const float* bias, int64_t T_, int C, const int32_t* cu, int N,
                                 int n_l2, int group, float l2_eps, const float* cs_in,
                                 float* cs_out, T* y, cudaStream_t s) {
  // one wave: every resident block slot gets an equal share of one slab's tokens
  int64_t cols = ((int64_t)sms * conv_blocks_per_sm(K) + slabs - 1) / slabs;
  const int64_t by_len = (n_tok + CONV_MIN_TOKENS - 1) / CONV_MIN_TOKENS;
  if (cols > by_len) cols = by_len;
  if (cols < 1) cols = 1;
  const dim3 grid((unsigned)cols, (unsigned)slabs);
  constexpr int smem = CONV_RING_BYTES * CONV_THREADS;
  static bool attr_set = false;  // idempotent attribute; a benign race between host threads
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(conv_silu_kernel<T, K>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  conv_silu_kernel<T, K><<<grid, CONV_THREADS, smem, s>>>(x, w, bias, n_tok, T_, C, cu, N, n_l2,
                                                          group, l2_eps, cs_in, cs_out, y);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_conv_t(const T* x, const float* w, const float* bias, int B, int64_t T_,
                                 int C, int K, const int32_t* cu, int N, int n_l2, int group,
                                 float l2_eps, const float* cs_in, float* cs_out, T* y,
                                 cudaStream_t s) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t n_tok = (int64_t)B * T_;
  const int slabs = (C / 8 + CONV_THREADS - 1) / CONV_THREADS;
  if (slabs > 65535) return cudaErrorInvalidConfiguration;
  switch (K) {
#define GDN_CONV_CASE(KK) \
  case KK:                \
    return launch_conv_k<T, KK>(sms, n_tok, slabs, x, w, bias, T_, C, cu, N, n_l2, group, \
                                l2_eps, cs_in, cs_out, y, s);
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
