// decode_fused.cu -- one decode token of the whole linear-attention layer core in one launch:
// causal conv over the cached inputs + SiLU + q/k L2 norm, the gates, the recurrent step of the
// gated delta rule on the cached state, and the gated RMSNorm of the output.
//
// Sources: "Qwen3.5 Gated DeltaNet 核心机制解析" -- cache and state switching (the decode path keeps
// conv_states, the last K-1 inputs of the conv, and recurrent_states, the delta-rule state, and
// advances both by one token) and the flowchart (conv -> split -> gates -> delta rule ->
// RMSNormGated(core_attn_out, z)); "解密Qwen3-Next的Gated DeltaNet：如何用75%混合层实现长文本高效推理"
// §2.2 (recurrent mode) and §3.2 (zero-centred RMSNorm).  Per (sequence n, v-head h), exactly
//     gdn_causal_conv1d_silu (one token, conv_state_in as the history) -> gdn_gates ->
//     gdn_recurrent_step -> gdn_gated_rmsnorm
// except that q, k, v stay in fp32 between the conv and the delta rule instead of being rounded to
// the activation type.
//
// HBM-bound like the plain decode step: the 64 KB state of the (sequence, head) is read and written
// once; its first rows (and the z gate) are requested before the conv prologue runs, so the
// prologue hides under their latency.  One block of 256 threads per (sequence, v-head); each warp
// streams 8 rows at a time as float4 lanes (a row is one 512-byte transaction), as in recurrent.cu.
// (Requesting all 16 rows of a warp up front needs 127 registers and two blocks per SM; measured
// slower, 267 us against 220 us per token on the 256-sequence workload.)
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int DF_THREADS = 256;
constexpr int DF_ROWS = 8;  // rows per warp per batch
constexpr int DF_D = 128;   // dk = dv

__device__ __forceinline__ float dwarp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// One channel's conv inputs: the new input, its K-1 cached predecessors (oldest first) and the
// K taps.  Loaded for all of a thread's channels before any of them is computed or its history
// written, so that the loads form one round trip.
struct ConvIn {
  float xt, bias;
  float hist[7];
  float w[8];
};

template <typename T>
__device__ __forceinline__ void conv_load(ConvIn& ci, const T* __restrict__ x,
                                          const float* __restrict__ w,
                                          const float* __restrict__ bias, int K, int64_t c,
                                          const float* __restrict__ cs_in) {
  ci.xt = to_f(x[c]);
  ci.bias = bias ? __ldg(bias + c) : 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) ci.w[i] = i < K ? __ldg(w + c * K + i) : 0.0f;
#pragma unroll
  for (int i = 0; i < 7; ++i) ci.hist[i] = i < K - 1 ? cs_in[c * (K - 1) + i] : 0.0f;
}

// silu(conv) of a loaded channel; writes its history shifted by this token when `write_state`
__device__ __forceinline__ float conv_finish(const ConvIn& ci, int K, int64_t c,
                                             float* __restrict__ cs_out, bool write_state) {
  float acc = ci.bias;
#pragma unroll
  for (int i = 0; i < 8; ++i) {  // tap i: cached input i, or the new input at i = K - 1
    // (i < K - 1 <= 7 whenever hist is read; the clamp only keeps the index constant-foldable)
    const float xi = i < K - 1 ? ci.hist[i < 7 ? i : 6] : (i == K - 1 ? ci.xt : 0.0f);
    acc = fmaf(ci.w[i], xi, acc);
  }
  if (write_state && K > 1) {
    float* hout = cs_out + c * (K - 1);
#pragma unroll
    for (int i = 0; i < 6; ++i)
      if (i + 1 < K - 1) hout[i] = ci.hist[i + 1];
    hout[K - 2] = ci.xt;
  }
  return siluf_(acc);
}

struct DecodeParams {
  const void* mix;
  const void* a;
  const void* b;
  const void* z;
  const float* conv_w;
  const float* conv_bias;
  const float* cs_in;
  float* cs_out;
  const float* A_log;
  const float* dt_bias;
  const float* norm_w;
  float* state;
  void* y;
  float l2_eps, norm_eps, scale;
  int K, Hk, Hv;
  int64_t C;  // mix channels: 2 Hk dk + Hv dv
};

template <typename T>
__global__ void __launch_bounds__(DF_THREADS, 3) decode_fused_kernel(const DecodeParams P) {
  __shared__ float q_s[DF_D], k_s[DF_D], v_s[DF_D], o_s[DF_D];
  __shared__ float red[16];
  __shared__ float gate_s[2];
  const int nh = blockIdx.x;  // n * Hv + h
  const int n = nh / P.Hv, h = nh - n * P.Hv;
  const int G = P.Hv / P.Hk, hk = h / G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float* S = P.state + (int64_t)nh * DF_D * DF_D;

  // ---- the first batch of state rows is requested before the prologue
  float4 s[DF_ROWS];
  {
    const float* Sb = S + (size_t)(warp * DF_ROWS) * DF_D;
#pragma unroll
    for (int u = 0; u < DF_ROWS; ++u)
      s[u] = __ldcs(reinterpret_cast<const float4*>(Sb + u * DF_D) + lane);
  }

  // the warp's second batch of rows, towards L2 (one 128-byte line per lane: row lane / 4, line
  // lane % 4), so that its loads after the first batch are L2 hits
  {
    const float* Sb2 = S + (size_t)(warp * DF_ROWS + (DF_THREADS / 32) * DF_ROWS) * DF_D;
    asm volatile("prefetch.global.L2 [%0];" ::"l"(Sb2 + (lane >> 2) * DF_D + 32 * (lane & 3)));
  }

  // the gate of the output norm, requested early as well
  const float zv = tid < DF_D ? to_f(reinterpret_cast<const T*>(P.z)[(int64_t)nh * DF_D + tid])
                              : 0.0f;

  // ---- conv + SiLU: threads 0..127 own q channel j and v channel j, threads 128..255 k channel j
  const T* x = reinterpret_cast<const T*>(P.mix) + (int64_t)n * P.C;
  const float* cs_in = P.cs_in + (int64_t)n * P.C * (P.K - 1);
  float* cs_out = P.cs_out + (int64_t)n * P.C * (P.K - 1);
  const int j = tid & (DF_D - 1);
  const bool qk_owner = (h % G) == 0;  // one v-head per k-head advances the q/k history
  // threads < 128: q channel j and v channel j; threads >= 128: k channel j
  const int64_t c_qk = tid < DF_D ? (int64_t)hk * DF_D + j : (int64_t)(P.Hk + hk) * DF_D + j;
  const int64_t c_v = 2 * (int64_t)P.Hk * DF_D + (int64_t)h * DF_D + j;
  ConvIn in_qk, in_v;
  conv_load(in_qk, x, P.conv_w, P.conv_bias, P.K, c_qk, cs_in);
  if (tid < DF_D) conv_load(in_v, x, P.conv_w, P.conv_bias, P.K, c_v, cs_in);
  const float qk = conv_finish(in_qk, P.K, c_qk, cs_out, qk_owner);  // q or k before the norm
  if (tid < DF_D) v_s[j] = conv_finish(in_v, P.K, c_v, cs_out, true);
  // per-head L2 norm of q (warps 0-3) and k (warps 4-7)
  const float ss = dwarp_sum(qk * qk);
  if (lane == 0) red[warp] = ss;
  if (tid == 0) {
    const float av = to_f(reinterpret_cast<const T*>(P.a)[nh]);
    const float bv = to_f(reinterpret_cast<const T*>(P.b)[nh]);
    gate_s[0] = sigmoidf_(bv);                                                // beta
    gate_s[1] = expf(-expf(__ldg(P.A_log + h)) * softplusf_(av + __ldg(P.dt_bias + h)));  // e^g
  }
  __syncthreads();
  {
    const int g0 = tid < DF_D ? 0 : 4;
    const float tot = red[g0] + red[g0 + 1] + red[g0 + 2] + red[g0 + 3];
    const float inv = rsqrtf(tot + P.l2_eps);
    if (tid < DF_D) q_s[j] = qk * inv; else k_s[j] = qk * inv;
  }
  __syncthreads();

  // ---- the recurrent step, row by row (recurrent.cu)
  const float b = gate_s[0], a = gate_s[1];
  const float4 k4 = reinterpret_cast<const float4*>(k_s)[lane];
  const float4 q4 = reinterpret_cast<const float4*>(q_s)[lane];
  const float kq = dwarp_sum(k4.x * q4.x + k4.y * q4.y + k4.z * q4.z + k4.w * q4.w);
  float oss = 0.0f;  // this warp's share of sum(o^2) for the norm (the same in every lane)
  for (int base = warp * DF_ROWS; base < DF_D; base += (DF_THREADS / 32) * DF_ROWS) {
    if (base != warp * DF_ROWS) {
      const float* Sb = S + (size_t)base * DF_D;
#pragma unroll
      for (int u = 0; u < DF_ROWS; ++u)
        s[u] = __ldcs(reinterpret_cast<const float4*>(Sb + u * DF_D) + lane);
    }
    float sk[DF_ROWS], sq[DF_ROWS];
#pragma unroll
    for (int u = 0; u < DF_ROWS; ++u) {
      sk[u] = dwarp_sum(s[u].x * k4.x + s[u].y * k4.y + s[u].z * k4.z + s[u].w * k4.w);
      sq[u] = dwarp_sum(s[u].x * q4.x + s[u].y * q4.y + s[u].z * q4.z + s[u].w * q4.w);
    }
#pragma unroll
    for (int u = 0; u < DF_ROWS; ++u) {
      const int r = base + u;
      const float uj = b * (v_s[r] - a * sk[u]);
      float4 o4;
      o4.x = fmaf(a, s[u].x, uj * k4.x);
      o4.y = fmaf(a, s[u].y, uj * k4.y);
      o4.z = fmaf(a, s[u].z, uj * k4.z);
      o4.w = fmaf(a, s[u].w, uj * k4.w);
      __stcs(reinterpret_cast<float4*>(S + (size_t)r * DF_D) + lane, o4);
      const float o = P.scale * fmaf(a, sq[u], uj * kq);  // uniform across the warp
      oss = fmaf(o, o, oss);
      if (lane == u) o_s[r] = o;
    }
  }
  if (lane == 0) red[8 + warp] = oss;
  __syncthreads();

  // ---- gated RMSNorm of the head's output: y = o rsqrt(mean o^2 + eps) (1 + w) silu(z)
  if (tid < DF_D) {
    const float tot = ((red[8] + red[9]) + (red[10] + red[11])) +
                      ((red[12] + red[13]) + (red[14] + red[15]));
    const float inv = rsqrtf(tot * (1.0f / DF_D) + P.norm_eps);
    const float yv = o_s[tid] * inv * (1.0f + __ldg(P.norm_w + tid)) * siluf_(zv);
    reinterpret_cast<T*>(P.y)[(int64_t)nh * DF_D + tid] = from_f<T>(yv);
  }
}

// The same step with both v-heads of a k-head in one block (Hv = 2 Hk): the q/k conv and norms
// are done once for the pair, and the prologue is spread over twice the state bytes.  Threads
// 0..127 own q channel j and v channel j of the first head, threads 128..255 k channel j and v
// channel j of the second; warps 0-3 update the first head's rows, warps 4-7 the second's, each
// 32 rows in four batches of 8.
template <typename T>
__global__ void __launch_bounds__(DF_THREADS, 3) decode_fused_pair_kernel(const DecodeParams P) {
  __shared__ float q_s[DF_D], k_s[DF_D], v_s[2][DF_D], o_s[2][DF_D];
  __shared__ float red[16];
  __shared__ float gate_s[2][2];
  const int nk = blockIdx.x;  // n * Hk + hk
  const int n = nk / P.Hk, hk = nk - n * P.Hk;
  const int64_t nh0 = (int64_t)n * P.Hv + 2 * hk;  // the pair's first v-head (n, 2 hk)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int hw = warp >> 2;  // the head whose rows this warp updates
  float* S = P.state + (nh0 + hw) * DF_D * DF_D;
  constexpr int kBatches = DF_D / (4 * DF_ROWS);  // 4 batches of 8 rows per warp
  const int row0 = DF_ROWS * (warp & 3);           // batch b: rows row0 + 32 b .. + 7

  // ---- the first batch of rows in flight before the prologue, the others towards L2
  float4 s[DF_ROWS];
#pragma unroll
  for (int u = 0; u < DF_ROWS; ++u)
    s[u] = __ldcs(reinterpret_cast<const float4*>(S + (size_t)(row0 + u) * DF_D) + lane);
#pragma unroll
  for (int b = 1; b < kBatches; ++b)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(S + (size_t)(row0 + 32 * b + (lane >> 2)) * DF_D +
                                                  32 * (lane & 3)));
  // z of both heads (contiguous)
  const float zv = to_f(reinterpret_cast<const T*>(P.z)[nh0 * DF_D + tid]);

  // ---- conv + SiLU
  const T* x = reinterpret_cast<const T*>(P.mix) + (int64_t)n * P.C;
  const float* cs_in = P.cs_in + (int64_t)n * P.C * (P.K - 1);
  float* cs_out = P.cs_out + (int64_t)n * P.C * (P.K - 1);
  const int j = tid & (DF_D - 1), hv = tid >> 7;
  const int64_t c_qk = hv == 0 ? (int64_t)hk * DF_D + j : (int64_t)(P.Hk + hk) * DF_D + j;
  const int64_t c_v = 2 * (int64_t)P.Hk * DF_D + (2 * hk + hv) * (int64_t)DF_D + j;
  ConvIn in_qk, in_v;
  conv_load(in_qk, x, P.conv_w, P.conv_bias, P.K, c_qk, cs_in);
  conv_load(in_v, x, P.conv_w, P.conv_bias, P.K, c_v, cs_in);
  const float qk = conv_finish(in_qk, P.K, c_qk, cs_out, true);  // q or k before the norm
  v_s[hv][j] = conv_finish(in_v, P.K, c_v, cs_out, true);
  const float ss = dwarp_sum(qk * qk);
  if (lane == 0) red[warp] = ss;
  if (j == 0) {  // threads 0 and 128: the gates of their head
    const int h = 2 * hk + hv;
    const float av = to_f(reinterpret_cast<const T*>(P.a)[nh0 + hv]);
    const float bv = to_f(reinterpret_cast<const T*>(P.b)[nh0 + hv]);
    gate_s[hv][0] = sigmoidf_(bv);
    gate_s[hv][1] = expf(-expf(__ldg(P.A_log + h)) * softplusf_(av + __ldg(P.dt_bias + h)));
  }
  __syncthreads();
  {
    const int g0 = hv == 0 ? 0 : 4;
    const float tot = red[g0] + red[g0 + 1] + red[g0 + 2] + red[g0 + 3];
    const float inv = rsqrtf(tot + P.l2_eps);
    if (hv == 0) q_s[j] = qk * inv; else k_s[j] = qk * inv;
  }
  __syncthreads();

  // ---- the recurrent step of this warp's head, four batches of 8 rows
  const float b = gate_s[hw][0], a = gate_s[hw][1];
  const float4 k4 = reinterpret_cast<const float4*>(k_s)[lane];
  const float4 q4 = reinterpret_cast<const float4*>(q_s)[lane];
  const float kq = dwarp_sum(k4.x * q4.x + k4.y * q4.y + k4.z * q4.z + k4.w * q4.w);
  float oss = 0.0f;
#pragma unroll 1
  for (int bt = 0; bt < kBatches; ++bt) {
    const int base = row0 + 32 * bt;
    if (bt > 0) {
#pragma unroll
      for (int u = 0; u < DF_ROWS; ++u)
        s[u] = __ldcs(reinterpret_cast<const float4*>(S + (size_t)(base + u) * DF_D) + lane);
    }
    float sk[DF_ROWS], sq[DF_ROWS];
#pragma unroll
    for (int u = 0; u < DF_ROWS; ++u) {
      sk[u] = dwarp_sum(s[u].x * k4.x + s[u].y * k4.y + s[u].z * k4.z + s[u].w * k4.w);
      sq[u] = dwarp_sum(s[u].x * q4.x + s[u].y * q4.y + s[u].z * q4.z + s[u].w * q4.w);
    }
#pragma unroll
    for (int u = 0; u < DF_ROWS; ++u) {
      const int r = base + u;
      const float uj = b * (v_s[hw][r] - a * sk[u]);
      float4 o4;
      o4.x = fmaf(a, s[u].x, uj * k4.x);
      o4.y = fmaf(a, s[u].y, uj * k4.y);
      o4.z = fmaf(a, s[u].z, uj * k4.z);
      o4.w = fmaf(a, s[u].w, uj * k4.w);
      __stcs(reinterpret_cast<float4*>(S + (size_t)r * DF_D) + lane, o4);
      const float o = P.scale * fmaf(a, sq[u], uj * kq);  // uniform across the warp
      oss = fmaf(o, o, oss);
      if (lane == u) o_s[hw][r] = o;
    }
  }
  if (lane == 0) red[8 + warp] = oss;
  __syncthreads();

  // ---- gated RMSNorm of each head's output (thread: head hv, column j)
  {
    const int r0 = 8 + 4 * hv;
    const float tot = (red[r0] + red[r0 + 1]) + (red[r0 + 2] + red[r0 + 3]);
    const float inv = rsqrtf(tot * (1.0f / DF_D) + P.norm_eps);
    const float yv = o_s[hv][j] * inv * (1.0f + __ldg(P.norm_w + j)) * siluf_(zv);
    reinterpret_cast<T*>(P.y)[nh0 * DF_D + tid] = from_f<T>(yv);
  }
}

}  // namespace

cudaError_t launch_decode_fused(const void* mix, const void* a, const void* b, const void* z,
                                gdn_dtype dt, const float* conv_w, const float* conv_bias, int K,
                                const float* cs_in, float* cs_out, const float* A_log,
                                const float* dt_bias, const float* norm_w, float l2_eps,
                                float norm_eps, float scale, float* state, int N, int Hk, int Hv,
                                void* y, cudaStream_t s) {
  const int64_t blocks = (int64_t)N * Hv;
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7fffffff) return cudaErrorInvalidConfiguration;
  DecodeParams p;
  p.mix = mix;
  p.a = a;
  p.b = b;
  p.z = z;
  p.conv_w = conv_w;
  p.conv_bias = conv_bias;
  p.cs_in = cs_in;
  p.cs_out = cs_out;
  p.A_log = A_log;
  p.dt_bias = dt_bias;
  p.norm_w = norm_w;
  p.state = state;
  p.y = y;
  p.l2_eps = l2_eps;
  p.norm_eps = norm_eps;
  p.scale = scale;
  p.K = K;
  p.Hk = Hk;
  p.Hv = Hv;
  p.C = 2 * (int64_t)Hk * DF_D + (int64_t)Hv * DF_D;
  if (Hv == 2 * Hk) {  // both v-heads of a k-head in one block
    const unsigned pairs = (unsigned)(blocks / 2);
    if (dt == GDN_BF16)
      decode_fused_pair_kernel<__nv_bfloat16><<<pairs, DF_THREADS, 0, s>>>(p);
    else
      decode_fused_pair_kernel<float><<<pairs, DF_THREADS, 0, s>>>(p);
  } else if (dt == GDN_BF16) {
    decode_fused_kernel<__nv_bfloat16><<<(unsigned)blocks, DF_THREADS, 0, s>>>(p);
  } else {
    decode_fused_kernel<float><<<(unsigned)blocks, DF_THREADS, 0, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace gdn
