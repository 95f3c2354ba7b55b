// recurrent.cu -- one-token decode step of the gated delta rule, state updated in place.
//
// Source: recurrent mode of "解密Qwen3-Next的Gated DeltaNet：如何用75%混合层实现长文本高效推理"
// §2.2 (recurrent_gated_delta_rule(..., initial_state=cached_state) -> (out, new_state)) and
// "Qwen3.5 Gated DeltaNet 核心机制解析" (recurrent path when the cache is valid and L = 1).
//
// Per (sequence, v-head), with a = exp(g), each value row j of S (dv x dk, fp32) evolves on its own:
//     sk_j = S[j,:].k      sq_j = S[j,:].q      u_j = beta (v_j - a sk_j)
//     S'[j,:] = a S[j,:] + u_j k^T                o_j = scale (a sq_j + u_j (k.q))
// which is S' = a S (I - beta k k^T) + beta v k^T and o = scale S' q.
//
// HBM-bound (about 0.9 flop per byte): the whole state is read once and written once per step.
// A warp owns 8 consecutive rows (4 KB); each lane holds 4 consecutive columns of a row as a
// float4, so a row is one 512-byte coalesced transaction per warp.  All 8 rows' loads are issued
// before any reduction, giving 32 KB in flight per 256-thread block; the state is touched exactly
// once, so loads and stores carry the evict-first (.cs) hint.
#include "gdn_internal.cuh"

namespace gdn {

constexpr int REC_THREADS = 256;
constexpr int REC_ROWS = 8;  // rows per warp per batch

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <typename T>
__global__ void __launch_bounds__(REC_THREADS, 3) recurrent_step_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const float* __restrict__ g, const float* __restrict__ beta, float scale,
    float* __restrict__ state, int Hk, int Hv, int dv, T* __restrict__ out) {
  constexpr int DK = 128;
  const int nh = blockIdx.x;  // n * Hv + h
  const int n = nh / Hv, h = nh - n * Hv;
  const int hk = h / (Hv / Hk);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  // the warp's first two batches of state rows are requested towards L2 before the q/k/gate
  // round trip (one 128-byte line per lane: row lane / 4 of the batch, line lane % 4)
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int row = warp * REC_ROWS + i * (REC_THREADS / 32) * REC_ROWS + (lane >> 2);
    if (row < dv)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(state + ((int64_t)nh * dv + row) * DK +
                                                      32 * (lane & 3)));
  }
  float k4[4], q4[4];
  load4(k + ((int64_t)n * Hk + hk) * DK + 4 * lane, k4);
  load4(q + ((int64_t)n * Hk + hk) * DK + 4 * lane, q4);
  const float kq = warp_sum(k4[0] * q4[0] + k4[1] * q4[1] + k4[2] * q4[2] + k4[3] * q4[3]);
  const float a = expf(__ldg(g + nh));
  const float b = __ldg(beta + nh);
  float* S = state + (int64_t)nh * dv * DK;
  const T* vrow = v + (int64_t)nh * dv;
  T* orow = out + (int64_t)nh * dv;

  // dv is a multiple of REC_ROWS (checked on the host), so a batch is either fully in range or
  // not started.
  for (int base = warp * REC_ROWS; base < dv; base += (REC_THREADS / 32) * REC_ROWS) {
    const float* Sb = S + (size_t)base * DK;
    float4 s[REC_ROWS];
#pragma unroll
    for (int u = 0; u < REC_ROWS; ++u) s[u] = __ldcs(reinterpret_cast<const float4*>(Sb + u * DK) + lane);
    float sk[REC_ROWS], sq[REC_ROWS];
#pragma unroll
    for (int u = 0; u < REC_ROWS; ++u) {
      sk[u] = warp_sum(s[u].x * k4[0] + s[u].y * k4[1] + s[u].z * k4[2] + s[u].w * k4[3]);
      sq[u] = warp_sum(s[u].x * q4[0] + s[u].y * q4[1] + s[u].z * q4[2] + s[u].w * q4[3]);
    }
#pragma unroll
    for (int u = 0; u < REC_ROWS; ++u) {
      const int j = base + u;
      const float uj = b * (to_f(vrow[j]) - a * sk[u]);
      float4 o4;
      o4.x = fmaf(a, s[u].x, uj * k4[0]);
      o4.y = fmaf(a, s[u].y, uj * k4[1]);
      o4.z = fmaf(a, s[u].z, uj * k4[2]);
      o4.w = fmaf(a, s[u].w, uj * k4[3]);
      __stcs(reinterpret_cast<float4*>(S + (size_t)j * DK) + lane, o4);
      if (lane == u) orow[j] = from_f<T>(scale * fmaf(a, sq[u], uj * kq));
    }
  }
}

cudaError_t launch_recurrent(const void* q, const void* k, const void* v, const float* g,
                             const float* beta, gdn_dtype dt, float scale, float* state, int N,
                             int Hk, int Hv, int dk, int dv, void* out, cudaStream_t s) {
  (void)dk;
  const int64_t blocks = (int64_t)N * Hv;
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7fffffff) return cudaErrorInvalidConfiguration;
  if (dt == GDN_BF16)
    recurrent_step_kernel<__nv_bfloat16><<<(unsigned)blocks, REC_THREADS, 0, s>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, g, beta, scale,
        state, Hk, Hv, dv, (__nv_bfloat16*)out);
  else
    recurrent_step_kernel<float><<<(unsigned)blocks, REC_THREADS, 0, s>>>(
        (const float*)q, (const float*)k, (const float*)v, g, beta, scale, state, Hk, Hv, dv,
        (float*)out);
  return cudaGetLastError();
}

}  // namespace gdn
