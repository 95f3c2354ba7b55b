// rmsnorm.cu -- zero-centred RMSNorm of the core output, gated by silu(z).
//
//   y[r,j] = x[r,j] * rsqrt(mean_j x[r,.]^2 + eps) * (1 + w[j]) * silu(z[r,j])
//
// Sources: "解密Qwen3-Next的Gated DeltaNet：如何用75%混合层实现长文本高效推理" §3.2 (weight
// stored zero-centred and used as 1 + w, normalisation in float) and "Qwen3.5 Gated DeltaNet
// 核心机制解析", output section (the norm of core_attn_out fuses the z gate, SwiGLU-like).
//
// HBM-bound: reads x and z, writes y, each once (3 * dim * elem bytes per row).  dim / 8 threads
// share a row (8 elements = one 16-byte bf16 transaction each); the row's sum of squares is a
// shuffle reduction inside that lane group.
#include "gdn_internal.cuh"

namespace gdn {

template <typename T, int TPR>
__global__ void __launch_bounds__(256) rmsnorm_gated_kernel(const T* __restrict__ x,
                                                            const T* __restrict__ z,
                                                            const float* __restrict__ w,
                                                            float eps, int64_t rows,
                                                            T* __restrict__ y) {
  constexpr int DIM = TPR * 8;
  constexpr int ROWS_PER_BLOCK = 256 / TPR;
  const int sub = threadIdx.x % TPR;
  const int64_t row0 = (int64_t)blockIdx.x * ROWS_PER_BLOCK + threadIdx.x / TPR;
  float wv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) wv[i] = 1.0f + __ldg(w + sub * 8 + i);
  const int64_t rstride = (int64_t)gridDim.x * ROWS_PER_BLOCK;
  for (int64_t r = row0; r - threadIdx.x / TPR < rows; r += rstride) {
    const bool live = r < rows;
    float xv[8], zv[8];
    float ss = 0.0f;
    if (live) {
      load8(x + r * DIM + sub * 8, xv);
      load8(z + r * DIM + sub * 8, zv);
#pragma unroll
      for (int i = 0; i < 8; ++i) ss = fmaf(xv[i], xv[i], ss);
    }
#pragma unroll
    for (int o = TPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (live) {
      const float inv = rsqrtf(ss * (1.0f / DIM) + eps);
      float yv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) yv[i] = xv[i] * inv * wv[i] * silu_fast(zv[i]);
      store8(y + r * DIM + sub * 8, yv);
    }
  }
}

template <typename T>
static cudaError_t launch_rmsnorm_t(const T* x, const T* z, const float* w, float eps,
                                    int64_t rows, int dim, T* y, cudaStream_t s) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int tpr = dim / 8;
  const int64_t rpb = 256 / tpr;
  int64_t blocks = (rows + rpb - 1) / rpb;
  const int64_t cap = (int64_t)sms * 8;
  if (blocks > cap) blocks = cap;
  switch (tpr) {
#define GDN_RMS_CASE(N) \
  case N: rmsnorm_gated_kernel<T, N><<<(unsigned)blocks, 256, 0, s>>>(x, z, w, eps, rows, y); break;
    GDN_RMS_CASE(1)
    GDN_RMS_CASE(2)
    GDN_RMS_CASE(4)
    GDN_RMS_CASE(8)
    GDN_RMS_CASE(16)
    GDN_RMS_CASE(32)
#undef GDN_RMS_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_rmsnorm(const void* x, const void* z, gdn_dtype dt, const float* w, float eps,
                           int64_t rows, int dim, void* y, cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  if (dt == GDN_BF16)
    return launch_rmsnorm_t((const __nv_bfloat16*)x, (const __nv_bfloat16*)z, w, eps, rows, dim,
                            (__nv_bfloat16*)y, s);
  return launch_rmsnorm_t((const float*)x, (const float*)z, w, eps, rows, dim, (float*)y, s);
}

}  // namespace gdn
