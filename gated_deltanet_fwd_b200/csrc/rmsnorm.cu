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
// shuffle reduction inside that lane group.  Each thread keeps RMS_U rows' loads in flight.
#include "gdn_internal.cuh"

namespace gdn {

constexpr int RMS_U = 4;  // rows in flight per thread

template <typename T, int TPR>
__global__ void __launch_bounds__(256, 4) rmsnorm_gated_kernel(const T* __restrict__ x,
                                                            const T* __restrict__ z,
                                                            const float* __restrict__ w,
                                                            float eps, int64_t rows,
                                                            T* __restrict__ y) {
  constexpr int DIM = TPR * 8;
  constexpr int ROWS_PER_BLOCK = 256 / TPR;
  const int sub = threadIdx.x % TPR;
  const int rsub = threadIdx.x / TPR;
  float wv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) wv[i] = 1.0f + __ldg(w + sub * 8 + i);
  const int64_t rstride = (int64_t)gridDim.x * ROWS_PER_BLOCK;
  // RMS_U rows per thread per pass: all their loads are issued before any is used
  for (int64_t rb = (int64_t)blockIdx.x * ROWS_PER_BLOCK; rb < rows; rb += RMS_U * rstride) {
    Raw8<T> xr[RMS_U], zr[RMS_U];
#pragma unroll
    for (int u = 0; u < RMS_U; ++u) {
      const int64_t r = rb + u * rstride + rsub;
      if (r < rows) {
        xr[u].load(x + r * DIM + sub * 8);
        zr[u].load(z + r * DIM + sub * 8);
      } else {
        xr[u].zero();
        zr[u].zero();
      }
    }
#pragma unroll
    for (int u = 0; u < RMS_U; ++u) {
      const int64_t r = rb + u * rstride + rsub;
      float xv[8], zv[8];
      xr[u].to_float(xv);
      zr[u].to_float(zv);
      float ss = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) ss = fmaf(xv[i], xv[i], ss);
#pragma unroll
      for (int o = TPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (r < rows) {
        const float inv = rsqrtf(ss * (1.0f / DIM) + eps);
        float yv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) yv[i] = xv[i] * inv * wv[i] * silu_fast(zv[i]);
        store8(y + r * DIM + sub * 8, yv);
      }
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
  // enough blocks for one pass of RMS_U rows per thread, at most one wave of resident blocks
  int64_t blocks = (rows + rpb * RMS_U - 1) / (rpb * RMS_U);
  auto run = [&](auto kern) {
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, 0);
    const int64_t cap = (int64_t)sms * (per_sm > 0 ? per_sm : 1);
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    kern<<<(unsigned)blocks, 256, 0, s>>>(x, z, w, eps, rows, y);
  };
  switch (tpr) {
#define GDN_RMS_CASE(N) \
  case N: run(rmsnorm_gated_kernel<T, N>); break;
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
