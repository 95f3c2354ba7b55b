// gates.cu -- beta = sigmoid(b), g = -exp(A_log) * softplus(a + dt_bias), elementwise.
//
// Source: "Qwen3-Next大模型架构解析：混合注意力与MoE优化实践" §2.2 (gate generation in the
// Qwen3NextGatedDeltaNet forward sketch) and the flowchart of "Qwen3.5 Gated DeltaNet 核心机制解析"
// (b -> Sigmoid -> beta; a -> Softplus + dt_bias; A_log -> Exp and Neg; Mul -> g).
//
// HBM-bound: per (token, head) it reads a and b (2 or 4 bytes each) and writes g and beta
// (4 bytes each).  A grid-stride loop over 4-element groups with one block per SM slot.
#include "gdn_internal.cuh"

namespace gdn {

template <typename T>
__global__ void __launch_bounds__(256) gates_kernel(const T* __restrict__ a,
                                                    const T* __restrict__ b,
                                                    const float* __restrict__ A_log,
                                                    const float* __restrict__ dt_bias,
                                                    int64_t total, int Hv, float* __restrict__ g,
                                                    float* __restrict__ beta) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int h = (int)(i % Hv);
    const float av = to_f(a[i]) + __ldg(dt_bias + h);
    const float bv = to_f(b[i]);
    beta[i] = sigmoidf_(bv);
    g[i] = -expf(__ldg(A_log + h)) * softplusf_(av);
  }
}

cudaError_t launch_gates(const void* a, const void* b, gdn_dtype dt, const float* A_log,
                         const float* dt_bias, int64_t n_tok, int Hv, float* g, float* beta,
                         cudaStream_t s) {
  const int64_t total = n_tok * Hv;
  if (total == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = (int64_t)sms * 8;
  if (blocks > cap) blocks = cap;
  if (dt == GDN_BF16)
    gates_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(
        (const __nv_bfloat16*)a, (const __nv_bfloat16*)b, A_log, dt_bias, total, Hv, g, beta);
  else
    gates_kernel<float><<<(unsigned)blocks, 256, 0, s>>>((const float*)a, (const float*)b, A_log,
                                                         dt_bias, total, Hv, g, beta);
  return cudaGetLastError();
}

}  // namespace gdn
