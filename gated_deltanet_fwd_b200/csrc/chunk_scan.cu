// chunk_scan.cu -- the prefix step of the intra-sequence scan of the tensor-core prefill.
//
// Method: the state map of a stretch of tokens under the gated delta rule is affine,
// S_out = S_in M + B (M the product of the per-token transitions e^{g_t}(I - beta_t k_t k_t^T), B
// the state the stretch produces from a zero state), so a sequence split into segments can carry
// its state from segment to segment by composing those maps -- the state passing between calls of
// the chunked mode ("解密Qwen3-Next的Gated DeltaNet：如何用75%混合层实现长文本高效推理" §2.2, state
// carried through initial_state), applied inside one call.  After phase 1 of the chain kernel has
// produced SOUT (the state leaving segment 0) and BSEG / MSEG of every middle segment, this kernel
// walks each long sequence's segments in order:
//     SIN_1 = SOUT,     SIN_{k+1} = SIN_k M_k + B_k      (k = 1 .. nseg - 2)
// in fp32.  Rows of S are independent, so one CTA takes 16 rows of one (sequence, v-head).
#include "chunk_tm.cuh"
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int PX_THREADS = 256;
constexpr int PX_ROWS = 16;

__global__ void __launch_bounds__(PX_THREADS) scan_prefix_kernel(
    const int32_t* __restrict__ cu, int64_t T, int N, int Hv, int64_t lseg, int64_t max_segs,
    float* __restrict__ st, int* status) {
  extern __shared__ float px_smem[];
  float* Ms = px_smem;                 // M_k: 128 x 128
  float* Sr = Ms + tm::D * tm::D;      // 16 rows of the running state: 16 x 128
  const int n = blockIdx.x, h = blockIdx.y, r0 = PX_ROWS * blockIdx.z;
  const int tid = threadIdx.x;
  // this sequence's segment count and the global index of its first segment
  int64_t nseg = 0, seg0 = 0;
  for (int m = 0; m <= n; ++m) {
    int64_t a, b;
    if (cu) {
      a = cu[m];
      b = cu[m + 1];
      if (a < 0 || b < a || b > T) {
        if (tid == 0 && blockIdx.y == 0 && blockIdx.z == 0) report(status, GDN_ERR_DEVICE_ARG);
        return;
      }
    } else {
      a = (int64_t)m * T;
      b = a + T;
    }
    const int64_t ns = tm::seg_count(b - a, lseg);
    if (m < n) seg0 += ns; else nseg = ns;
  }
  if (nseg < 2) return;  // one chain: nothing to compose
  const size_t hs = tm::STATE_FLOATS;
  const float* sout = st + ((size_t)n * Hv + h) * hs;
  const float* bseg = st + (size_t)N * Hv * hs;
  const float* mseg = bseg + (size_t)max_segs * Hv * hs;
  float* sin_ = const_cast<float*>(mseg) + (size_t)max_segs * Hv * hs;

  for (int e = tid; e < PX_ROWS * tm::D; e += PX_THREADS)
    Sr[e] = sout[(size_t)(r0 + e / tm::D) * tm::D + (e % tm::D)];
  const int r = tid >> 4, c0 = 8 * (tid & 15);  // output row and its 8 columns
  for (int64_t k = 1; k < nseg; ++k) {
    const size_t g = ((size_t)(seg0 + k) * Hv + h) * hs;
    __syncthreads();  // Sr complete
    for (int e = tid; e < PX_ROWS * tm::D; e += PX_THREADS)
      sin_[g + (size_t)(r0 + e / tm::D) * tm::D + (e % tm::D)] = Sr[e];
    if (k == nseg - 1) break;
    // S <- S M_k + B_k on this block of rows
    for (int e = tid; e < tm::D * tm::D / 4; e += PX_THREADS)
      reinterpret_cast<float4*>(Ms)[e] = reinterpret_cast<const float4*>(mseg + g)[e];
    __syncthreads();
    float acc[8];
    {
      const float4* b4 = reinterpret_cast<const float4*>(bseg + g + (size_t)(r0 + r) * tm::D + c0);
      const float4 b0 = b4[0], b1 = b4[1];
      acc[0] = b0.x; acc[1] = b0.y; acc[2] = b0.z; acc[3] = b0.w;
      acc[4] = b1.x; acc[5] = b1.y; acc[6] = b1.z; acc[7] = b1.w;
    }
#pragma unroll 4
    for (int l = 0; l < tm::D; ++l) {
      const float sv = Sr[r * tm::D + l];
      const float4 m0 = *reinterpret_cast<const float4*>(Ms + l * tm::D + c0);
      const float4 m1 = *reinterpret_cast<const float4*>(Ms + l * tm::D + c0 + 4);
      acc[0] = fmaf(sv, m0.x, acc[0]); acc[1] = fmaf(sv, m0.y, acc[1]);
      acc[2] = fmaf(sv, m0.z, acc[2]); acc[3] = fmaf(sv, m0.w, acc[3]);
      acc[4] = fmaf(sv, m1.x, acc[4]); acc[5] = fmaf(sv, m1.y, acc[5]);
      acc[6] = fmaf(sv, m1.z, acc[6]); acc[7] = fmaf(sv, m1.w, acc[7]);
    }
    __syncthreads();  // every thread has read Sr and Ms
#pragma unroll
    for (int q = 0; q < 8; ++q) Sr[r * tm::D + c0 + q] = acc[q];
  }
}

}  // namespace

cudaError_t launch_scan_prefix(const int32_t* cu, int N, int B, int64_t T, int Hv, int64_t lseg,
                               void* ws, int* status, cudaStream_t s) {
  const int64_t n_tok = (int64_t)B * T;
  if (N == 0 || lseg <= 0) return cudaSuccess;
  if (N > 0x7fffffff || Hv > 65535) return cudaErrorInvalidConfiguration;
  float* st = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(ws) +
                                       tm::states_offset(N, n_tok, Hv));
  const size_t smem = (size_t)(tm::D * tm::D + PX_ROWS * tm::D) * sizeof(float);
  static bool attr_set = false;  // idempotent attribute; a benign race between host threads
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(scan_prefix_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  scan_prefix_kernel<<<dim3((unsigned)N, (unsigned)Hv, tm::D / PX_ROWS), PX_THREADS, smem, s>>>(
      cu, T, N, Hv, lseg, tm::max_segs(N, n_tok, lseg), st, status);
  return cudaGetLastError();
}

}  // namespace gdn
