// gdn_internal.cuh -- helpers shared by the libgdn kernels (device side) and the launchers'
// internal declarations.  Nothing here is exported.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn.h"

namespace gdn {

// ---------------------------------------------------------------- element I/O -------------
// Activations are bf16 or fp32; math is fp32.  Loads of 8 consecutive elements are one 16-byte
// transaction for bf16 and two for fp32.

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// 8 consecutive elements <-> 8 floats.  `p` must be 16-byte aligned.
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&f)[8]) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float (&f)[8]) {
  float4 a = reinterpret_cast<const float4*>(p)[0];
  float4 b = reinterpret_cast<const float4*>(p)[1];
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&f)[8]) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void store8(float* p, const float (&f)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
}

// Raw (still encoded) 8-element vectors, so loads can be issued early without holding 8 floats.
template <typename T>
struct Raw8;
template <>
struct Raw8<__nv_bfloat16> {
  uint4 u;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) {
    u = *reinterpret_cast<const uint4*>(p);
  }
  __device__ __forceinline__ void zero() { u = make_uint4(0, 0, 0, 0); }
  __device__ __forceinline__ void to_float(float (&f)[8]) const {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 t = __bfloat1622float2(h[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
};
template <>
struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = reinterpret_cast<const float4*>(p)[0];
    b = reinterpret_cast<const float4*>(p)[1];
  }
  __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ void to_float(float (&f)[8]) const {
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
};

// 4 consecutive elements -> 4 floats (8-byte bf16 load or one float4).
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float (&f)[4]) {
  uint2 u = *reinterpret_cast<const uint2*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
  float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
}
__device__ __forceinline__ void load4(const float* p, float (&f)[4]) {
  float4 a = *reinterpret_cast<const float4*>(p);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + expf(-x)); }
__device__ __forceinline__ float siluf_(float x) { return x / (1.0f + expf(-x)); }
// SiLU for kernels whose result is rounded to bf16: the fast exponential and division intrinsics
// (relative error ~1e-6, far below bf16's 2^-8) keep these HBM-bound kernels off the ALU roof.
// For x < -87 the exponential overflows to +inf and the quotient is the correct limit, -0.
__device__ __forceinline__ float silu_fast(float x) { return __fdividef(x, 1.0f + __expf(-x)); }
__device__ __forceinline__ float softplusf_(float x) {
  return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
}

// Device-side fault reporting: the first error wins; never traps.
__device__ __forceinline__ void report(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Sequence lookup for packed (varlen) token streams.  Returns the sequence that owns token t
// (cu[n] <= t < cu[n+1]); with cu == nullptr sequence n is batch row t / T.
__device__ __forceinline__ int seq_of_token(const int32_t* cu, int N, int64_t T, int64_t t) {
  if (!cu) return (int)(t / T);
  int lo = 0, hi = N - 1;  // last n with cu[n] <= t
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if ((int64_t)cu[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------- launchers ---------------
// Each returns cudaSuccess or the launch error; arguments were validated by the caller.

cudaError_t launch_gates(const void* a, const void* b, gdn_dtype dt, const float* A_log,
                         const float* dt_bias, int64_t n_tok, int Hv, float* g, float* beta,
                         cudaStream_t s);

cudaError_t launch_conv(const void* x, gdn_dtype dt, const float* w, const float* bias, int B,
                        int64_t T, int C, int K, const int32_t* cu, int N, int n_l2, int group,
                        float l2_eps, const float* cs_in, float* cs_out, void* y,
                        cudaStream_t s);

cudaError_t launch_rmsnorm(const void* x, const void* z, gdn_dtype dt, const float* w, float eps,
                           int64_t rows, int dim, void* y, cudaStream_t s);

cudaError_t launch_recurrent(const void* q, const void* k, const void* v, const float* g,
                             const float* beta, gdn_dtype dt, float scale, float* state, int N,
                             int Hk, int Hv, int dk, int dv, void* out, cudaStream_t s);

cudaError_t launch_decode_fused(const void* mix, const void* a, const void* b, const void* z,
                                gdn_dtype dt, const float* conv_w, const float* conv_bias, int K,
                                const float* cs_in, float* cs_out, const float* A_log,
                                const float* dt_bias, const float* norm_w, float l2_eps,
                                float norm_eps, float scale, float* state, int N, int Hk, int Hv,
                                void* y, cudaStream_t s);

// Element distances between consecutive tokens of q, k and v (dense: Hk*dk, Hk*dk, Hv*dv).
struct TokStrides {
  int64_t q, k, v;
};

// CUDA-core chunk path (any supported shape / dtype).
cudaError_t launch_chunk_simt(const void* q, const void* k, const void* v, TokStrides ts,
                              const float* g,
                              const float* beta, gdn_dtype dt, float scale, const float* S0,
                              const int32_t* cu, int N, int B, int64_t T, int Hk, int Hv, int dk,
                              int dv, int chunk, void* out, float* S_T, int* status,
                              cudaStream_t s);

// Optional fusions of the layer's neighbouring steps into the two-kernel tensor-core prefill: the
// gates computed from their pre-activations inside the prep kernel (a, b set), and the gated
// RMSNorm applied to the outputs in the chain's output epilogue (z set; `out` then receives y).
struct ChunkFusion {
  const __nv_bfloat16* a = nullptr;  // [tokens, Hv] gate pre-activations (fused gates when set)
  const __nv_bfloat16* b = nullptr;
  const float* A_log = nullptr;
  const float* dt_bias = nullptr;
};

// TMA tensor maps (tma_maps.cu), 128-byte swizzle, bf16:
//   make_tok_map:    [rows, heads, 128] with `tok_stride` elements between rows; box {64, 1, 64}
//   make_rows64_map: [rows, 64] dense;                                          box {64, box_rows}
bool make_tok_map(CUtensorMap* m, const void* base, int heads, int64_t rows, int64_t tok_stride);
bool make_rows64_map(CUtensorMap* m, const void* base, int64_t rows, uint32_t box_rows);

// Two-kernel tensor-core prefill (bf16, dk = dv = 128, chunk = 64): the parallel prep kernel,
// then the chain kernel.  `ws` holds at least tm::workspace_bytes(N, B*T, Hv) bytes.
cudaError_t launch_chunk_prep(const void* q, const void* k, TokStrides ts, const float* g,
                              const float* beta, const int32_t* cu, int N, int B, int64_t T,
                              int Hk, int Hv, void* ws, int* status, cudaStream_t s,
                              const ChunkFusion& fuse = ChunkFusion());
// phase 0: one chain per (sequence, v-head); phases 1 and 3 (with launch_scan_prefix between
// them): the intra-sequence scan with segments of lseg tokens (chunk_tm.cuh), for which `ws` holds
// at least tm::workspace_bytes_scan(N, B*T, Hv, lseg) bytes.
cudaError_t launch_chunk_chain(const void* q, const void* k, const void* v, TokStrides ts,
                               float scale, const float* S0, const int32_t* cu, int N, int B,
                               int64_t T, int Hk, int Hv, void* out, float* S_T, void* ws,
                               int phase, int64_t lseg, int* status, cudaStream_t s);
// One-thread planner: writes the call's segment length (0, lseg, 2 lseg or 4 lseg) into the
// workspace for the two chain phases and the prefix to read.
cudaError_t launch_scan_plan(const int32_t* cu, int N, int B, int64_t T, int Hv, int sms,
                             int64_t lseg, void* ws, int* status, cudaStream_t s);
cudaError_t launch_scan_prefix(const int32_t* cu, int N, int B, int64_t T, int Hv, int64_t lseg,
                               void* ws, int* status, cudaStream_t s);

// Tensor-core chunk path without scratch (one CTA pair per sequence and head): bf16,
// dk = dv = 128, chunk = 64.
cudaError_t launch_chunk_tc(const void* q, const void* k, const void* v, TokStrides ts,
                            const float* g,
                            const float* beta, float scale, const float* S0, const int32_t* cu,
                            int N, int B, int64_t T, int Hk, int Hv, void* out, float* S_T,
                            int* status, cudaStream_t s);

}  // namespace gdn
