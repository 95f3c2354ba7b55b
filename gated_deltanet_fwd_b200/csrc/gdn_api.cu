// gdn_api.cu -- the exported C ABI (include/gdn.h): host-side argument checks, then one launch.
//
// Every check happens before anything is enqueued, so a rejected call leaves the stream
// untouched.  Device-side faults are reported through the workspace status word (chunk prefill)
// and never trap.
#include <stdio.h>

#include <nvtx3/nvToolsExt.h>

#include "chunk_tm.cuh"
#include "gdn_internal.cuh"

using namespace gdn;

namespace {

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// An NVTX range named after the ABI call for the duration of its host side (argument checks and
// launches), so that a profiler's timeline shows which call enqueued which kernels.  Without an
// attached tool the push and pop are no-ops.
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange&) = delete;
  CallRange& operator=(const CallRange&) = delete;
};

inline bool bad_dtype(gdn_dtype d) { return d != GDN_BF16 && d != GDN_F32; }

inline gdn_status from_cuda(cudaError_t e) { return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA; }

// Pointers that must be present and 16-byte aligned.
inline bool ptr_ok(const void* p) { return p != nullptr && aligned16(p); }

constexpr size_t kStatusBytes = 256;  // status word + padding to keep the workspace aligned

// SM count of the current device (148 if it cannot be read): sets the scan's segment length
int sm_count() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 148;
  return sms;
}
// The two-kernel tensor-core prefill (bf16, dk = dv = 128, chunk 64) when the workspace has room
// for it: with room for the scan's states the planner picks a segment length (or none) and the
// call runs prep, phase 1, prefix, phase 3; with room only for the per-chunk operands, prep and one
// chain per (sequence, v-head).  Returns false (nothing launched) when the workspace is too small.
bool run_two_kernel(const void* q, const void* k, const void* v, TokStrides ts, const float* g,
                    const float* beta, float scale, const float* S0, const int32_t* cu, int N,
                    int B, int64_t T, int Hk, int Hv, void* out, float* S_T, void* ws,
                    size_t ws_bytes, int* status, cudaStream_t s, const ChunkFusion& fuse,
                    cudaError_t* err) {
  const int64_t n_tok = (int64_t)B * T;
  const int sms = sm_count();
  const int64_t lseg = gdn::tm::scan_segment_tokens(n_tok, Hv, sms);
  cudaError_t e;
  if (lseg > 0 && ws_bytes >= gdn::tm::workspace_bytes_scan(N, n_tok, Hv, lseg)) {
    e = launch_scan_plan(cu, N, B, T, Hv, sms, lseg, ws, status, s);
    if (e == cudaSuccess)
      e = launch_chunk_prep(q, k, ts, g, beta, cu, N, B, T, Hk, Hv, ws, status, s, fuse);
    if (e == cudaSuccess)
      e = launch_chunk_chain(q, k, v, ts, scale, S0, cu, N, B, T, Hk, Hv, out, S_T, ws, 1, lseg,
                             status, s);
    if (e == cudaSuccess) e = launch_scan_prefix(cu, N, B, T, Hv, lseg, ws, status, s);
    if (e == cudaSuccess)
      e = launch_chunk_chain(q, k, v, ts, scale, S0, cu, N, B, T, Hk, Hv, out, S_T, ws, 3, lseg,
                             status, s);
  } else if (ws_bytes >= gdn::tm::workspace_bytes(N, n_tok, Hv)) {
    e = launch_chunk_prep(q, k, ts, g, beta, cu, N, B, T, Hk, Hv, ws, status, s, fuse);
    if (e == cudaSuccess)
      e = launch_chunk_chain(q, k, v, ts, scale, S0, cu, N, B, T, Hk, Hv, out, S_T, ws, 0, 0,
                             status, s);
  } else {
    return false;
  }
  *err = e;
  return true;
}

inline bool overlaps(const void* x, size_t xb, const void* y, size_t yb) {
  const char* a = (const char*)x;
  const char* b = (const char*)y;
  return a < b + yb && b < a + xb;
}

}  // namespace

extern "C" {

const char* gdn_status_string(gdn_status s) {
  switch (s) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG: invalid argument";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED: shape or dtype not implemented";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA: CUDA runtime or launch failure";
    case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT: a device-side wait ran out";
    case GDN_ERR_DEVICE_ARG: return "GDN_ERR_DEVICE_ARG: a kernel found a bad device argument";
  }
  return "unknown gdn_status";
}

gdn_status gdn_gates(const void* a, const void* b, gdn_dtype ab_dtype, const float* A_log,
                     const float* dt_bias, int64_t n_tok, int Hv, float* g, float* beta,
                     void* stream) {
  CallRange range_("gdn_gates");
  if (bad_dtype(ab_dtype) || n_tok < 0 || Hv < 1) return GDN_ERR_INVALID_ARG;
  if (n_tok == 0) return GDN_OK;
  if (!a || !b || !A_log || !dt_bias || !g || !beta) return GDN_ERR_INVALID_ARG;
  return from_cuda(launch_gates(a, b, ab_dtype, A_log, dt_bias, n_tok, Hv, g, beta,
                                as_stream(stream)));
}

gdn_status gdn_causal_conv1d_silu(const void* x, gdn_dtype dtype, const float* w,
                                  const float* bias, int B, int64_t T, int C, int K,
                                  const int32_t* cu_seqlens, int N, int n_l2norm_ch,
                                  int l2norm_group, float l2_eps, const float* conv_state_in,
                                  float* conv_state_out, void* y, void* stream) {
  CallRange range_("gdn_causal_conv1d_silu");
  if (bad_dtype(dtype) || B < 0 || T < 0 || C < 1 || K < 1 || N < 0) return GDN_ERR_INVALID_ARG;
  if (cu_seqlens ? (B != 1 && !(B == 0 && T == 0)) : (N != B)) return GDN_ERR_INVALID_ARG;
  if (n_l2norm_ch < 0 || n_l2norm_ch > C || l2norm_group < 0) return GDN_ERR_INVALID_ARG;
  if (!(l2_eps >= 0.0f)) return GDN_ERR_INVALID_ARG;
  if (K > 8 || C % 8 != 0) return GDN_ERR_UNSUPPORTED;
  if (l2norm_group != 0 && l2norm_group != 32 && l2norm_group != 64 && l2norm_group != 128 &&
      l2norm_group != 256)
    return GDN_ERR_UNSUPPORTED;
  if (l2norm_group == 0 ? n_l2norm_ch != 0 : n_l2norm_ch % l2norm_group != 0)
    return GDN_ERR_INVALID_ARG;
  const int64_t n_tok = (int64_t)B * T;
  if (cu_seqlens && n_tok > 0 && N < 1) return GDN_ERR_INVALID_ARG;
  if (n_tok == 0 && (N == 0 || !conv_state_out)) return GDN_OK;
  if (!w) return GDN_ERR_INVALID_ARG;
  if (n_tok > 0 && (!ptr_ok(x) || !ptr_ok(y))) return GDN_ERR_INVALID_ARG;
  if (n_tok > 0) {
    const size_t eb = dtype == GDN_BF16 ? 2 : 4;
    const char* xb = (const char*)x;
    const char* yb = (const char*)y;
    const size_t bytes = (size_t)n_tok * C * eb;
    if (xb < yb + bytes && yb < xb + bytes) return GDN_ERR_INVALID_ARG;  // x, y overlap
  }
  if (conv_state_in && conv_state_out && K > 1) {
    const size_t bytes = (size_t)N * C * (K - 1) * sizeof(float);
    const char* i0 = (const char*)conv_state_in;
    const char* o0 = (const char*)conv_state_out;
    if (i0 < o0 + bytes && o0 < i0 + bytes) return GDN_ERR_INVALID_ARG;
  }
  cudaStream_t s = as_stream(stream);
  if (n_tok == 0) {
    // every sequence is empty: the state passes through unchanged
    if (K == 1) return GDN_OK;
    const size_t bytes = (size_t)N * C * (K - 1) * sizeof(float);
    if (conv_state_in)
      return from_cuda(cudaMemcpyAsync(conv_state_out, conv_state_in, bytes,
                                       cudaMemcpyDeviceToDevice, s));
    return from_cuda(cudaMemsetAsync(conv_state_out, 0, bytes, s));
  }
  return from_cuda(launch_conv(x, dtype, w, bias, B, T, C, K, cu_seqlens, N, n_l2norm_ch,
                               l2norm_group, l2_eps, conv_state_in,
                               K > 1 ? conv_state_out : nullptr, y, s));
}

size_t gdn_chunk_fwd_workspace_size(int N, int B, int64_t T, int Hk, int Hv, int dk, int dv,
                                    int chunk) {
  (void)Hk;
  if (dk == gdn::tm::D && dv == gdn::tm::D && chunk == gdn::tm::C && N >= 0 && B >= 0 && T >= 0 &&
      Hv >= 1) {
    const int64_t n_tok = (int64_t)B * T;
    const int64_t lseg = gdn::tm::scan_segment_tokens(n_tok, Hv, sm_count());
    return (gdn::tm::workspace_bytes_scan(N, n_tok, Hv, lseg) + 255) & ~size_t(255);
  }
  return kStatusBytes;
}

gdn_status gdn_workspace_status(const void* workspace, void* stream, int* device_status) {
  if (!workspace || !device_status) return GDN_ERR_INVALID_ARG;
  int v = -1;
  cudaStream_t s = as_stream(stream);
  if (cudaMemcpyAsync(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return GDN_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return GDN_ERR_CUDA;
  *device_status = v;
  return GDN_OK;
}

gdn_status gdn_chunk_fwd_strided(const void* q, int64_t q_tok_stride, const void* k,
                                 int64_t k_tok_stride, const void* v, int64_t v_tok_stride,
                                 const float* g, const float* beta, gdn_dtype dtype, float scale,
                                 const float* initial_state, const int32_t* cu_seqlens, int N,
                                 int B, int64_t T, int Hk, int Hv, int dk, int dv, int chunk,
                                 void* out, float* final_state, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  CallRange range_("gdn_chunk_fwd_strided");
  if (bad_dtype(dtype) || N < 0 || B < 0 || T < 0 || Hk < 1 || Hv < 1 || dk < 1 || dv < 1)
    return GDN_ERR_INVALID_ARG;
  if (Hv % Hk != 0) return GDN_ERR_INVALID_ARG;
  if (cu_seqlens ? (B != 1) : (N != B)) return GDN_ERR_INVALID_ARG;
  if (!(scale == scale)) return GDN_ERR_INVALID_ARG;  // NaN
  if (dk % 16 != 0 || dv % 16 != 0 || dk > 128 || dv > 128) return GDN_ERR_UNSUPPORTED;
  if (chunk != 16 && chunk != 32 && chunk != 64) return GDN_ERR_UNSUPPORTED;
  // token strides: at least one token's heads, and whole 16-byte rows
  if (q_tok_stride < (int64_t)Hk * dk || k_tok_stride < (int64_t)Hk * dk ||
      v_tok_stride < (int64_t)Hv * dv || q_tok_stride % 8 || k_tok_stride % 8 ||
      v_tok_stride % 8)
    return GDN_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < kStatusBytes) return GDN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return GDN_ERR_INVALID_ARG;
  if (N == 0) return GDN_OK;
  const int64_t n_tok = (int64_t)B * T;
  if (n_tok > 0 && (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(g) || !ptr_ok(beta) ||
                    !ptr_ok(out)))
    return GDN_ERR_INVALID_ARG;
  if ((initial_state && !aligned16(initial_state)) || (final_state && !aligned16(final_state)))
    return GDN_ERR_INVALID_ARG;
  if (cu_seqlens && ((uintptr_t)cu_seqlens & 3u)) return GDN_ERR_INVALID_ARG;
  if (initial_state && final_state) {
    const size_t bytes = (size_t)N * Hv * dv * dk * sizeof(float);
    const char* i0 = (const char*)initial_state;
    const char* o0 = (const char*)final_state;
    if (i0 < o0 + bytes && o0 < i0 + bytes) return GDN_ERR_INVALID_ARG;
  }
  cudaStream_t s = as_stream(stream);
  int* status = reinterpret_cast<int*>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return GDN_ERR_CUDA;
  const TokStrides ts{q_tok_stride, k_tok_stride, v_tok_stride};
  cudaError_t e;
  if (dtype == GDN_BF16 && dk == gdn::tm::D && dv == gdn::tm::D && chunk == gdn::tm::C) {
    if (!run_two_kernel(q, k, v, ts, g, beta, scale, initial_state, cu_seqlens, N, B, T, Hk, Hv,
                        out, final_state, workspace, workspace_bytes, status, s, ChunkFusion(),
                        &e)) {
      e = launch_chunk_tc(q, k, v, ts, g, beta, scale, initial_state, cu_seqlens, N, B, T, Hk,
                          Hv, out, final_state, status, s);
    }
  } else
    e = launch_chunk_simt(q, k, v, ts, g, beta, dtype, scale, initial_state, cu_seqlens, N, B, T,
                          Hk, Hv, dk, dv, chunk, out, final_state, status, s);
  return from_cuda(e);
}

gdn_status gdn_chunk_fwd(const void* q, const void* k, const void* v, const float* g,
                         const float* beta, gdn_dtype dtype, float scale,
                         const float* initial_state, const int32_t* cu_seqlens, int N, int B,
                         int64_t T, int Hk, int Hv, int dk, int dv, int chunk, void* out,
                         float* final_state, void* workspace, size_t workspace_bytes,
                         void* stream) {
  return gdn_chunk_fwd_strided(q, (int64_t)Hk * dk, k, (int64_t)Hk * dk, v, (int64_t)Hv * dv, g,
                               beta, dtype, scale, initial_state, cu_seqlens, N, B, T, Hk, Hv, dk,
                               dv, chunk, out, final_state, workspace, workspace_bytes, stream);
}

gdn_status gdn_chunk_fwd_gated_norm(const void* q, int64_t q_tok_stride, const void* k,
                                    int64_t k_tok_stride, const void* v, int64_t v_tok_stride,
                                    const void* a, const void* b, const float* A_log,
                                    const float* dt_bias, const void* z, const float* norm_w,
                                    float norm_eps, gdn_dtype dtype, float scale,
                                    const float* initial_state, const int32_t* cu_seqlens, int N,
                                    int B, int64_t T, int Hk, int Hv, int dk, int dv, int chunk,
                                    void* y, float* final_state, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  CallRange range_("gdn_chunk_fwd_gated_norm");
  if (bad_dtype(dtype) || N < 0 || B < 0 || T < 0 || Hk < 1 || Hv < 1 || dk < 1 || dv < 1)
    return GDN_ERR_INVALID_ARG;
  if (Hv % Hk != 0) return GDN_ERR_INVALID_ARG;
  if (cu_seqlens ? (B != 1) : (N != B)) return GDN_ERR_INVALID_ARG;
  if (!(scale == scale) || !(norm_eps >= 0.0f)) return GDN_ERR_INVALID_ARG;
  if (q_tok_stride < (int64_t)Hk * dk || k_tok_stride < (int64_t)Hk * dk ||
      v_tok_stride < (int64_t)Hv * dv || q_tok_stride % 8 || k_tok_stride % 8 ||
      v_tok_stride % 8)
    return GDN_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < kStatusBytes) return GDN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return GDN_ERR_INVALID_ARG;
  if (dtype != GDN_BF16 || dk != gdn::tm::D || dv != gdn::tm::D || chunk != gdn::tm::C)
    return GDN_ERR_UNSUPPORTED;
  const int64_t n_tok = (int64_t)B * T;
  if (workspace_bytes < gdn::tm::workspace_bytes(N, n_tok, Hv)) return GDN_ERR_UNSUPPORTED;
  if (N == 0) return GDN_OK;
  if (n_tok > 0) {
    if (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(z) || !ptr_ok(y) || !ptr_ok(norm_w))
      return GDN_ERR_INVALID_ARG;
    if (!a || !b || !A_log || !dt_bias) return GDN_ERR_INVALID_ARG;
    const size_t zb = (size_t)n_tok * Hv * dv * 2;
    if (overlaps(y, zb, z, zb)) return GDN_ERR_INVALID_ARG;
  }
  if ((initial_state && !aligned16(initial_state)) || (final_state && !aligned16(final_state)))
    return GDN_ERR_INVALID_ARG;
  if (cu_seqlens && ((uintptr_t)cu_seqlens & 3u)) return GDN_ERR_INVALID_ARG;
  if (initial_state && final_state) {
    const size_t bytes = (size_t)N * Hv * dv * dk * sizeof(float);
    if (overlaps(initial_state, bytes, final_state, bytes)) return GDN_ERR_INVALID_ARG;
  }
  cudaStream_t s = as_stream(stream);
  int* status = reinterpret_cast<int*>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return GDN_ERR_CUDA;
  ChunkFusion fuse;
  fuse.a = reinterpret_cast<const __nv_bfloat16*>(a);
  fuse.b = reinterpret_cast<const __nv_bfloat16*>(b);
  fuse.A_log = A_log;
  fuse.dt_bias = dt_bias;
  const TokStrides ts{q_tok_stride, k_tok_stride, v_tok_stride};
  cudaError_t e = cudaSuccess;
  // the delta-rule output goes to y, and the gated RMSNorm runs over it in place
  run_two_kernel(q, k, v, ts, nullptr, nullptr, scale, initial_state, cu_seqlens, N, B, T, Hk,
                 Hv, y, final_state, workspace, workspace_bytes, status, s, fuse, &e);
  if (e == cudaSuccess && n_tok > 0)
    e = launch_rmsnorm(y, z, GDN_BF16, norm_w, norm_eps, n_tok * Hv, dv, y, s);
  return from_cuda(e);
}

gdn_status gdn_recurrent_step(const void* q, const void* k, const void* v, const float* g,
                              const float* beta, gdn_dtype dtype, float scale, float* state,
                              int N, int Hk, int Hv, int dk, int dv, void* out, void* stream) {
  CallRange range_("gdn_recurrent_step");
  if (bad_dtype(dtype) || N < 0 || Hk < 1 || Hv < 1 || dk < 1 || dv < 1)
    return GDN_ERR_INVALID_ARG;
  if (Hv % Hk != 0) return GDN_ERR_INVALID_ARG;
  if (!(scale == scale)) return GDN_ERR_INVALID_ARG;
  if (dk != 128 || dv % 8 != 0 || dv > 256) return GDN_ERR_UNSUPPORTED;
  if (N == 0) return GDN_OK;
  if (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(g) || !ptr_ok(beta) || !ptr_ok(state) ||
      !ptr_ok(out))
    return GDN_ERR_INVALID_ARG;
  return from_cuda(launch_recurrent(q, k, v, g, beta, dtype, scale, state, N, Hk, Hv, dk, dv, out,
                                    as_stream(stream)));
}

gdn_status gdn_decode_layer_step(const void* mix, const void* a, const void* b, const void* z,
                                 gdn_dtype dtype, const float* conv_w, const float* conv_bias,
                                 int K, const float* conv_state_in, float* conv_state_out,
                                 const float* A_log, const float* dt_bias, const float* norm_w,
                                 float l2_eps, float norm_eps, float scale, float* state, int N,
                                 int Hk, int Hv, int dk, int dv, void* y, void* stream) {
  CallRange range_("gdn_decode_layer_step");
  if (bad_dtype(dtype) || N < 0 || Hk < 1 || Hv < 1 || dk < 1 || dv < 1 || K < 1)
    return GDN_ERR_INVALID_ARG;
  if (Hv % Hk != 0) return GDN_ERR_INVALID_ARG;
  if (!(scale == scale) || !(l2_eps >= 0.0f) || !(norm_eps >= 0.0f)) return GDN_ERR_INVALID_ARG;
  if (dk != 128 || dv != 128 || K > 8) return GDN_ERR_UNSUPPORTED;
  if (N == 0) return GDN_OK;
  if (!ptr_ok(mix) || !a || !b || !ptr_ok(z) || !conv_w || !A_log || !dt_bias || !norm_w ||
      !ptr_ok(state) || !ptr_ok(y))
    return GDN_ERR_INVALID_ARG;
  const size_t C = 2 * (size_t)Hk * dk + (size_t)Hv * dv;
  if (K > 1) {
    if (!conv_state_in || !conv_state_out) return GDN_ERR_INVALID_ARG;
    const size_t bytes = (size_t)N * C * (K - 1) * sizeof(float);
    const char* i0 = (const char*)conv_state_in;
    const char* o0 = (const char*)conv_state_out;
    if (i0 < o0 + bytes && o0 < i0 + bytes) return GDN_ERR_INVALID_ARG;
  }
  return from_cuda(launch_decode_fused(mix, a, b, z, dtype, conv_w, conv_bias, K, conv_state_in,
                                       conv_state_out, A_log, dt_bias, norm_w, l2_eps, norm_eps,
                                       scale, state, N, Hk, Hv, y, as_stream(stream)));
}

gdn_status gdn_gated_rmsnorm(const void* x, const void* z, gdn_dtype dtype, const float* w,
                             float eps, int64_t n_rows, int dim, void* y, void* stream) {
  CallRange range_("gdn_gated_rmsnorm");
  if (bad_dtype(dtype) || n_rows < 0 || dim < 1 || !(eps >= 0.0f)) return GDN_ERR_INVALID_ARG;
  if (dim != 8 && dim != 16 && dim != 32 && dim != 64 && dim != 128 && dim != 256)
    return GDN_ERR_UNSUPPORTED;
  if (n_rows == 0) return GDN_OK;
  if (!ptr_ok(x) || !ptr_ok(z) || !ptr_ok(y) || !w) return GDN_ERR_INVALID_ARG;
  {
    const size_t bytes = (size_t)n_rows * dim * (dtype == GDN_BF16 ? 2 : 4);
    const char* zb = (const char*)z;
    const char* yb = (const char*)y;
    if (zb < yb + bytes && yb < zb + bytes) return GDN_ERR_INVALID_ARG;  // y may alias x only
  }
  return from_cuda(launch_rmsnorm(x, z, dtype, w, eps, n_rows, dim, y, as_stream(stream)));
}

}  // extern "C"
