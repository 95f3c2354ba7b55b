// chunk_tm.cuh -- shared layout of the two-kernel tensor-core prefill (bf16, dk = dv = 128,
// chunks of 64 tokens): the prep kernel (chunk_prep.cu) writes, per (chunk, v-head), the
// state-independent operands of the chunk into the caller's workspace; the chain kernel
// (chunk_chain.cu) streams them in with TMA while it carries the state from chunk to chunk.
//
// Workspace (from its 256-byte-aligned base):
//   [0, 1024)                 status word (first int) and padding
//   TP  [slots][Hv][128][64]  bf16: rows 0..63 T' = (I + A)^{-1} diag(beta), rows 64..127 the
//                             decay-masked P = e^{gamma_r - gamma_s} q_r.k_s (s <= r); rows are
//                             128 bytes, loaded by the chain as one 128-byte-swizzled tile
//   GD  [slots][Hv][128]      fp32: Gamma_r = e^{gamma_r} (64), then d_s = e^{gamma_63 - gamma_s}
//                             (64), gamma the in-chunk cumulative log-decay (zero past the
//                             sequence end, so gamma_63 is the chunk's total log-decay)
// A "slot" is the ordinal of a chunk among all chunks of all sequences, in sequence order; there
// are at most ceil(B*T / 64) + N of them.
#pragma once

#include <stdint.h>

namespace gdn {
namespace tm {

constexpr int C = 64;                  // chunk length
constexpr int D = 128;                 // dk = dv
constexpr uint32_t TP_BYTES = 16384;   // [T'; P] per (slot, v-head)
constexpr uint32_t GD_BYTES = 512;     // Gamma, d per (slot, v-head)
constexpr size_t HEADER_BYTES = 1024;  // status word + padding

__host__ __device__ inline int64_t max_slots(int N, int64_t n_tok) {
  return (n_tok + C - 1) / C + N;
}

__host__ __device__ inline size_t tp_offset() { return HEADER_BYTES; }

__host__ __device__ inline size_t gd_offset(int N, int64_t n_tok, int Hv) {
  return HEADER_BYTES + (size_t)max_slots(N, n_tok) * Hv * TP_BYTES;
}

__host__ __device__ inline size_t workspace_bytes(int N, int64_t n_tok, int Hv) {
  return gd_offset(N, n_tok, Hv) + (size_t)max_slots(N, n_tok) * Hv * GD_BYTES;
}

// Sequence n's token range [s_beg, s_end) and the slot of its first chunk.  Returns false for a
// malformed cu_seqlens (a range outside [0, T] or decreasing) met up to sequence n, in which case
// nothing may be read through it.  O(n) reads of cu_seqlens.
__device__ __forceinline__ bool seq_chunks(const int32_t* cu, int64_t T, int n, int64_t& s_beg,
                                           int64_t& s_end, int64_t& slot0) {
  if (!cu) {
    const int64_t per = (T + C - 1) / C;
    s_beg = (int64_t)n * T;
    s_end = s_beg + T;
    slot0 = (int64_t)n * per;
    return true;
  }
  int64_t base = 0;
  for (int m = 0; m < n; ++m) {
    const int64_t a = cu[m], b = cu[m + 1];
    if (a < 0 || b < a || b > T) return false;
    base += (b - a + C - 1) / C;
  }
  s_beg = cu[n];
  s_end = cu[n + 1];
  if (s_beg < 0 || s_end < s_beg || s_end > T) return false;
  slot0 = base;
  return true;
}

}  // namespace tm
}  // namespace gdn
