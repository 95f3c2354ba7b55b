// chunk_tm.cuh -- shared layout of the two-kernel tensor-core prefill (bf16, dk = dv = 128,
// chunks of 64 tokens): the prep kernel (chunk_prep.cu) writes, per (chunk, v-head), the
// state-independent operands of the chunk into the caller's workspace; the chain kernel
// (chunk_chain.cu) streams them in with TMA while it carries the state from chunk to chunk.
//
// Workspace (from its 256-byte-aligned base):
//   [0, 1024)                 status word (first int), the scan's segment length (int64 at byte
//                             8, written on the device by the planner), padding
//   TP  [slots][Hv][128][64]  bf16: rows 0..63 T' = (I + A)^{-1} diag(beta), rows 64..127 the
//                             decay-masked P = e^{gamma_r - gamma_s} q_r.k_s (s <= r); rows are
//                             128 bytes, loaded by the chain as one 128-byte-swizzled tile
//   GD  [slots][Hv][128]      fp32: Gamma_r = e^{gamma_r} (64), then d_s = e^{gamma_63 - gamma_s}
//                             (64), gamma the in-chunk cumulative log-decay (zero past the
//                             sequence end, so gamma_63 is the chunk's total log-decay)
// A "slot" is the ordinal of a chunk among all chunks of all sequences, in sequence order; there
// are at most ceil(B*T / 64) + N of them.
//
// With room for them, four state arrays follow (the intra-sequence scan, below):
//   SOUT [N][Hv][128][128]          fp32: state leaving segment 0 of each sequence
//   BSEG, MSEG, SIN [segs][Hv][128][128] fp32: per segment, the state it produces from a zero
//                                   state, its transition (dk x dk), and its true entry state
//
// Intra-sequence scan.  The state map of a stretch of tokens is affine, S_out = S_in M + B, with
// M the product of the per-token transitions e^{g} (I - beta k k^T) and B the state the stretch
// produces from a zero state.  A sequence longer than two segments (lseg tokens each, a multiple
// of 64) is processed in three phases instead of one serial chain:
//   phase 1, all in parallel: segment 0 from the sequence's initial state (outputs, leaving state
//            SOUT), and for every middle segment k (1 .. nseg-2) its B (chain from a zero state,
//            no outputs) and its M (chain from the identity with v = 0, no outputs);
//   prefix:  SIN_1 = SOUT, SIN_{k+1} = SIN_k M_k + B_k;
//   phase 3, all in parallel: segments 1 .. nseg-1 from SIN_k (outputs; the last one leaves the
//            final state).
// The critical path is two segments instead of the whole sequence; the middle segments run three
// times.  Sequences of at most two segments (and every sequence when lseg is 0) run as one chain.
#pragma once

#include <stdint.h>

namespace gdn {
namespace tm {

constexpr int C = 64;                  // chunk length
constexpr int D = 128;                 // dk = dv
constexpr uint32_t TP_BYTES = 16384;   // [T'; P] per (slot, v-head)
constexpr uint32_t GD_BYTES = 512;     // Gamma, d per (slot, v-head)
constexpr size_t HEADER_BYTES = 1024;  // status word + padding
constexpr size_t PLAN_OFF = 8;         // int64 segment length chosen for the call (0: no scan)

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

// ---------------------------------------------------------------- intra-sequence scan ------

constexpr size_t STATE_FLOATS = (size_t)D * D;

__host__ __device__ inline int64_t max_segs(int N, int64_t n_tok, int64_t lseg) {
  return lseg > 0 ? n_tok / lseg + N : 0;
}

// byte offset of the state arrays (SOUT, BSEG, MSEG, SIN), right after the GD array
__host__ __device__ inline size_t states_offset(int N, int64_t n_tok, int Hv) {
  return workspace_bytes(N, n_tok, Hv);
}

__host__ __device__ inline size_t workspace_bytes_scan(int N, int64_t n_tok, int Hv, int64_t lseg) {
  return states_offset(N, n_tok, Hv) +
         ((size_t)N + 3 * (size_t)max_segs(N, n_tok, lseg)) * Hv * STATE_FLOATS * sizeof(float);
}

// Segment length for the scan: a power of two number of chunks near the work per SM if the
// chunk-heads of the whole call were spread evenly (at least 8 chunks); 0 for no scan.
inline int64_t scan_segment_tokens(int64_t n_tok, int Hv, int sms) {
  if (sms <= 0 || n_tok <= 0) return 0;
  const int64_t per_sm = ((n_tok + C - 1) / C) * Hv / sms;
  int64_t chunks = 8;
  while (chunks * 2 <= per_sm) chunks *= 2;
  return chunks * C;
}

enum UnitKind { U_MAIN0 = 0, U_BSEG = 1, U_MSEG = 2, U_MAINK = 3 };

__host__ __device__ inline int64_t seg_count(int64_t len, int64_t lseg) {
  if (len <= 0) return 0;
  if (lseg <= 0 || len <= 2 * lseg) return 1;
  return (len + lseg - 1) / lseg;
}

// units of one sequence (per v-head) in a phase: phases 0 (no scan) and 1 give segment 0 (also for
// an empty sequence) and two units per middle segment; phase 3 one unit per later segment
__host__ __device__ inline int64_t units_of(int phase, int64_t nseg) {
  if (phase == 3) return nseg > 1 ? nseg - 1 : 0;
  return 1 + (nseg > 2 ? 2 * (nseg - 2) : 0);
}

struct Unit {
  int n, kind;
  int64_t k, nseg;       // segment index within sequence n, and the sequence's segment count
  int64_t t_beg, t_end;  // token range
  int64_t slot0;         // chunk slot of the first chunk
  int64_t seg;           // global segment index (n, k)
};

// Longest-first order of a phase's units, so that the hardware's in-order block dispatch packs
// them well: rank 0 = whole sequences longer than one segment, 1 = full-length segments and the
// middle segments' maps, 2 = the rest.  Phase 0 (no scan) keeps sequence order.
__host__ __device__ inline int unit_rank(int phase, int kind, int64_t k, int64_t nseg, int64_t len,
                                         int64_t lseg) {
  if (phase == 0) return 0;
  if (kind == U_MAIN0 && nseg <= 1) return len > lseg ? 0 : 2;
  if (kind == U_MAINK && k == nseg - 1) return len - k * lseg == lseg ? 1 : 2;
  return 1;
}

// Unit `u` (index among the units of `phase`, per v-head, in longest-first order).  Returns false
// past the last unit, or with *bad set for a malformed cu_seqlens met on the way (nothing may be
// read through it then).  O(N) reads of cu_seqlens per rank.
__device__ inline bool find_unit(const int32_t* cu, int64_t T, int N, int64_t lseg, int phase,
                                 int64_t u, Unit& out, bool* bad) {
  *bad = false;
  for (int rank = 0; rank < 3; ++rank) {
    int64_t slot_base = 0, seg_base = 0;
    for (int m = 0; m < N; ++m) {
      int64_t a, b;
      if (cu) {
        a = cu[m];
        b = cu[m + 1];
        if (a < 0 || b < a || b > T) {
          *bad = true;
          return false;
        }
      } else {
        a = (int64_t)m * T;
        b = a + T;
      }
      const int64_t len = b - a;
      const int64_t nseg = seg_count(len, lseg);
      const int64_t nu = units_of(phase, nseg);
      for (int64_t i = 0; i < nu; ++i) {
        int64_t k;
        int kind;
        if (phase == 3) {
          k = i + 1;
          kind = U_MAINK;
        } else if (i == 0) {
          k = 0;
          kind = U_MAIN0;
        } else {
          k = 1 + (i - 1) / 2;
          kind = ((i - 1) & 1) ? U_MSEG : U_BSEG;
        }
        if (unit_rank(phase, kind, k, nseg, len, lseg) != rank) continue;
        if (u-- > 0) continue;
        const int64_t span = nseg <= 1 ? len : lseg;
        out.n = m;
        out.kind = kind;
        out.k = k;
        out.nseg = nseg;
        out.t_beg = a + k * span;
        out.t_end = out.t_beg + span < b ? out.t_beg + span : b;
        out.slot0 = slot_base + k * (span / C);
        out.seg = seg_base + k;
        return true;
      }
      slot_base += (len + C - 1) / C;
      seg_base += nseg;
    }
    if (phase == 0) break;
  }
  return false;
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
