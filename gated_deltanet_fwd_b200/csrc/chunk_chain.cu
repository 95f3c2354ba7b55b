// chunk_chain.cu -- the state-carrying half of the tensor-core prefill (bf16, dk = dv = 128,
// chunks of 64 tokens): one CTA per unit -- a whole sequence, or one segment of it under the
// intra-sequence scan (chunk_tm.cuh), for one v-head -- walks the unit's chunks in order with the
// fp32 state held in tensor memory.
//
// Method: the chunked parallel mode of "解密Qwen3-Next的Gated DeltaNet：如何用75%混合层实现长文本
// 高效推理" §2.2 (parallel inside a chunk, the state carried from chunk to chunk) for the gated
// delta rule S_t = e^{g_t} S_{t-1}(I - beta_t k_t k_t^T) + beta_t v_t k_t^T, o_t = scale S_t q_t.
// With the chunk's state-independent operands from the prep kernel (T', P, Gamma, d; see
// chunk_prep.cu), a chunk entering with state S (dv x dk) gives
//   U^T = V^T T'^T - (S K^T diag(Gamma)) T'^T          (the corrected values, dv x L)
//   O^T = S (diag(Gamma) Q)^T + U^T P^T                 (outputs, times scale)
//   S  <- Gamma_63 S + (U^T diag(d)) K
// which is exactly L steps of the recurrence.
//
// Orientation: tensor-memory lane j is value row j of S, so S itself is the A operand of the
// MMAs that need it (a bf16 copy in tensor memory next to the fp32 master), and so are the
// epilogue results X' = -(S K^T) diag(Gamma), U^T and U^T diag(d).  The serial path of a chunk
// never touches shared memory; every B operand (K, Q, V^T, T', P) is a TMA-loaded tile:
//   MMA_kq [D_k | D_q] = S_bf16 [K; Q]^T      M 128, N 128, K-dim 128   (critical)
//   MMA_v  D_U  = V^T T'^T                    M 128, N 64,  K-dim 64    (A = V^T from smem)
//   MMA_u  D_U += X' T'^T                     M 128, N 64,  K-dim 64    (critical)
//   MMA_s  S   += (U^T diag(d)) K             M 128, N 128, K-dim 64    (critical)
//   MMA_o  D_o  = U^T P^T                     M 128, N 64,  K-dim 64    (into D_k's columns)
// and O^T = diag(Gamma)-scaled D_q + D_o in the output epilogue.
// Warp roles (320 threads): warps 0-3 the critical epilogues (X', U^T, the bf16 refresh of S),
// warps 4-7 the side work (S scaled by Gamma_63, the output epilogue), warp 8 the TMA producer,
// warp 9 the MMA issuer.  Hand-offs to the issuer are named barriers;
// waits on MMA commits and TMA arrivals are bounded mbarrier waits -- a wait that runs out records
// GDN_ERR_TIMEOUT, and from then on every role skips its work but keeps the barrier sequence, so
// the CTA leaves together with nothing in flight.
#include "chunk_tm.cuh"
#include "gdn_internal.cuh"
#include "ptx.cuh"

namespace gdn {
namespace {

using namespace ptx;

// Warps: 0-3 the critical epilogues, 4-7 the side group, 8 the TMA producer, 9 the MMA issuer.
// Ten warps over four SM sub-partitions put three on two of them, so a thread may hold at most
// 168 registers.
constexpr int CH_THREADS = 320;
constexpr int W_PROD = 8, W_MMA = 9;

// shared memory (from a 1024-aligned base); a stage holds one chunk's tiles
constexpr uint32_t ST_KQ = 0;          // [K; Q]: per 64-column half, 64 K rows then 64 Q rows
                                       // (128 B each); the halves 16384 apart
constexpr uint32_t ST_V = 32768;       // V: two 64-column halves x 64 rows x 128 B
constexpr uint32_t ST_TP = 49152;      // [T'; P]: 128 rows x 128 B
constexpr uint32_t ST_GD = 65536;      // Gamma[64], d[64] fp32
constexpr uint32_t STAGE = 66560;      // 65 KB, a multiple of 1024
constexpr uint32_t SM_GAM = 2 * STAGE;      // Gamma of the two chunks whose outputs are pending
constexpr uint32_t SM_BAR = SM_GAM + 512;    // mbarriers, abort flag, tensor-memory slot
// the request stays well below the SM's 228 KB, leaving the rest of the unified L1 / shared
// memory to the L1 cache (which holds the side group's per-thread output staging)
constexpr uint32_t CH_SMEM = SM_BAR + 256 + 1024;  // + slack for the 1024-byte alignment
constexpr uint32_t STAGE_TX = 4 * 16384 + 512;
static_assert(CH_SMEM <= 232448, "shared memory budget");
static_assert(ST_V == ST_KQ + 32768 && ST_TP == ST_V + 16384, "stage layout");

enum { B_FULL0 = 0, B_EMPTY0 = 2, B_K = 4, B_U = 5, B_S = 6, B_O = 7, B_DRAIN = 8, B_N = 9 };

// named barriers: producer/consumer hand-offs to the MMA issuer and between the two groups
enum { NB_X = 1, NB_U = 2, NB_S = 3, NB_SR = 4 };
constexpr int NB_ALL = 288;  // epilogue group + side group + issuer warp
constexpr int NB_EI = 160;   // epilogue group + issuer warp
constexpr int NB_EH = 256;   // epilogue group + side group

// tensor-memory columns
constexpr uint32_t TM_S = 0, TM_K = 128, TM_Q = 192, TM_U = 256, TM_SB = 320, TM_X = 384,
                   TM_UT = 416, TM_UD = 448;

// Optional phase timing, compiled in only with -DGDN_CHAIN_TRACE: clock64 stamps of CTA 0, 32 slots
// per chunk, written to ChainParams::trace.
#ifdef GDN_CHAIN_TRACE
#define CH_TS(c, k)                                                            \
  do {                                                                         \
    if (P.trace && blockIdx.x == 0 && (c) < 256) P.trace[(c) * 32 + (k)] = clock64(); \
  } while (0)
#else
#define CH_TS(c, k) \
  do {              \
  } while (0)
#endif

struct ChainParams {
  const float* S0;
  const int32_t* cu;
  const unsigned char* ws;
  __nv_bfloat16* out;
  float* S_T;
  int* status;
  int64_t T;
  int64_t gd_off;
  float scale;
  int N, Hk, Hv;
  // intra-sequence scan (chunk_tm.cuh): phase 0 = one chain per sequence, 1 / 3 = scan phases
  int phase;
  const int64_t* plan;  // segment length in tokens chosen on the device (0: no scan); scan only
  int64_t max_segs;
  float* st;        // state arrays SOUT, BSEG, MSEG, SIN (scan phases only)
  int debug_skip_chunk;  // failure-test builds only: the producer withholds this chunk's tiles
  unsigned long long* trace;  // phase timing (trace builds only), else unused
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// descriptor of the same operand tile `bytes` further on
__device__ __forceinline__ uint64_t dadd(uint64_t d, uint32_t bytes) {
  return d + (uint64_t)(bytes >> 4);
}

// 64 fp32 columns of this warp's lanes
__device__ __forceinline__ void ld64(uint32_t taddr, float (&v)[64]) {
  tmem_ld16(taddr + 0, *reinterpret_cast<float(*)[16]>(v + 0));
  tmem_ld16(taddr + 16, *reinterpret_cast<float(*)[16]>(v + 16));
  tmem_ld16(taddr + 32, *reinterpret_cast<float(*)[16]>(v + 32));
  tmem_ld16(taddr + 48, *reinterpret_cast<float(*)[16]>(v + 48));
}

__global__ void __launch_bounds__(CH_THREADS, 1) chunk_chain_kernel(
    const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
    const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_tp,
    const ChainParams P) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM_BAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM_BAR + B_N * 8);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM_BAR + B_N * 8 + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x % P.Hv;
  const int hk = h / (P.Hv / P.Hk);

  // ---- the unit this CTA runs: a whole sequence, or one segment of it (uniform across the CTA)
  tm::Unit U;
  {
    bool bad = false;
    const int64_t lseg = P.phase == 0 ? 0 : *P.plan;
    if (!tm::find_unit(P.cu, P.T, P.N, lseg, P.phase, blockIdx.x / P.Hv, U, &bad)) {
      if (bad && tid == 0) report(P.status, GDN_ERR_DEVICE_ARG);
      return;  // nothing allocated yet
    }
  }
  const int n = U.n;
  const int64_t s_beg = U.t_beg, s_end = U.t_end, slot0 = U.slot0;
  const size_t hs = tm::STATE_FLOATS;
  const size_t sidx = ((size_t)n * P.Hv + h) * hs;  // this sequence's state in S0 / S_T / SOUT
  const size_t gidx = ((size_t)U.seg * P.Hv + h) * hs;  // this segment's state in BSEG/MSEG/SIN
  float* const st_out = P.st;
  float* const st_b = P.st + (size_t)P.N * P.Hv * hs;
  float* const st_m = st_b + (size_t)P.max_segs * P.Hv * hs;
  float* const st_in = st_m + (size_t)P.max_segs * P.Hv * hs;
  // entry state (null: zero; the identity for a segment's transition) and where the leaving state
  // goes (null: nowhere)
  const bool ident = U.kind == tm::U_MSEG;
  const float* src_state = U.kind == tm::U_MAIN0   ? (P.S0 ? P.S0 + sidx : nullptr)
                           : U.kind == tm::U_MAINK ? st_in + gidx
                                                   : nullptr;
  float* dst_state = U.kind == tm::U_MAIN0   ? (U.nseg <= 1 ? (P.S_T ? P.S_T + sidx : nullptr)
                                                            : st_out + sidx)
                     : U.kind == tm::U_BSEG  ? st_b + gidx
                     : U.kind == tm::U_MSEG  ? st_m + gidx
                     : (U.k == U.nseg - 1 ? (P.S_T ? P.S_T + sidx : nullptr) : nullptr);
  const bool has_out = U.kind == tm::U_MAIN0 || U.kind == tm::U_MAINK;
  const bool zero_v = U.kind == tm::U_MSEG;  // the transition: the chain of v = 0 from the identity

  const int nchunks = (int)((s_end - s_beg + tm::C - 1) / tm::C);
  if (nchunks == 0) {  // empty sequence: the state passes through
    if (dst_state)
      for (int e = tid; e < tm::D * tm::D; e += CH_THREADS)
        dst_state[e] = src_state ? src_state[e] : 0.0f;
    return;
  }

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[B_FULL0 + i], 1);
      mbar_init(&bars[B_EMPTY0 + i], 1);
    }
    mbar_init(&bars[B_K], 1);
    mbar_init(&bars[B_U], 1);
    mbar_init(&bars[B_S], 1);
    mbar_init(&bars[B_O], 1);
    mbar_init(&bars[B_DRAIN], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail = [&](int code) {
    report(P.status, code);
    *abort_flag = 1;
  };
  // a bounded wait, skipped once the CTA is aborting
  auto wait = [&](int b, uint32_t parity) -> bool {
    if (*abort_flag) return false;
    if (mbar_wait(&bars[b], parity)) return true;
    fail(GDN_ERR_TIMEOUT);
    return false;
  };
  auto chunk_t0 = [&](int c) { return s_beg + (int64_t)tm::C * c; };

  if (warp < 8) {
    if (warp < 4) {
      // ------------------------------------------------------------ critical epilogues -------
      const int j = 32 * warp + lane;  // value row of S = tensor-memory lane
      const uint32_t lo = (uint32_t)(32 * warp) << 16;
      // initial state: fp32 master and bf16 operand copy
      {
        const float* src = src_state ? src_state + (size_t)j * tm::D : nullptr;
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {  // 32 columns at a time
          float v[32];
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 f = src ? __ldg(reinterpret_cast<const float4*>(src + 32 * blk) + q4)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
            v[4 * q4] = f.x;
            v[4 * q4 + 1] = f.y;
            v[4 * q4 + 2] = f.z;
            v[4 * q4 + 3] = f.w;
          }
          if (ident) {
#pragma unroll
            for (int q = 0; q < 32; ++q) v[q] = (32 * blk + q == j) ? 1.0f : 0.0f;
          }
          tmem_st16(tmem + lo + TM_S + 32 * blk, *reinterpret_cast<float(*)[16]>(v));
          tmem_st16(tmem + lo + TM_S + 32 * blk + 16, *reinterpret_cast<float(*)[16]>(v + 16));
          uint32_t pk[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) pk[q] = pack_bf16x2(v[2 * q], v[2 * q + 1]);
          tmem_st16u(tmem + lo + TM_SB + 16 * blk, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        named_bar_arrive(NB_SR, NB_EH);  // the side group may now scale S
        named_bar(NB_S, NB_ALL);
      }
      for (int c = 0; c < nchunks; ++c) {
        const int st = c & 1;
        const float* gd = reinterpret_cast<const float*>(smem + st * STAGE + ST_GD);
        wait(B_FULL0 + st, (c >> 1) & 1);  // the chunk's Gamma and d are visible to this thread
        // ---- X' = -(S K^T) diag(Gamma), 32 columns at a time
        if (wait(B_K, c & 1)) {
          if (tid == 0) CH_TS(c, 5);
          tc_fence_after();
          float dk[64];
          ld64(tmem + lo + TM_K, dk);
          tmem_ld_wait();
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t pk[16];
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
              const float4 gm = *reinterpret_cast<const float4*>(gd + 32 * hh + 4 * q4);
              const float* x = dk + 32 * hh + 4 * q4;
              pk[2 * q4] = pack_bf16x2(-gm.x * x[0], -gm.y * x[1]);
              pk[2 * q4 + 1] = pack_bf16x2(-gm.z * x[2], -gm.w * x[3]);
            }
            tmem_st16u(tmem + lo + TM_X + 16 * hh, pk);
          }
          tmem_st_wait();
        }
        if (tid == 0) CH_TS(c, 6);
        tc_fence_before();
        named_bar_arrive(NB_X, NB_EI);
        // ---- U^T and U^T diag(d)
        if (wait(B_U, c & 1)) {
          if (tid == 0) CH_TS(c, 7);
          tc_fence_after();
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            float u[32];
            tmem_ld32(tmem + lo + TM_U + 32 * hh, u);
            tmem_ld_wait();
            uint32_t pk[16], pd[16];
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
              const float4 dd = *reinterpret_cast<const float4*>(gd + 64 + 32 * hh + 4 * q4);
              const float* x = u + 4 * q4;
              pk[2 * q4] = pack_bf16x2(x[0], x[1]);
              pk[2 * q4 + 1] = pack_bf16x2(x[2], x[3]);
              pd[2 * q4] = pack_bf16x2(x[0] * dd.x, x[1] * dd.y);
              pd[2 * q4 + 1] = pack_bf16x2(x[2] * dd.z, x[3] * dd.w);
            }
            tmem_st16u(tmem + lo + TM_UT + 16 * hh, pk);
            tmem_st16u(tmem + lo + TM_UD + 16 * hh, pd);
          }
          tmem_st_wait();
        }
        tc_fence_before();
        // a full barrier, not an arrival: the group then never runs a barrier instance ahead of
        // the issuer, even when an abort makes it skip its waits
        if (tid == 0) CH_TS(c, 8);
        named_bar(NB_U, NB_ALL);
        if (tid == 0) CH_TS(c, 9);
        // ---- refresh of the bf16 copy of the new state (not after the last chunk)
        const bool s_ok = wait(B_S, c & 1);
        if (tid == 0) CH_TS(c, 10);
        if (c + 1 < nchunks) {
          if (s_ok) {
            tc_fence_after();
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              float v[64];
              ld64(tmem + lo + TM_S + 64 * hh, v);
              tmem_ld_wait();
              uint32_t pk[32];
#pragma unroll
              for (int q = 0; q < 32; ++q) pk[q] = pack_bf16x2(v[2 * q], v[2 * q + 1]);
              tmem_st16u(tmem + lo + TM_SB + 32 * hh, *reinterpret_cast<uint32_t(*)[16]>(pk));
              tmem_st16u(tmem + lo + TM_SB + 32 * hh + 16,
                         *reinterpret_cast<uint32_t(*)[16]>(pk + 16));
            }
          }
          tc_fence_before();
          named_bar_arrive(NB_SR, NB_EH);  // S read: the side group may scale it
          tmem_st_wait();
          if (tid == 0) CH_TS(c, 11);
          tc_fence_before();
          named_bar(NB_S, NB_ALL);
        }

      }
    } else {
      // ------------------------------------------------------------ side group (warps 4-7) ---
      const int t4 = tid - 128;
      const int j = 32 * (warp - 4) + lane;
      const uint32_t lo = (uint32_t)(32 * (warp - 4)) << 16;
      // Gamma of the chunks whose outputs are pending (the stage may be refilled before then)
      float* gam_o = reinterpret_cast<float*>(smem + SM_GAM);
      // S <- Gamma_63(c) S in tensor memory (after the critical group has read S); keeps Gamma(c)
      auto scale_s = [&](int c) {
        named_bar(NB_SR, NB_EH);
        tc_fence_after();
        if (!wait(B_FULL0 + (c & 1), (c >> 1) & 1)) return;
        const float* gd = reinterpret_cast<const float*>(smem + (c & 1) * STAGE + ST_GD);
        if (t4 < 64) gam_o[(c & 1) * 64 + t4] = gd[t4];
        const float gl = gd[63];
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
          float v[32];
          tmem_ld32(tmem + lo + TM_S + 32 * hh, v);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 32; ++q) v[q] *= gl;
#pragma unroll
          for (int q4 = 0; q4 < 2; ++q4)
            tmem_st16(tmem + lo + TM_S + 32 * hh + 16 * q4, *reinterpret_cast<float(*)[16]>(v + 16 * q4));
        }
        tmem_st_wait();
      };
      named_bar_arrive(NB_S, NB_ALL);  // D_q is free
      scale_s(0);
      tc_fence_before();
      for (int c = 0; c < nchunks; ++c) {
        named_bar(NB_U, NB_ALL);  // S scaled by Gamma_63(c); a full barrier (see the other group)
        // ---- outputs of chunk c: O^T = diag(Gamma) (S Q^T) + U^T P^T, held as scaled bf16 pairs
        // (rows 2q, 2q + 1) of value column j
        uint32_t ob[32];
        const bool o_ok = has_out && wait(B_O, c & 1);
        if (t4 == 0) CH_TS(c, 12);
        if (o_ok) {
          tc_fence_after();
          const float* gm = gam_o + (c & 1) * 64;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            float dq[32], doo[32];
            tmem_ld16(tmem + lo + TM_Q + 32 * hh, *reinterpret_cast<float(*)[16]>(dq));
            tmem_ld16(tmem + lo + TM_Q + 32 * hh + 16, *reinterpret_cast<float(*)[16]>(dq + 16));
            tmem_ld16(tmem + lo + TM_K + 32 * hh, *reinterpret_cast<float(*)[16]>(doo));
            tmem_ld16(tmem + lo + TM_K + 32 * hh + 16, *reinterpret_cast<float(*)[16]>(doo + 16));
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const float2 g2 = *reinterpret_cast<const float2*>(gm + 32 * hh + 2 * q);
              ob[16 * hh + q] = pack_bf16x2(P.scale * fmaf(g2.x, dq[2 * q], doo[2 * q]),
                                            P.scale * fmaf(g2.y, dq[2 * q + 1], doo[2 * q + 1]));
            }
          }
        }
        tc_fence_before();
        if (c + 1 < nchunks) named_bar_arrive(NB_S, NB_ALL);  // D_q and D_o read
        // ---- S scaled by Gamma_63 for chunk c + 1 (needed before the issuer's next NB_U)
        if (c + 1 < nchunks) {
          scale_s(c + 1);
          if (t4 == 0) CH_TS(c, 14);
          tc_fence_before();
        }
        if (o_ok && !*abort_flag) {
          // lanes j, j ^ 1 swap halves: an even lane stores row 2q at columns j, j + 1, an odd lane
          // row 2q + 1 at columns j - 1, j -- each store a 4-byte pair, each warp store two
          // contiguous 64-byte row segments
          const int64_t t0 = chunk_t0(c);
          const int L = (int)min((int64_t)tm::C, s_end - t0);
          const int odd = j & 1;
          const int64_t rs = (int64_t)P.Hv * tm::D;  // elements between consecutive tokens
          uint32_t* dst = reinterpret_cast<uint32_t*>(P.out + (t0 + odd) * rs + h * tm::D + (j & ~1));
          const uint32_t sel = odd ? 0x7632u : 0x5410u;
          const int64_t step = rs;  // two token rows of bf16, counted in 4-byte units
#pragma unroll 8
          for (int q = 0; q < 32; ++q) {
            const uint32_t mine = ob[q];
            const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 1);
            const uint32_t pair = odd ? __byte_perm(other, mine, sel) : __byte_perm(mine, other, sel);
            if (2 * q + odd < L) *dst = pair;
            dst += step;
          }
        }
        if (t4 == 0) CH_TS(c, 13);
      }
    }
  } else {
    if (warp == W_PROD) {
      // ------------------------------------------------------------ TMA producer -------------
      if (lane == 0) {
        prefetch_tensormap(&map_q);
        prefetch_tensormap(&map_k);
        prefetch_tensormap(&map_v);
        prefetch_tensormap(&map_tp);
        int issued = 0;
        for (int c = 0; c < nchunks; ++c) {
          const int st = c & 1;
          if (c >= 2 && !wait(B_EMPTY0 + st, ((c >> 1) & 1) ^ 1)) break;
          if (*abort_flag) break;
          const int32_t t0 = (int32_t)chunk_t0(c);
          unsigned char* sp = smem + st * STAGE;
          uint64_t* fb = &bars[B_FULL0 + st];
          mbar_arrive_expect_tx(fb, zero_v ? STAGE_TX - 16384 : STAGE_TX);
  #ifdef GDN_FAULT_INJECTION
          if (c == P.debug_skip_chunk) continue;  // nothing lands: the waits on this stage run out
  #endif
          tma_load_3d(sp + ST_KQ, &map_k, fb, 0, hk, t0);
          tma_load_3d(sp + ST_KQ + 8192, &map_q, fb, 0, hk, t0);
          tma_load_3d(sp + ST_KQ + 16384, &map_k, fb, 64, hk, t0);
          tma_load_3d(sp + ST_KQ + 24576, &map_q, fb, 64, hk, t0);
          if (!zero_v) {
            tma_load_3d(sp + ST_V, &map_v, fb, 0, h, t0);
            tma_load_3d(sp + ST_V + 8192, &map_v, fb, 64, h, t0);
          }
          const int64_t slot = slot0 + c;
          tma_load_2d(sp + ST_TP, &map_tp, fb, 0, (int32_t)((slot * P.Hv + h) * 128));
          bulk_load(sp + ST_GD, P.ws + P.gd_off + ((size_t)slot * P.Hv + h) * tm::GD_BYTES,
                    tm::GD_BYTES, fb);
          issued = c + 1;
        }
        // never leave the CTA with copies still landing in shared memory (each wait bounded; a
        // stage whose copies were never issued simply runs out)
        for (int c = issued - 2 < 0 ? 0 : issued - 2; c < issued; ++c)
          if (!mbar_wait(&bars[B_FULL0 + (c & 1)], (uint32_t)(c >> 1) & 1))
            report(P.status, GDN_ERR_TIMEOUT);
      }
    } else if (warp == W_MMA) {
      // ------------------------------------------------------------ MMA issuer ---------------
      const uint32_t id_n64 = idesc_bf16(128, 64, 0, 0);   // A tensor memory, B K-major
      const uint32_t id_kq = idesc_bf16(128, 128, 0, 0);   // A tensor memory, B = [K; Q] K-major
      const uint32_t id_v = idesc_bf16(128, 64, 1, 0);     // A = V^T (MN-major smem), B K-major
      const uint32_t id_s = idesc_bf16(128, 128, 0, 1);    // B = K (MN-major)
      named_bar(NB_S, NB_ALL);  // S and its bf16 copy initialised; D_q free
      for (int c = 0; c < nchunks; ++c) {
        const int st = c & 1;
        const uint32_t sp = sbase + st * STAGE;
        if (lane == 0) CH_TS(c, 0);
        const bool have = wait(B_FULL0 + st, (c >> 1) & 1);
        if (c > 0) named_bar(NB_S, NB_ALL);  // refresh of S done, D_q read
        if (lane == 0) CH_TS(c, 1);
        const bool go = have && !*abort_flag;
        const bool leader = lane == 0;
        const uint64_t dKQ = sdesc_sw128(sp + ST_KQ, 16, 1024);    // [K; Q] as K-major B
        const uint64_t dVt = sdesc_sw128(sp + ST_V, 8192, 1024);   // V^T as MN-major A
        const uint64_t dTp = sdesc_sw128(sp + ST_TP, 16, 1024);    // T' as K-major B
        const uint64_t dP = sdesc_sw128(sp + ST_TP + 8192, 16, 1024);  // P as K-major B
        const uint64_t dKn = sdesc_sw128(sp + ST_KQ, 16384, 1024);  // K as MN-major B
        if (go && leader) {
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_bf16_ts(tmem + TM_K, tmem + TM_SB + 8 * ks,
                        dadd(dKQ, (ks >> 2) * 16384 + (ks & 3) * 32), id_kq, ks > 0);
          mma_commit(&bars[B_K]);
          if (!zero_v) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_bf16_ss(tmem + TM_U, dadd(dVt, ks * 2048), dadd(dTp, ks * 32), id_v, ks > 0);
          }
        }
        if (lane == 0) CH_TS(c, 2);
        __syncwarp();
        named_bar(NB_X, NB_EI);  // X' written
        if (lane == 0) CH_TS(c, 3);
        if (go && leader && !*abort_flag) {
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_bf16_ts(tmem + TM_U, tmem + TM_X + 8 * ks, dadd(dTp, ks * 32), id_n64,
                        !zero_v || ks > 0);
          mma_commit(&bars[B_U]);
        }
        __syncwarp();
        named_bar(NB_U, NB_ALL);  // U^T, U^T diag(d) written; S scaled by Gamma_63
        if (lane == 0) CH_TS(c, 4);
        if (go && leader && !*abort_flag) {
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_bf16_ts(tmem + TM_S, tmem + TM_UD + 8 * ks, dadd(dKn, ks * 2048), id_s, 1);
          mma_commit(&bars[B_S]);
          if (has_out) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_bf16_ts(tmem + TM_K, tmem + TM_UT + 8 * ks, dadd(dP, ks * 32), id_n64, ks > 0);
            mma_commit(&bars[B_O]);
          }
          mma_commit(&bars[B_EMPTY0 + st]);
        }
        __syncwarp();
      }
      if (lane == 0) {
        // every MMA has completed before tensor memory is read back or released
        mma_commit(&bars[B_DRAIN]);
        if (!mbar_wait(&bars[B_DRAIN], 0)) fail(GDN_ERR_TIMEOUT);
      }
    }
  }

  // the issuer's drain (and any abort) is visible to every thread after this barrier
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp < 4 && dst_state && !*abort_flag) {
    const int j = 32 * warp + lane;
    const uint32_t lo = (uint32_t)(32 * warp) << 16;
    float* dst = dst_state + (size_t)j * tm::D;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float v[64];
      ld64(tmem + lo + TM_S + 64 * hh, v);
      tmem_ld_wait();
#pragma unroll
      for (int q4 = 0; q4 < 16; ++q4)
        reinterpret_cast<float4*>(dst + 64 * hh)[q4] =
            make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

int g_debug_skip_chunk = -1;  // failure-test builds: chunk whose tiles the producer withholds
unsigned long long* g_chain_trace = nullptr;  // trace builds: device buffer of 256 x 32 stamps

}  // namespace

cudaError_t launch_chunk_chain(const void* q, const void* k, const void* v, TokStrides ts,
                               float scale, const float* S0, const int32_t* cu, int N, int B,
                               int64_t T, int Hk, int Hv, void* out, float* S_T, void* ws,
                               int phase, int64_t lseg, int* status, cudaStream_t s) {
  const int64_t n_tok = (int64_t)B * T;
  const int64_t msegs = tm::max_segs(N, n_tok, lseg);  // lseg: the smallest the planner may pick
  // units per v-head: phase 0 one per sequence; phase 1 at most one per sequence and two per
  // segment; phase 3 at most one per segment
  const int64_t units = (phase == 0 ? (int64_t)N : phase == 1 ? N + 2 * msegs : msegs) * Hv;
  if (units == 0) return cudaSuccess;
  if (units > 0x7fffffff) return cudaErrorInvalidConfiguration;
  const int64_t slots = tm::max_slots(N, n_tok);
  CUtensorMap mq, mk, mv, mtp;
  const int64_t map_rows = n_tok > 0 ? n_tok : 1;
  unsigned char* wsb = reinterpret_cast<unsigned char*>(ws);
  if (!make_tok_map(&mq, q, Hk, map_rows, ts.q) || !make_tok_map(&mk, k, Hk, map_rows, ts.k) ||
      !make_tok_map(&mv, v, Hv, map_rows, ts.v) ||
      !make_rows64_map(&mtp, wsb + tm::tp_offset(), slots * Hv * 128, 128))
    return cudaErrorInvalidValue;
  ChainParams p;
  p.S0 = S0;
  p.cu = cu;
  p.ws = wsb;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.S_T = S_T;
  p.status = status;
  p.T = T;
  p.gd_off = (int64_t)tm::gd_offset(N, n_tok, Hv);
  p.scale = scale;
  p.N = N;
  p.Hk = Hk;
  p.Hv = Hv;
  p.phase = phase;
  p.plan = reinterpret_cast<const int64_t*>(wsb + tm::PLAN_OFF);
  p.max_segs = msegs;
  p.st = phase == 0 ? nullptr
                    : reinterpret_cast<float*>(wsb + tm::states_offset(N, n_tok, Hv));
  p.debug_skip_chunk = g_debug_skip_chunk;
  p.trace = g_chain_trace;
  static bool attr_set = false;  // idempotent attribute; a benign race between host threads
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(chunk_chain_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, CH_SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  chunk_chain_kernel<<<(unsigned)units, CH_THREADS, CH_SMEM, s>>>(mq, mk, mv, mtp, p);
  return cudaGetLastError();
}

}  // namespace gdn

#ifdef GDN_CHAIN_TRACE
// Trace builds only: device buffer (256 chunks x 32 slots of 8 bytes) for the phase stamps of CTA 0.
extern "C" void gdn_debug_set_chain_trace(void* buf) {
  gdn::g_chain_trace = reinterpret_cast<unsigned long long*>(buf);
}
#endif

#ifdef GDN_FAULT_INJECTION
// Failure-test builds only (libgdn_debug.so, not the product library): the next prefills on the
// tensor-core path withhold the tiles of chunk `c` of every sequence (-1: none), so that the waits
// on them run out after the build's short wait limit and the kernels report GDN_ERR_TIMEOUT.
extern "C" void gdn_debug_set_skip_chunk(int c) { gdn::g_debug_skip_chunk = c; }
#endif
