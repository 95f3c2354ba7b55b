// chunk_tc.cu -- chunk-parallel gated delta rule on the tcgen05 tensor cores (bf16 operands,
// fp32 accumulation in tensor memory, fp32 state), for dk = dv = 128 and chunks of 64 tokens.
//
// Method: the chunked parallel mode (chunk_gated_delta_rule) of "解密Qwen3-Next的Gated DeltaNet：
// 如何用75%混合层实现长文本高效推理" §2.2 -- parallel inside a chunk, state carried across chunks --
// applied to the gated delta rule S_t = e^{g_t} S_{t-1}(I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
// o_t = scale S_t q_t.  For a chunk of L <= 64 tokens entering with state S0 (dv x dk), with
// gamma_r the in-chunk cumulative log-decay, Gamma_r = e^{gamma_r}:
//   A[r,s] = beta_r e^{gamma_r - gamma_s} k_r.k_s (s < r),   T = (I + A)^{-1},   T' = T diag(beta)
//   P[r,s] = e^{gamma_r - gamma_s} q_r.k_s (s <= r)
//   X = V - diag(Gamma) K S0^T,   U = T' X                      (the per-token corrections)
//   O = scale (diag(Gamma) Q S0^T + P U)
//   S_L = Gamma_L S0 + U^T diag(e^{gamma_L - gamma}) K
// which is exactly L steps of the recurrence.  Only differences of in-chunk cumulative log-decays
// are exponentiated, so nothing over- or underflows.
//
// Each (sequence, v-head) chain runs on a cluster of two CTAs (two SMs):
//   * the prep CTA (rank 0) runs ahead of the chain: it loads K and Q, computes D1 = [K; Q] K^T on
//     the tensor cores, builds the decay masks of A (fp32) and P, inverts I + A (fp32 forward
//     substitution on the 16 x 16 diagonal blocks, tf32 mma.sync for the off-diagonal block
//     products) and writes T' and P, as one bf16 [T'; P] operand tile, straight into the chain
//     CTA's shared memory (a bulk copy over distributed shared memory that completes on the
//     chain CTA's mbarrier);
//   * the chain CTA (rank 1) runs the serial part, four M = 128 tcgen05 MMAs per chunk:
//       DKS  = [K; Q] S0^T      (128 x 128, K-dim 128)  -> K S0^T (for X) and Q S0^T (for O)
//       DU   = [T'; P] X        (128 x 128, K-dim 64)   -> U in rows 0..63
//       DU   = [T'; P] U        (after U is copied out) -> P U in rows 64..127
//       DS  += K^T (D U)        (128 x 128, K-dim 64)   -> onto the decayed fp32 state,
//                                                          D = diag(e^{gamma_L - gamma})
//     and O = scale (Gamma_r (Q S0^T)_r + (P U)_r) in the output epilogue.  The fp32 state S^T lives
//     in tensor memory (scaled by Gamma_L in place while the first MMA runs); its bf16 copy in
//     shared memory is the next chunk's operand.  Sixteen warps (four warpgroups, 32 value columns
//     per thread) work the epilogues; one elected thread issues the MMAs; inside the chain the only
//     synchronisation is named barriers and waits on the chain's own MMA commits.
// Both CTAs have a producer warp that streams their chunk tiles with TMA.  Every mbarrier wait is
// bounded; a wait that runs out records GDN_ERR_TIMEOUT and the cluster winds down.
#include <mutex>

#include "gdn_internal.cuh"
#include "ptx.cuh"

namespace gdn {
namespace {

using namespace ptx;

constexpr int TC_WORKERS = 512;                // 16 warps of prep or chain work per CTA
constexpr int TC_THREADS = TC_WORKERS + 32;    // + one producer warp
constexpr int PRODUCER_WARP = 16;
constexpr int AS = 68;  // fp32 row stride of the A and T scratch matrices (floats)
constexpr int MS = 20;  // fp32 row stride of the 16 x 16 block-product scratch

// chain CTA shared memory (bytes from a 1024-aligned base)
constexpr uint32_t CH_KQ = 0;           // 2 stages x [K;Q] tile: 2 dk-halves x 128 rows x 128 B
constexpr uint32_t KQ_STAGE = 32768;
constexpr uint32_t CH_V = 65536;        // 2 stages x V tile: 2 dv-halves x 64 rows x 128 B
constexpr uint32_t V_STAGE = 16384;
constexpr uint32_t CH_SB = 98304;       // S^T bf16 (MN-major B operand): 2 x 128 rows x 128 B
constexpr uint32_t CH_XU = 131072;      // X, then U (MN-major B operand): 2 x 64 rows x 128 B
constexpr uint32_t CH_TP = 147456;      // 2 buffers x [T'; P] (K-major A), written by the prep CTA
constexpr uint32_t TP_BUF = 16384;
// prep CTA shared memory
constexpr uint32_t PR_KQ = 0;           // 3 stages x [K;Q] tile
constexpr int PR_STAGES = 3;
constexpr uint32_t PR_AF = 98304;                     // fp32 A [64][AS]
constexpr uint32_t PR_TF = PR_AF + 64 * AS * 4;       // fp32 T [64][AS]
constexpr uint32_t PR_MB = PR_TF + 64 * AS * 4;       // fp32 4 x [16][MS] block products
constexpr uint32_t PR_PV = PR_MB + 4 * 16 * MS * 4;   // gamma * log2(e)[64], beta[64]
constexpr uint32_t PR_TPL = 139264;                   // 2 x [T'; P] staging tiles (bulk-copied)
// mbarriers (same offsets in both CTAs; each CTA initialises and uses its own subset)
constexpr uint32_t OFF_BAR = 180224;
constexpr uint32_t N_BARS = 16;
constexpr uint32_t OFF_GX = OFF_BAR + 256;  // prefetched gates: 2 x (g[64], beta[64]) fp32
constexpr uint32_t SMEM_USED = OFF_GX + 1024;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // slack for 1024-byte alignment
static_assert(PR_PV + 512 <= PR_TPL && PR_TPL % 1024 == 0, "prep layout");
static_assert(PR_TPL + 2 * TP_BUF <= OFF_BAR, "prep staging");
static_assert(CH_TP + 2 * TP_BUF <= OFF_BAR, "chain layout");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

enum {
  B_FULL0 = 0,        // 3 TMA stages (chain uses 2)
  B_EMPTY0 = 3,       // 3 stages
  B_PREP_FULL0 = 6,   // chain CTA: [T'; P] buffer b written (arrived by the prep CTA)
  B_PREP_EMPTY0 = 8,  // prep CTA: [T'; P] buffer b consumed (arrived by the chain CTA)
  B_D1_FULL = 10,     // prep CTA
  B_M_KS = 11,        // chain CTA: MMA commits
  B_M_U = 12,
  B_M_S = 13,
  B_DRAIN = 14,
  B_COUNT = 15
};
static_assert(B_COUNT <= (int)N_BARS, "barrier space");

// tensor-memory columns (chain CTA; the prep CTA holds D1 only)
// D_KS alternates between two column blocks by chunk parity, so that a chunk's output can be read
// out while the next chunk's first MMA runs.
constexpr uint32_t TM_KS = 0, TM_U = 128, TM_S = 256, TM_KS2 = 384;

constexpr float kLog2e = 1.4426950408889634f;

// Optional phase timing, compiled in only with -DGDN_TC_TRACE: per-role clock64 accumulators of
// cluster 0, written to TcParams::trace (16 slots per role) when the role finishes.
#ifdef GDN_TC_TRACE
#define TC_TRACE_DECL(active)                                 \
  const bool tr_on_ = (active) && blockIdx.x < 2;           \
  unsigned long long tr_acc_[16] = {};                        \
  unsigned long long tr_last_ = clock64();
#define TC_TS(k)                                              \
  do {                                                        \
    if (tr_on_) {                                             \
      const unsigned long long n_ = clock64();                \
      tr_acc_[k] += n_ - tr_last_;                            \
      tr_last_ = n_;                                          \
    }                                                         \
  } while (0)
#define TC_TRACE_FLUSH(role)                                                  \
  do {                                                                        \
    if (tr_on_ && P.trace)                                                    \
      for (int k_ = 0; k_ < 16; ++k_) P.trace[(role) * 16 + k_] = tr_acc_[k_]; \
  } while (0)
#else
#define TC_TRACE_DECL(active)
#define TC_TS(k) \
  do {           \
  } while (0)
#define TC_TRACE_FLUSH(role) \
  do {                       \
  } while (0)
#endif

struct TcParams {
  const float* g;
  const float* beta;
  const float* S0;
  const int32_t* cu;
  __nv_bfloat16* out;
  float* S_T;
  int* status;
  unsigned long long* trace;  // phase timing (trace builds only), else unused
  float scale;
  int N, Hk, Hv;
  int64_t T;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void unpack8(uint4 u, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

__device__ __forceinline__ uint4 pack8(const float* f) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Descriptor of the same operand tile `bytes` further on (start-address field, 16-byte units;
// shared-memory addresses stay below 256 KB, so the field never carries).
__device__ __forceinline__ uint64_t dadd(uint64_t d, uint32_t bytes) {
  return d + (uint64_t)(bytes >> 4);
}
// K-major 128-byte-swizzled operand with two 64-element K halves `half` bytes apart: k-step ks.
__device__ __forceinline__ uint32_t kstep_kmajor(int ks, uint32_t half) {
  return (uint32_t)(ks >> 2) * half + (uint32_t)(ks & 3) * 32u;
}

// ---------------------------------------------------------------- cluster helpers ----------

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
                   "memory");
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}

// Arrive on an mbarrier of a peer CTA (release at CTA scope: used only to hand back a buffer
// whose readers, this CTA's MMAs, have completed).
__device__ __forceinline__ void mbar_arrive_peer(uint32_t peer_bar) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(peer_bar) : "memory");
}

// 4-byte asynchronous global -> shared copy; `valid` false writes zero instead.
__device__ __forceinline__ void cp_async4(uint32_t dst, const float* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Copies `bytes` of this CTA's shared memory into a peer CTA's shared memory; the bytes are
// counted on the peer's mbarrier as they land.
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t peer_dst, uint32_t local_src,
                                                  uint32_t bytes, uint32_t peer_bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, "
      "[%3];" ::"r"(peer_dst),
      "r"(local_src), "r"(bytes), "r"(peer_bar)
      : "memory");
}

// ---------------------------------------------------------------- the kernel ---------------

__global__ void __launch_bounds__(TC_THREADS, 1) chunk_tc_kernel(
    const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
    const __grid_constant__ CUtensorMap map_v, const TcParams P) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_BAR + N_BARS * 8);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_BAR + N_BARS * 8 + 4);
  // prep CTA: number of [T'; P] bulk copies its leader has issued into the chain CTA (read by the
  // chain CTA at exit, so that no copy can still be landing in its shared memory when it leaves)
  volatile int* prep_issued = reinterpret_cast<volatile int*>(smem + OFF_BAR + N_BARS * 8 + 8);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();  // 0 = prep, 1 = chain
  const int unit = blockIdx.x >> 1;
  const int n = unit / P.Hv, h = unit % P.Hv;
  const int hk = h / (P.Hv / P.Hk);

  int64_t s_beg, s_end;
  if (P.cu) {
    s_beg = P.cu[n];
    s_end = P.cu[n + 1];
  } else {
    s_beg = (int64_t)n * P.T;
    s_end = s_beg + P.T;
  }
  if (P.cu && (s_beg < 0 || s_end < s_beg || s_end > P.T)) {
    if (tid == 0 && rank == 1) report(P.status, GDN_ERR_DEVICE_ARG);
    return;  // uniform across the cluster: both CTAs see the same sequence, nothing allocated
  }
  const int nchunks = (int)((s_end - s_beg + 63) / 64);

  if (tid == 0) {
    for (int i = 0; i < PR_STAGES; ++i) {
      mbar_init(&bars[B_FULL0 + i], 1);
      mbar_init(&bars[B_EMPTY0 + i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[B_PREP_FULL0 + i], 1);
      mbar_init(&bars[B_PREP_EMPTY0 + i], 1);
    }
    mbar_init(&bars[B_D1_FULL], 1);
    mbar_init(&bars[B_M_KS], 1);
    mbar_init(&bars[B_M_U], 1);
    mbar_init(&bars[B_M_S], 1);
    mbar_init(&bars[B_DRAIN], 1);
    *abort_flag = 0;
    *prep_issued = 0;
    fence_barrier_init();
    // the chain CTA expects one [T'; P] tile per chunk from the prep CTA's bulk copies
    if (rank == 1) {
      for (int i = 0; i < 2 && i < nchunks; ++i)
        mbar_arrive_expect_tx(&bars[B_PREP_FULL0 + i], TP_BUF);
    }
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, rank == 1 ? 512 : 64);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail = [&](int code) {
    report(P.status, code);
    *abort_flag = 1;
  };
  int tp_consumed_final = 0;  // chain leader: [T'; P] arrivals it waited for

  if (warp == PRODUCER_WARP) {
    // ------------------------------------------------------------ TMA producers -----------
    if (lane == 0) {
      prefetch_tensormap(&map_q);
      prefetch_tensormap(&map_k);
      prefetch_tensormap(&map_v);
      const int stages = rank == 1 ? 2 : PR_STAGES;
      const uint32_t kq_base = rank == 1 ? CH_KQ : PR_KQ;
      int issued = 0;
      for (int c = 0; c < nchunks; ++c) {
        if (*abort_flag) break;
        const int st = c % stages;
        const uint32_t use = (uint32_t)(c / stages);
        if (!mbar_wait(&bars[B_EMPTY0 + st], (use & 1) ^ 1)) {
          fail(GDN_ERR_TIMEOUT);
          break;
        }
        const int32_t t0 = (int32_t)(s_beg + 64 * c);
        unsigned char* kq = smem + kq_base + st * KQ_STAGE;
        uint64_t* fb = &bars[B_FULL0 + st];
        mbar_arrive_expect_tx(fb, rank == 1 ? 3 * 16384 : 2 * 16384);
        tma_load_3d(kq, &map_k, fb, 0, hk, t0);
        tma_load_3d(kq + 8192, &map_q, fb, 0, hk, t0);
        tma_load_3d(kq + 16384, &map_k, fb, 64, hk, t0);
        tma_load_3d(kq + 16384 + 8192, &map_q, fb, 64, hk, t0);
        if (rank == 1) {
          unsigned char* vv = smem + CH_V + st * V_STAGE;
          tma_load_3d(vv, &map_v, fb, 0, h, t0);
          tma_load_3d(vv + 8192, &map_v, fb, 64, h, t0);
        }
        issued = c + 1;
      }
      // never leave the CTA with copies still landing in shared memory
      for (int c = issued - stages < 0 ? 0 : issued - stages; c < issued; ++c)
        mbar_wait(&bars[B_FULL0 + c % stages], (uint32_t)(c / stages) & 1);
    }
  } else if (rank == 0) {
    // ------------------------------------------------------------ prep CTA (512 threads) ---
    const int p = tid, pwg = p >> 7, pw = (p >> 5) & 3;
    const bool leader = (p == 0);
    float* Af = reinterpret_cast<float*>(smem + PR_AF);
    float* Tf = reinterpret_cast<float*>(smem + PR_TF);
    float* Mb = reinterpret_cast<float*>(smem + PR_MB);
    float* gl2 = reinterpret_cast<float*>(smem + PR_PV);  // gamma * log2(e) of the chunk
    float* bet = gl2 + 64;
    const uint32_t id_d1 = idesc_bf16(128, 64, 0, 0);
    const uint64_t dkq0 = sdesc_sw128(sbase + PR_KQ, 16, 1024);
    // gates of the next chunk are fetched one chunk ahead by warp 0 (asynchronous copies into
    // gx[c & 1]: g of rows 0..63, then beta); rows past the sequence end read as zero
    const float* gx = reinterpret_cast<const float*>(smem + OFF_GX);
    auto fetch_gates = [&](int c) {
      const int64_t tc = s_beg + 64 * c;
      const int Lc = (int)min((int64_t)64, s_end - tc);
      const uint32_t dst = sbase + OFF_GX + (uint32_t)(c & 1) * 512u;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int rr = 32 * hh + lane;
        const bool v = rr < Lc;
        const int64_t off = v ? (tc + rr) * P.Hv + h : 0;
        cp_async4(dst + 4u * rr, P.g + off, v);
        cp_async4(dst + 256u + 4u * rr, P.beta + off, v);
      }
      cp_async_commit();
    };
    if (warp == 0 && nchunks > 0) fetch_gates(0);
    TC_TRACE_DECL(leader);
    for (int c = 0; c < nchunks; ++c) {
      const int st = c % PR_STAGES, b = c & 1;
      unsigned char* tpl = smem + PR_TPL + b * TP_BUF;  // local staging of this chunk's [T'; P]
      bool ok = true;
      TC_TS(7);
      // D1 = [K; Q] K^T as soon as the chunk has landed
      if (leader) {
        ok = mbar_wait(&bars[B_FULL0 + st], (uint32_t)(c / PR_STAGES) & 1);
        TC_TS(8);
        if (ok) {
          tc_fence_after();
          const uint64_t dkq = dadd(dkq0, st * KQ_STAGE);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint64_t d = dadd(dkq, kstep_kmajor(ks, 16384));
            mma_bf16_ss(tmem, d, d, id_d1, ks > 0);
          }
          mma_commit(&bars[B_D1_FULL]);
        }
        TC_TS(9);
      }
      // cumulative log-decays and write strengths while D1 runs; rows past the sequence end carry
      // zero log-decay and zero beta, which makes their corrections exactly zero
      if (warp == 0) {
        cp_async_wait_all();
        __syncwarp();
        const float* gc = gx + (c & 1) * 128;
        float x0 = gc[lane], x1 = gc[32 + lane];
        const float b0 = gc[64 + lane], b1 = gc[96 + lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float y0 = __shfl_up_sync(0xffffffffu, x0, o);
          const float y1 = __shfl_up_sync(0xffffffffu, x1, o);
          if (lane >= o) {
            x0 += y0;
            x1 += y1;
          }
        }
        x1 += __shfl_sync(0xffffffffu, x0, 31);
        gl2[lane] = x0 * kLog2e;
        gl2[32 + lane] = x1 * kLog2e;
        bet[lane] = b0;
        bet[32 + lane] = b1;
        __syncwarp();
        if (c + 1 < nchunks) fetch_gates(c + 1);
      }
      TC_TS(0);
      // the chain CTA has released this chunk's [T'; P] buffer (the leader waits; the barrier
      // below orders everyone's writes after it)
      if (leader) ok = ok && mbar_wait(&bars[B_PREP_EMPTY0 + b], ((c >> 1) & 1) ^ 1);
      ok = ok && mbar_wait(&bars[B_D1_FULL], c & 1);
      if (leader && ok) mbar_arrive(&bars[B_EMPTY0 + st]);  // D1 has read this stage
      // one decision for all prep threads; also makes gl2 / bet visible to them
      if (!named_bar_and(1, TC_WORKERS, ok)) {
        fail(GDN_ERR_TIMEOUT);
        break;
      }
      TC_TS(1);
      tc_fence_after();
      {
        // warpgroup pwg owns D1 columns 16 pwg .. 16 pwg + 15 of row R = 32 pw + lane:
        // rows 0..63 are K K^T (-> A, fp32), rows 64..127 are Q K^T (-> P, bf16 to the chain CTA).
        // e^{gamma_r - gamma_s} = 2^{(gamma_r - gamma_s) log2 e}, s <= r, never above 1.
        const int R = 32 * pw + lane, r = R & 63, cs = 16 * pwg;
        float d[16], gs[16];
        tmem_ld16(tmem + ((uint32_t)(32 * pw) << 16) + cs, d);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          *reinterpret_cast<float4*>(gs + 4 * q4) = *reinterpret_cast<const float4*>(gl2 + cs + 4 * q4);
        const float gr = gl2[r];
        const float br = R < 64 ? bet[r] : 1.0f;
        tmem_ld_wait();
        float v[16];
        if (cs <= r) {
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const int s = cs + q;
            const bool keep = R < 64 ? (s < r) : (s <= r);
            v[q] = keep ? br * ex2(gr - gs[q]) * d[q] : 0.0f;
          }
        } else {  // the whole 16-column block lies above the diagonal
#pragma unroll
          for (int q = 0; q < 16; ++q) v[q] = 0.0f;
        }
        if (R < 64) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            *reinterpret_cast<float4*>(Af + r * AS + cs + 4 * q4) =
                make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
        } else {
          *reinterpret_cast<uint4*>(tpl + sw128(64 + r, cs)) = pack8(&v[0]);
          *reinterpret_cast<uint4*>(tpl + sw128(64 + r, cs + 8)) = pack8(&v[8]);
        }
      }
      tc_fence_before();
      TC_TS(2);
      named_bar(1, TC_WORKERS);  // A complete; D1 free for the next chunk
      TC_TS(3);
      // ---- T = (I + A)^{-1}.  Diagonal 16 x 16 blocks: fp32 forward substitution, one column
      // per lane (warps 0, 1: two blocks each), right-looking so that each row of the column is
      // final one FMA after the previous one.
      if (warp < 2) {
        const int blk = 2 * warp + (lane >> 4), jj = lane & 15, col = 16 * blk + jj;
        const float* ab = Af + 16 * blk * AS + 16 * blk;
        float x[16], a[16], an[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = (r == jj) ? 1.0f : 0.0f;
#pragma unroll
        for (int t = 1; t < 16; ++t) a[t] = ab[t * AS];
#pragma unroll
        for (int r = 0; r < 15; ++r) {
#pragma unroll
          for (int t = r + 2; t < 16; ++t) an[t] = ab[t * AS + r + 1];  // next column, early
#pragma unroll
          for (int t = r + 1; t < 16; ++t) x[t] = fmaf(-a[t], x[r], x[t]);
#pragma unroll
          for (int t = r + 2; t < 16; ++t) a[t] = an[t];
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Tf[(16 * blk + r) * AS + col] = x[r];
      }
      named_bar(1, TC_WORKERS);
      TC_TS(4);
      // Off-diagonal blocks by distance:  T_ij = -T_ii sum_{k=j}^{i-1} A_ik T_kj.
      // Distance 1: warps 1..3 each own block (i, i-1).
      if (warp >= 1 && warp < 4) {
        const int i = warp, j = warp - 1;
        float acc[2][4] = {};
        warp_mm16(Af + 16 * i * AS + 16 * j, AS, Tf + 16 * j * AS + 16 * j, AS, acc, lane);
        float* Mi = Mb + i * 16 * MS;
        warp_store16(Mi, MS, acc, 1.0f, lane);
        __syncwarp();
        float t2[2][4] = {};
        warp_mm16(Tf + 16 * i * AS + 16 * i, AS, Mi, MS, t2, lane);
        warp_store16(Tf + 16 * i * AS + 16 * j, AS, t2, -1.0f, lane);
      }
      named_bar(1, TC_WORKERS);
      // Distance 2: warps 2, 3 own blocks (2,0), (3,1); warp 0 meanwhile forms the part of
      // block (3,0)'s sum that is already known, A_30 T_00 + A_31 T_10.
      if (warp == 2 || warp == 3) {
        const int i = warp, j = warp - 2;
        float acc[2][4] = {};
        warp_mm16(Af + 16 * i * AS + 16 * j, AS, Tf + 16 * j * AS + 16 * j, AS, acc, lane);
        warp_mm16(Af + 16 * i * AS + 16 * (j + 1), AS, Tf + 16 * (j + 1) * AS + 16 * j, AS, acc,
                  lane);
        float* Mi = Mb + i * 16 * MS;
        warp_store16(Mi, MS, acc, 1.0f, lane);
        __syncwarp();
        float t2[2][4] = {};
        warp_mm16(Tf + 16 * i * AS + 16 * i, AS, Mi, MS, t2, lane);
        warp_store16(Tf + 16 * i * AS + 16 * j, AS, t2, -1.0f, lane);
      } else if (warp == 0) {
        float acc[2][4] = {};
        warp_mm16(Af + 48 * AS + 0, AS, Tf + 0 * AS + 0, AS, acc, lane);
        warp_mm16(Af + 48 * AS + 16, AS, Tf + 16 * AS + 0, AS, acc, lane);
        warp_store16(Mb + 0 * 16 * MS, MS, acc, 1.0f, lane);
      }
      named_bar(1, TC_WORKERS);
      // Distance 3: warp 3 owns block (3,0).
      if (warp == 3) {
        float acc[2][4];
        {
          const int g = lane >> 2, t = lane & 3;
#pragma unroll
          for (int nn = 0; nn < 2; ++nn) {
            acc[nn][0] = Mb[g * MS + 8 * nn + 2 * t];
            acc[nn][1] = Mb[g * MS + 8 * nn + 2 * t + 1];
            acc[nn][2] = Mb[(g + 8) * MS + 8 * nn + 2 * t];
            acc[nn][3] = Mb[(g + 8) * MS + 8 * nn + 2 * t + 1];
          }
        }
        warp_mm16(Af + 48 * AS + 32, AS, Tf + 32 * AS + 0, AS, acc, lane);
        float* Mi = Mb + 3 * 16 * MS;
        warp_store16(Mi, MS, acc, 1.0f, lane);
        __syncwarp();
        float t2[2][4] = {};
        warp_mm16(Tf + 48 * AS + 48, AS, Mi, MS, t2, lane);
        warp_store16(Tf + 48 * AS + 0, AS, t2, -1.0f, lane);
      }
      named_bar(1, TC_WORKERS);
      TC_TS(5);
      // T' = T diag(beta) -> rows 0..63 of the chain CTA's [T'; P] tile (bf16, K-major); zero
      // above the diagonal (the solve leaves that part of Tf unwritten).  8 columns per thread.
      {
        const int r = p >> 3, s0 = 8 * (p & 7);
        float tv[8], bv[8];
        *reinterpret_cast<float4*>(tv) = *reinterpret_cast<const float4*>(Tf + r * AS + s0);
        *reinterpret_cast<float4*>(tv + 4) = *reinterpret_cast<const float4*>(Tf + r * AS + s0 + 4);
        *reinterpret_cast<float4*>(bv) = *reinterpret_cast<const float4*>(bet + s0);
        *reinterpret_cast<float4*>(bv + 4) = *reinterpret_cast<const float4*>(bet + s0 + 4);
#pragma unroll
        for (int q = 0; q < 8; ++q) tv[q] = (s0 + q <= r) ? tv[q] * bv[q] : 0.0f;
        *reinterpret_cast<uint4*>(tpl + sw128(r, s0)) = pack8(tv);
      }
      TC_TS(10);
      fence_proxy_async_smem();  // the staged tile is read by the bulk copy (async proxy)
      TC_TS(11);
      named_bar(1, TC_WORKERS);
      TC_TS(12);
      // the chain CTA arms its barrier for these bytes itself; the copy only completes them
      if (leader) {
        bulk_copy_to_peer(peer_addr(sbase + CH_TP + b * TP_BUF, 1), smem_u32(tpl), TP_BUF,
                          peer_addr(smem_u32(&bars[B_PREP_FULL0 + b]), 1));
        *prep_issued = c + 1;
      }
      TC_TS(6);
    }
    TC_TRACE_FLUSH(2);
    if (warp == 0) cp_async_wait_all();  // no gate copy may still be landing at exit
    if (leader) {
      // every D1 MMA has completed before the CTA releases its tensor memory
      mma_commit(&bars[B_DRAIN]);
      if (!mbar_wait(&bars[B_DRAIN], 0)) report(P.status, GDN_ERR_TIMEOUT);
    }
  } else {
    // ------------------------------------------------------------ chain CTA (512 threads) --
    const int e = tid, wg = e >> 7, ew = (e >> 5) & 3;
    const bool leader = (e == 0);
    const int i = 32 * ew + lane;  // tensor-memory lane = row of S^T (dk index)
    const int jb = 32 * wg;        // this thread's 32 value columns
    const int jh = jb >> 6, jo = jb & 63;  // 64-column half of the operand tiles, offset inside
    const uint32_t lane_off = (uint32_t)(32 * ew) << 16;
    const uint32_t id_ks = idesc_bf16(128, 128, 0, 1);
    const uint32_t id_u = idesc_bf16(128, 128, 0, 1);
    const uint32_t id_s = idesc_bf16(128, 128, 1, 1);
    // operand descriptors at each tile's first k-step
    const uint64_t dKQ = sdesc_sw128(sbase + CH_KQ, 16, 1024);       // [K; Q] (K-major)
    const uint64_t dKT = sdesc_sw128(sbase + CH_KQ, 16384, 1024);    // K^T (MN-major)
    const uint64_t dSB = sdesc_sw128(sbase + CH_SB, 16384, 1024);    // S^T (MN-major)
    const uint64_t dTP = sdesc_sw128(sbase + CH_TP, 16, 1024);       // [T'; P] (K-major)
    const uint64_t dXU = sdesc_sw128(sbase + CH_XU, 8192, 1024);     // X, then U (MN-major)
    const uint64_t dDU = sdesc_sw128(sbase + CH_V, 8192, 1024);      // D U (MN-major)
    // The fp32 state lives in tensor memory (TM_S: lane i = row of S^T, 128 value columns); this
    // thread owns lane i, columns jb..jb+31.  Its bf16 copy in shared memory is step 1's operand.
    const size_t sbase_g = ((size_t)n * P.Hv + h) * 128 * 128;
    const uint32_t s_tm = tmem + TM_S + jb + lane_off;
    unsigned char* sb = smem + CH_SB + jh * 16384;
#pragma unroll
    for (int pc = 0; pc < 2; ++pc) {
      float v16[16];
#pragma unroll
      for (int jj = 0; jj < 16; ++jj)
        v16[jj] = P.S0 ? __ldg(P.S0 + sbase_g + (size_t)(jb + 16 * pc + jj) * 128 + i) : 0.0f;
      tmem_st16(s_tm + 16 * pc, v16);
      *reinterpret_cast<uint4*>(sb + sw128(i, jo + 16 * pc)) = pack8(&v16[0]);
      *reinterpret_cast<uint4*>(sb + sw128(i, jo + 16 * pc + 8)) = pack8(&v16[8]);
    }
    // log-decays of the next chunk are fetched one chunk ahead by warp 0 (asynchronous copies
    // into gx[c & 1], complete before the chunk's last barrier); rows past the end read as zero
    const float* gx = reinterpret_cast<const float*>(smem + OFF_GX);
    auto fetch_g = [&](int c) {
      const int64_t tc = s_beg + 64 * c;
      const int Lc = (int)min((int64_t)64, s_end - tc);
      const uint32_t dst = sbase + OFF_GX + (uint32_t)(c & 1) * 256u;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int rr = 32 * hh + lane;
        const bool v = rr < Lc;
        cp_async4(dst + 4u * rr, P.g + (v ? (tc + rr) * P.Hv + h : 0), v);
      }
      cp_async_commit();
    };
    if (warp == 0 && nchunks > 0) {
      fetch_g(0);
      cp_async_wait_all();
    }
    tmem_st_wait();
    fence_proxy_async_smem();
    tc_fence_before();
    named_bar(1, TC_WORKERS);
    TC_TRACE_DECL(leader || e == 64);

    // O = scale (Gamma_r (Q S0^T)_r + (P U)_r) of chunk c, rows r = i - 64 (threads of rows
    // 64..127), columns jb..jb+31
    auto write_out = [&](int c, float g_r) {
      const int64_t t0 = s_beg + 64 * c;
      const int L = (int)min((int64_t)64, s_end - t0);
      const int r = i - 64;
      const uint32_t tk = (c & 1) ? TM_KS2 : TM_KS;
      float qs[32], pu[32];
      tmem_ld16(tmem + tk + jb + lane_off, *reinterpret_cast<float(*)[16]>(qs));
      tmem_ld16(tmem + tk + jb + 16 + lane_off, *reinterpret_cast<float(*)[16]>(qs + 16));
      tmem_ld16(tmem + TM_U + jb + lane_off, *reinterpret_cast<float(*)[16]>(pu));
      tmem_ld16(tmem + TM_U + jb + 16 + lane_off, *reinterpret_cast<float(*)[16]>(pu + 16));
      tmem_ld_wait();
      if (r < L) {
        __nv_bfloat16* orow = P.out + ((t0 + r) * P.Hv + h) * 128 + jb;
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          float f[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) f[q] = P.scale * fmaf(g_r, qs[8 * c8 + q], pu[8 * c8 + q]);
          *reinterpret_cast<uint4*>(orow + 8 * c8) = pack8(f);
        }
      }
    };
    float g_row_prev = 0.0f;
    bool all_ok = true;
    int tp_consumed = 0;  // [T'; P] copies whose arrival the leader has waited for

    // Exits are decided jointly (named_bar_and): a wait that ran out in any thread makes all 512
    // leave at the same barrier.
    for (int c = 0; c < nchunks; ++c) {
      const int st = c & 1, b = c & 1;
      const uint32_t par = c & 1;
      const uint32_t tm_ks = (c & 1) ? TM_KS2 : TM_KS;
      const int64_t t0 = s_beg + 64 * c;
      const int L = (int)min((int64_t)64, s_end - t0);
      unsigned char* vt = smem + CH_V + st * V_STAGE;
      TC_TS(7);
      // in-chunk cumulative log-decay (inclusive scan over the chunk's 64 rows)
      float gl = gx[(c & 1) * 64 + lane], gh = gx[(c & 1) * 64 + 32 + lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y0 = __shfl_up_sync(0xffffffffu, gl, o);
        const float y1 = __shfl_up_sync(0xffffffffu, gh, o);
        if (lane >= o) {
          gl += y0;
          gh += y1;
        }
      }
      gh += __shfl_sync(0xffffffffu, gl, 31);
      const float glast = __shfl_sync(0xffffffffu, gh, 31);
      if (warp == 0 && c + 1 < nchunks) fetch_g(c + 1);
      // this thread's row r: i for rows 0..63, i - 64 for rows 64..127
      const float g_row = __expf((ew & 1) ? gh : gl);           // Gamma_r
      const float d_row = __expf(glast - ((ew & 1) ? gh : gl)); // e^{gamma_63 - gamma_r}
      const float gC = __expf(glast);
      // the chunk's K, Q, V have landed (step 1 needs nothing from the prep CTA)
      bool ok = mbar_wait(&bars[B_FULL0 + st], (c >> 1) & 1);
      TC_TS(0);
      // step 1: D_KS = [K; Q] S0^T
      if (leader && ok) {
        tc_fence_after();
        const uint64_t da = dadd(dKQ, st * KQ_STAGE);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_bf16_ss(tmem + tm_ks, dadd(da, kstep_kmajor(ks, 16384)), dadd(dSB, ks * 2048), id_ks,
                      ks > 0);
        mma_commit(&bars[B_M_KS]);
      }
      // S <- Gamma_L S in tensor memory while step 1 runs (step 5 then accumulates onto it; the
      // previous chunk's step 5 has completed)
      {
        float v[32];
        tmem_ld32(s_tm, v);
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) v[jj] *= gC;
        tmem_st16(s_tm, *reinterpret_cast<float(*)[16]>(v));
        tmem_st16(s_tm + 16, *reinterpret_cast<float(*)[16]>(v + 16));
        tmem_st_wait();
      }
      ok = ok && mbar_wait(&bars[B_M_KS], par);
      TC_TS(1);
      tc_fence_after();
      if (ok && ew < 2) {
        // X = V - Gamma_r (K S0^T), rows r = i, columns jb..jb+31
        float ks[32];
        uint4 vraw[4];
        tmem_ld16(tmem + tm_ks + jb + lane_off, *reinterpret_cast<float(*)[16]>(ks));
        tmem_ld16(tmem + tm_ks + jb + 16 + lane_off, *reinterpret_cast<float(*)[16]>(ks + 16));
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8)
          vraw[c8] = *reinterpret_cast<const uint4*>(vt + jh * 8192 + sw128(i, jo + 8 * c8));
        tmem_ld_wait();
        unsigned char* xu = smem + CH_XU + jh * 8192;
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          float vf[8];
          unpack8(vraw[c8], vf);
#pragma unroll
          for (int q = 0; q < 8; ++q) vf[q] = fmaf(-g_row, ks[8 * c8 + q], vf[q]);
          *reinterpret_cast<uint4*>(xu + sw128(i, jo + 8 * c8)) = pack8(vf);
        }
      }
      // meanwhile rows 64..127 (the other two warps of each warpgroup): the previous chunk's
      // output (its D_KS block and the P U rows stay valid until this chunk's step 3)
      if (ok && ew >= 2 && c >= 1) write_out(c - 1, g_row_prev);
      TC_TS(12);
      fence_proxy_async_smem();
      TC_TS(13);
      tc_fence_before();
      if (!named_bar_and(1, TC_WORKERS, ok)) {
        fail(GDN_ERR_TIMEOUT);
        all_ok = false;
        break;
      }
      TC_TS(2);
      // step 3: D_U = [T'; P] X  (needs this chunk's T' and P from the prep CTA)
      ok = !leader || mbar_wait(&bars[B_PREP_FULL0 + b], (c >> 1) & 1);
      if (leader && ok) tp_consumed = c + 1;
      // re-arm the buffer's barrier for chunk c + 2, whose copy the prep CTA can only start
      // after this chunk hands the buffer back
      if (leader && ok && c + 2 < nchunks) mbar_arrive_expect_tx(&bars[B_PREP_FULL0 + b], TP_BUF);
      if (leader && ok) {
        tc_fence_after();
        const uint64_t dt = dadd(dTP, b * TP_BUF);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_bf16_ss(tmem + TM_U, dadd(dt, ks * 32), dadd(dXU, ks * 2048), id_u, ks > 0);
        mma_commit(&bars[B_M_U]);
      }
      ok = ok && mbar_wait(&bars[B_M_U], par);
      TC_TS(3);
      tc_fence_after();
      if (ok && ew < 2) {
        // U rows 0..63 -> bf16 operands: U itself (for P U; overwrites X, whose MMA has
        // completed) and e^{gamma_63 - gamma_s} U_s (for the state increment; into this stage's
        // V buffer, which X has consumed)
        float uv[32];
        tmem_ld32(tmem + TM_U + jb + lane_off, uv);
        unsigned char* xu = smem + CH_XU + jh * 8192;
        unsigned char* ud = vt + jh * 8192;
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8)
          *reinterpret_cast<uint4*>(xu + sw128(i, jo + 8 * c8)) = pack8(&uv[8 * c8]);
#pragma unroll
        for (int q = 0; q < 32; ++q) uv[q] *= d_row;
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8)
          *reinterpret_cast<uint4*>(ud + sw128(i, jo + 8 * c8)) = pack8(&uv[8 * c8]);
      }
      TC_TS(14);
      fence_proxy_async_smem();
      TC_TS(15);
      tc_fence_before();
      if (!named_bar_and(1, TC_WORKERS, ok)) {
        fail(GDN_ERR_TIMEOUT);
        all_ok = false;
        break;
      }
      TC_TS(4);
      // steps 3b and 5: D_U = [T'; P] U (rows 64..127 are P U);  D_S += K^T (D U)
      if (leader) {
        tc_fence_after();
        const uint64_t dt = dadd(dTP, b * TP_BUF);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_bf16_ss(tmem + TM_U, dadd(dt, ks * 32), dadd(dXU, ks * 2048), id_u, ks > 0);
        const uint64_t dk = dadd(dKT, st * KQ_STAGE);
        const uint64_t dd = dadd(dDU, st * V_STAGE);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_bf16_ss(tmem + TM_S, dadd(dk, ks * 2048), dadd(dd, ks * 2048), id_s, 1);
        mma_commit(&bars[B_M_S]);
        mma_commit(&bars[B_EMPTY0 + st]);
      }
      ok = mbar_wait(&bars[B_M_S], par);
      TC_TS(5);
      tc_fence_after();
      // the [T'; P] buffer of this chunk has been read by both of its MMAs: hand it back
      if (leader && ok) mbar_arrive_peer(peer_addr(smem_u32(&bars[B_PREP_EMPTY0 + b]), 0));
      TC_TS(8);
      TC_TS(9);
      if (ok) {
        float sv[32];
        tmem_ld32(s_tm, sv);
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8)
          *reinterpret_cast<uint4*>(sb + sw128(i, jo + 8 * c8)) = pack8(&sv[8 * c8]);
        TC_TS(10);
        fence_proxy_async_smem();
        TC_TS(11);
      }
      if (warp == 0) cp_async_wait_all();  // next chunk's log-decays, visible after the barrier
      tc_fence_before();
      if (!named_bar_and(1, TC_WORKERS, ok)) {
        fail(GDN_ERR_TIMEOUT);
        all_ok = false;
        break;
      }
      g_row_prev = g_row;
      TC_TS(6);
    }
    if (all_ok && nchunks > 0 && ew >= 2) {
      tc_fence_after();
      write_out(nchunks - 1, g_row_prev);
    }
    TC_TRACE_FLUSH(leader ? 3 : 4);
    if (warp == 0) cp_async_wait_all();  // no gate copy may still be landing at exit
    if (leader) {
      // after an abort MMAs may still be in flight: wait for all of them before tensor memory
      // is read or released; if even that wait runs out, the state is not read back
      mma_commit(&bars[B_DRAIN]);
      if (!mbar_wait(&bars[B_DRAIN], 0)) fail(GDN_ERR_TIMEOUT);
    }
    named_bar(1, TC_WORKERS);  // the leader's drain result is visible to every worker
    tp_consumed_final = tp_consumed;
    if (P.S_T && !*abort_flag) {
      float sv[32];
      tmem_ld32(s_tm, sv);
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) P.S_T[sbase_g + (size_t)(jb + jj) * 128 + i] = sv[jj];
    }
  }

  // Neither CTA leaves while the other may still touch its shared memory.  After this barrier the
  // prep CTA issues nothing more; a [T'; P] copy it issued that the chain CTA never waited for
  // (only after an abort) may still be landing in the chain CTA, so the chain leader waits for
  // those arrivals (bounded) before the final barrier lets both CTAs go.
  tc_fence_before();
  cluster_sync();
  if (rank == 1 && tid == 0) {
    uint32_t issued_remote;
    asm volatile("ld.shared::cluster.u32 %0, [%1];"
                 : "=r"(issued_remote)
                 : "r"(peer_addr(smem_u32((const void*)prep_issued), 0))
                 : "memory");
    for (int c = tp_consumed_final; c < (int)issued_remote; ++c)
      if (!mbar_wait(&bars[B_PREP_FULL0 + (c & 1)], (uint32_t)(c >> 1) & 1)) {
        report(P.status, GDN_ERR_TIMEOUT);
        break;
      }
  }
  cluster_sync();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, rank == 1 ? 512 : 64);
  }
}

// ---------------------------------------------------------------- host side ---------------

cudaError_t launch_chunk_tc_impl(const void* q, const void* k, const void* v, TokStrides ts,
                                 const float* g, const float* beta, float scale, const float* S0,
                                 const int32_t* cu, int N, int B, int64_t T, int Hk, int Hv,
                                 void* out, float* S_T, int* status, unsigned long long* trace,
                                 cudaStream_t s) {
  const int64_t rows = (int64_t)B * T;
  const int64_t units = (int64_t)N * Hv;
  if (units == 0) return cudaSuccess;
  if (2 * units > 0x7fffffff) return cudaErrorInvalidConfiguration;
  CUtensorMap mq, mk, mv;
  const int64_t map_rows = rows > 0 ? rows : 1;
  if (!make_tok_map(&mq, q, Hk, map_rows, ts.q) || !make_tok_map(&mk, k, Hk, map_rows, ts.k) ||
      !make_tok_map(&mv, v, Hv, map_rows, ts.v))
    return cudaErrorInvalidValue;
  TcParams p;
  p.g = g;
  p.beta = beta;
  p.S0 = S0;
  p.cu = cu;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.S_T = S_T;
  p.status = status;
  p.trace = trace;
  p.scale = scale;
  p.N = N;
  p.Hk = Hk;
  p.Hv = Hv;
  p.T = T;
  cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * units));
  cfg.blockDim = dim3(TC_THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, chunk_tc_kernel, mq, mk, mv, p);
}

}  // namespace

cudaError_t launch_chunk_tc(const void* q, const void* k, const void* v, TokStrides ts,
                            const float* g, const float* beta, float scale, const float* S0,
                            const int32_t* cu, int N, int B, int64_t T, int Hk, int Hv, void* out,
                            float* S_T, int* status, cudaStream_t s) {
  return launch_chunk_tc_impl(q, k, v, ts, g, beta, scale, S0, cu, N, B, T, Hk, Hv, out, S_T,
                              status, nullptr, s);
}

}  // namespace gdn
