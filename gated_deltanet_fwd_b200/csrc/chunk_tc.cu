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
// One CTA per (sequence, v-head); the chunks of that chain run in order.  All five contractions are
// M = 128 tcgen05 MMAs with 128-byte-swizzled shared-memory operands:
//   D1  = [K; Q] K^T          (128 x 64,  K-dim 128)   -> K K^T and Q K^T for the prep warps
//   DKS = [K; Q] S0^T         (128 x 128, K-dim 128)   -> K S0^T (for X) and Q S0^T (for O)
//   DU  = [T'; P] X           (128 x 128, K-dim 64)    -> U in rows 0..63
//   DU  = [T'; P] U           (after U is copied out)  -> P U in rows 64..127
//   DS += K^T (D U)           (128 x 128, K-dim 64)    -> onto the decayed fp32 state, D = diag(e^{gamma_L - gamma})
// and O = scale (Gamma_r (Q S0^T)_r + (P U)_r) is formed in the output epilogue.  The fp32 state S^T
// lives in tensor memory: at the start of each chunk it is scaled by Gamma_L in place (while the
// first MMA runs) and the last MMA accumulates the chunk's increment onto it; its bf16 copy in
// shared memory is the next chunk's operand.
// Warp roles (512 threads):
//   warp 0      TMA producer: K, Q, V tiles of each chunk into a two-stage ring
//   warps 4-7   prep, running ahead of the state chain: issue D1, cumulative log-decays and write
//               strengths, the decay masks of A (fp32) and P, invert I + A
//               (fp32 forward substitution on the 16 x 16 diagonal blocks, tf32 mma.sync for the
//               off-diagonal block products), write T'
//   warps 8-15  state chain: issue the four chain MMAs from one elected thread, build X, convert U
//               (plain and decayed), write O, refresh the bf16 state operand.  Inside the chain the only
//               synchronisation is named barriers and waits on the chain's own MMA commits.
// Every mbarrier wait is bounded; a wait that runs out records GDN_ERR_TIMEOUT and the CTA winds
// down.
#include <mutex>

#include "gdn_internal.cuh"
#include "ptx.cuh"

namespace gdn {
namespace {

using namespace ptx;

constexpr int TC_THREADS = 512;
constexpr int AS = 68;  // fp32 row stride of the A and T scratch matrices (floats)
constexpr int MS = 20;  // fp32 row stride of the 16 x 16 block-product scratch

// shared-memory layout (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;          // 2 stages x [K;Q] A tile: 2 dk-halves x 128 rows x 128 B
constexpr uint32_t KQ_STAGE = 32768;
constexpr uint32_t OFF_V = 65536;       // 2 stages x V tile: 2 dv-halves x 64 rows x 128 B
constexpr uint32_t V_STAGE = 16384;
constexpr uint32_t OFF_SB = 98304;      // S^T bf16 (MN-major B operand): 2 x 128 rows x 128 B
constexpr uint32_t OFF_XU = 131072;     // X, then U (MN-major B operand): 2 x 64 rows x 128 B
constexpr uint32_t OFF_TP = 147456;     // 2 buffers x [T'; P] (K-major A): 128 rows x 128 B
constexpr uint32_t TP_BUF = 16384;
constexpr uint32_t OFF_AF = 180224;                    // fp32 A [64][AS]
constexpr uint32_t OFF_TF = OFF_AF + 64 * AS * 4;      // fp32 T [64][AS]
constexpr uint32_t OFF_MB = OFF_TF + 64 * AS * 4;      // fp32 4 x [16][MS] block products
constexpr uint32_t OFF_PV = OFF_MB + 4 * 16 * MS * 4;  // prep: a_t = e^{g_t}[64], beta[64]
constexpr uint32_t OFF_BAR = OFF_PV + 2 * 64 * 4;      // mbarriers
constexpr uint32_t N_BARS = 16;
constexpr uint32_t SMEM_USED = OFF_BAR + N_BARS * 8 + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;      // slack for 1024-byte alignment
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// tensor-memory columns
constexpr uint32_t TM_D1 = 0, TM_KS = 64, TM_U = 192, TM_S = 320;

enum {
  B_FULL0 = 0, B_FULL1, B_EMPTY0, B_EMPTY1, B_D1_FULL, B_PREP_FULL0, B_PREP_FULL1,
  B_PREP_EMPTY0, B_PREP_EMPTY1, B_M_KS, B_M_U, B_M_S, B_DRAIN_P, B_DRAIN_S, B_COUNT
};
static_assert(B_COUNT <= (int)N_BARS, "barrier space");

// Optional phase timing, compiled in only with -DGDN_TC_TRACE: per-role clock64 accumulators of
// CTA 0, written to TcParams::trace (8 slots per role) when the role finishes.
#ifdef GDN_TC_TRACE
#define TC_TRACE_DECL(active)                        \
  const bool tr_on_ = (active) && blockIdx.x == 0; \
  unsigned long long tr_acc_[8] = {};               \
  unsigned long long tr_last_ = clock64();
#define TC_TS(k)                                     \
  do {                                               \
    if (tr_on_) {                                    \
      const unsigned long long n_ = clock64();       \
      tr_acc_[k] += n_ - tr_last_;                   \
      tr_last_ = n_;                                 \
    }                                                \
  } while (0)
#define TC_TRACE_FLUSH(role)                                                    \
  do {                                                                          \
    if (tr_on_ && P.trace)                                                      \
      for (int k_ = 0; k_ < 8; ++k_) P.trace[(role) * 8 + k_] = tr_acc_[k_];   \
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

constexpr float kLog2e = 1.4426950408889634f;

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

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x / P.Hv, h = blockIdx.x % P.Hv;
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
    if (tid == 0) report(P.status, GDN_ERR_DEVICE_ARG);
    return;  // uniform across the CTA: nothing allocated yet
  }
  const int nchunks = (int)((s_end - s_beg + 63) / 64);

  if (tid == 0) {
    mbar_init(&bars[B_FULL0], 1);
    mbar_init(&bars[B_FULL1], 1);
    mbar_init(&bars[B_EMPTY0], 2);  // chain MMAs (last: step 5) done + prep done
    mbar_init(&bars[B_EMPTY1], 2);
    mbar_init(&bars[B_D1_FULL], 1);
    mbar_init(&bars[B_PREP_FULL0], 1);
    mbar_init(&bars[B_PREP_FULL1], 1);
    mbar_init(&bars[B_PREP_EMPTY0], 1);
    mbar_init(&bars[B_PREP_EMPTY1], 1);
    mbar_init(&bars[B_M_KS], 1);
    mbar_init(&bars[B_M_U], 1);
    mbar_init(&bars[B_M_S], 1);
    mbar_init(&bars[B_DRAIN_P], 1);
    mbar_init(&bars[B_DRAIN_S], 1);
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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer -----------
    if (lane == 0) {
      prefetch_tensormap(&map_q);
      prefetch_tensormap(&map_k);
      prefetch_tensormap(&map_v);
      int issued = 0;
      for (int c = 0; c < nchunks; ++c) {
        if (*abort_flag) break;
        const int st = c & 1;
        if (!mbar_wait(&bars[B_EMPTY0 + st], ((c >> 1) & 1) ^ 1)) { fail(GDN_ERR_TIMEOUT); break; }
        const int32_t t0 = (int32_t)(s_beg + 64 * c);
        unsigned char* kq = smem + OFF_KQ + st * KQ_STAGE;
        unsigned char* vv = smem + OFF_V + st * V_STAGE;
        mbar_arrive_expect_tx(&bars[B_FULL0 + st], 3 * 16384);
        tma_load_3d(kq, &map_k, &bars[B_FULL0 + st], 0, hk, t0);
        tma_load_3d(kq + 8192, &map_q, &bars[B_FULL0 + st], 0, hk, t0);
        tma_load_3d(kq + 16384, &map_k, &bars[B_FULL0 + st], 64, hk, t0);
        tma_load_3d(kq + 16384 + 8192, &map_q, &bars[B_FULL0 + st], 64, hk, t0);
        tma_load_3d(vv, &map_v, &bars[B_FULL0 + st], 0, h, t0);
        tma_load_3d(vv + 8192, &map_v, &bars[B_FULL0 + st], 64, h, t0);
        issued = c + 1;
      }
      // never leave the CTA with copies still landing in shared memory
      for (int c = issued - 2 < 0 ? 0 : issued - 2; c < issued; ++c)
        mbar_wait(&bars[B_FULL0 + (c & 1)], (c >> 1) & 1);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ prep (128 threads) ------
    const int p = tid - 128, pw = warp - 4;
    const bool leader = (p == 0);
    float* Af = reinterpret_cast<float*>(smem + OFF_AF);
    float* Tf = reinterpret_cast<float*>(smem + OFF_TF);
    float* Mb = reinterpret_cast<float*>(smem + OFF_MB);
    float* gl2 = reinterpret_cast<float*>(smem + OFF_PV);  // gamma * log2(e) of the chunk
    float* bet = gl2 + 64;
    const uint32_t id_d1 = idesc_bf16(128, 64, 0, 0);
    // gates of the next chunk are fetched one chunk ahead (prep warp 0, rows lane and 32 + lane)
    float pf_g0 = 0.0f, pf_g1 = 0.0f, pf_b0 = 0.0f, pf_b1 = 0.0f;
    auto fetch_gates = [&](int c) {
      const int64_t tc = s_beg + 64 * c;
      const int Lc = (int)min((int64_t)64, s_end - tc);
      pf_g0 = lane < Lc ? __ldg(P.g + (tc + lane) * P.Hv + h) : 0.0f;
      pf_g1 = 32 + lane < Lc ? __ldg(P.g + (tc + 32 + lane) * P.Hv + h) : 0.0f;
      pf_b0 = lane < Lc ? __ldg(P.beta + (tc + lane) * P.Hv + h) : 0.0f;
      pf_b1 = 32 + lane < Lc ? __ldg(P.beta + (tc + 32 + lane) * P.Hv + h) : 0.0f;
    };
    if (pw == 0 && nchunks > 0) fetch_gates(0);
    TC_TRACE_DECL(leader);
    for (int c = 0; c < nchunks; ++c) {
      const int st = c & 1, b = c & 1;
      unsigned char* tp = smem + OFF_TP + b * TP_BUF;
      bool ok = true;
      TC_TS(7);
      // D1 = [K; Q] K^T as soon as the chunk has landed (prep owns D1's tensor memory)
      if (leader) {
        ok = mbar_wait(&bars[B_FULL0 + st], (c >> 1) & 1);
        if (ok) {
          tc_fence_after();
          const uint32_t kqa = sbase + OFF_KQ + st * KQ_STAGE;
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t half = kqa + (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u;
            mma_bf16_ss(tmem + TM_D1, sdesc_sw128(half, 16, 1024), sdesc_sw128(half, 16, 1024),
                        id_d1, ks > 0);
          }
          mma_commit(&bars[B_D1_FULL]);
        }
      }
      // per-token decays and write strengths while D1 runs; rows past the sequence end carry
      // zero log-decay (a_t = 1) and zero beta, which makes their corrections exactly zero
      if (pw == 0) {
        float x0 = pf_g0, x1 = pf_g1;
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
        bet[lane] = pf_b0;
        bet[32 + lane] = pf_b1;
        if (c + 1 < nchunks) fetch_gates(c + 1);
      }
      TC_TS(0);
      ok = ok && mbar_wait(&bars[B_PREP_EMPTY0 + b], ((c >> 1) & 1) ^ 1) &&
           mbar_wait(&bars[B_D1_FULL], c & 1);
      // one decision for all prep threads; also makes gl2 / bet visible to them
      if (!named_bar_and(1, 128, ok)) {
        fail(GDN_ERR_TIMEOUT);
        break;
      }
      TC_TS(1);
      tc_fence_after();
      {
        // this thread's row of D1: rows 0..63 are K K^T, rows 64..127 are Q K^T
        // e^{gamma_r - gamma_s} = 2^{(gamma_r - gamma_s) log2 e}: only differences of in-chunk
        // cumulative log-decays are exponentiated (s <= r, so never above 1).  Each 32-column half
        // is loaded in full (tensor memory and shared memory) before anything is stored.
        const int r = 32 * (pw & 1) + lane;
        const float gr = gl2[r];
        const float br = pw < 2 ? bet[r] : 1.0f;
        float* arow = Af + r * AS;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float d[32], gs[32];
          tmem_ld16(tmem + TM_D1 + ((uint32_t)(32 * pw) << 16) + 32 * half,
                    *reinterpret_cast<float(*)[16]>(d));
          tmem_ld16(tmem + TM_D1 + ((uint32_t)(32 * pw) << 16) + 32 * half + 16,
                    *reinterpret_cast<float(*)[16]>(d + 16));
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            *reinterpret_cast<float4*>(gs + 4 * q4) =
                *reinterpret_cast<const float4*>(gl2 + 32 * half + 4 * q4);
          tmem_ld_wait();
          float v[32];
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            const int sidx = 32 * half + q;
            const bool keep = pw < 2 ? (sidx < r) : (sidx <= r);
            v[q] = keep ? br * ex2(gr - gs[q]) * d[q] : 0.0f;
          }
          if (pw < 2) {
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              *reinterpret_cast<float4*>(arow + 32 * half + 4 * q4) =
                  make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
          } else {
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8)
              *reinterpret_cast<uint4*>(tp + sw128(64 + r, 32 * half + 8 * q8)) = pack8(&v[8 * q8]);
          }
        }
      }
      TC_TS(2);
      named_bar(1, 128);  // A complete
      TC_TS(3);
      // ---- T = (I + A)^{-1}.  Diagonal 16 x 16 blocks: fp32 forward substitution, one column
      // per lane, four partial sums per row.
      if (pw < 2) {
        const int blk = 2 * pw + (lane >> 4), jj = lane & 15, col = 16 * blk + jj;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          const float* arow = Af + (16 * blk + r) * AS + 16 * blk;
          float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f, s3 = 0.0f;
#pragma unroll
          for (int s = 0; s < r; s += 4) {
            s0 = fmaf(arow[s], x[s], s0);
            if (s + 1 < r) s1 = fmaf(arow[s + 1], x[s + 1], s1);
            if (s + 2 < r) s2 = fmaf(arow[s + 2], x[s + 2], s2);
            if (s + 3 < r) s3 = fmaf(arow[s + 3], x[s + 3], s3);
          }
          x[r] = ((r == jj) ? 1.0f : 0.0f) - ((s0 + s1) + (s2 + s3));
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Tf[(16 * blk + r) * AS + col] = x[r];
      }
      named_bar(1, 128);
      TC_TS(4);
      // Off-diagonal blocks by distance:  T_ij = -T_ii sum_{k=j}^{i-1} A_ik T_kj.
      // Distance 1: warps 1..3 each own block (i, i-1).
      if (pw >= 1) {
        const int i = pw, j = pw - 1;
        float acc[2][4] = {};
        warp_mm16(Af + 16 * i * AS + 16 * j, AS, Tf + 16 * j * AS + 16 * j, AS, acc, lane);
        float* Mi = Mb + i * 16 * MS;
        warp_store16(Mi, MS, acc, 1.0f, lane);
        __syncwarp();
        float t2[2][4] = {};
        warp_mm16(Tf + 16 * i * AS + 16 * i, AS, Mi, MS, t2, lane);
        warp_store16(Tf + 16 * i * AS + 16 * j, AS, t2, -1.0f, lane);
      }
      named_bar(1, 128);
      // Distance 2: warps 2, 3 own blocks (2,0), (3,1); warp 0 meanwhile forms the part of
      // block (3,0)'s sum that is already known, A_30 T_00 + A_31 T_10.
      if (pw >= 2) {
        const int i = pw, j = pw - 2;
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
      } else if (pw == 0) {
        float acc[2][4] = {};
        warp_mm16(Af + 48 * AS + 0, AS, Tf + 0 * AS + 0, AS, acc, lane);
        warp_mm16(Af + 48 * AS + 16, AS, Tf + 16 * AS + 0, AS, acc, lane);
        warp_store16(Mb + 0 * 16 * MS, MS, acc, 1.0f, lane);
      }
      named_bar(1, 128);
      // Distance 3: warp 3 owns block (3,0).
      if (pw == 3) {
        float acc[2][4];
        {
          const int g = lane >> 2, t = lane & 3;
          const float* M0 = Mb;
#pragma unroll
          for (int nn = 0; nn < 2; ++nn) {
            acc[nn][0] = M0[g * MS + 8 * nn + 2 * t];
            acc[nn][1] = M0[g * MS + 8 * nn + 2 * t + 1];
            acc[nn][2] = M0[(g + 8) * MS + 8 * nn + 2 * t];
            acc[nn][3] = M0[(g + 8) * MS + 8 * nn + 2 * t + 1];
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
      named_bar(1, 128);
      TC_TS(5);
      // T' = T diag(beta) -> rows 0..63 of the [T'; P] tile (bf16, K-major); zero above the
      // diagonal (the solve leaves that part of Tf unwritten)
      {
        const int r = p >> 1, s0 = 32 * (p & 1);
        const float* trow = Tf + r * AS;
        float tv[32], bv[32];
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          *reinterpret_cast<float4*>(tv + 4 * q4) = *reinterpret_cast<const float4*>(trow + s0 + 4 * q4);
          *reinterpret_cast<float4*>(bv + 4 * q4) = *reinterpret_cast<const float4*>(bet + s0 + 4 * q4);
        }
#pragma unroll
        for (int q = 0; q < 32; ++q) tv[q] = (s0 + q <= r) ? tv[q] * bv[q] : 0.0f;
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8)
          *reinterpret_cast<uint4*>(tp + sw128(r, s0 + 8 * c8)) = pack8(&tv[8 * c8]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar(1, 128);
      if (leader) {
        mbar_arrive(&bars[B_PREP_FULL0 + b]);
        mbar_arrive(&bars[B_EMPTY0 + st]);
      }
      TC_TS(6);
    }
    TC_TRACE_FLUSH(2);
    if (leader) {
      mma_commit(&bars[B_DRAIN_P]);
      mbar_wait(&bars[B_DRAIN_P], 0);
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ state chain (256 threads) -
    const int e = tid - 256, hf = e >> 7, ew = (e >> 5) & 3;
    const bool leader = (e == 0);
    const int i = 32 * ew + lane;  // tensor-memory lane = row of S^T (dk index)
    const int jb = 64 * hf;        // this thread's 64 value columns
    const uint32_t lane_off = (uint32_t)(32 * ew) << 16;
    const uint32_t id_ks = idesc_bf16(128, 128, 0, 1);
    const uint32_t id_u = idesc_bf16(128, 128, 0, 1);
    const uint32_t id_s = idesc_bf16(128, 128, 1, 1);
    // The fp32 state lives in tensor memory (TM_S: lane i = row of S^T, 128 value columns); this
    // thread owns lane i, columns jb..jb+63.  Its bf16 copy in shared memory is step 1's operand.
    const size_t sbase_g = ((size_t)n * P.Hv + h) * 128 * 128;
    const uint32_t s_tm = tmem + TM_S + jb + lane_off;
    unsigned char* sb = smem + OFF_SB + hf * 16384;
#pragma unroll
    for (int pc = 0; pc < 4; ++pc) {
      float v16[16];
#pragma unroll
      for (int jj = 0; jj < 16; ++jj)
        v16[jj] = P.S0 ? __ldg(P.S0 + sbase_g + (size_t)(jb + 16 * pc + jj) * 128 + i) : 0.0f;
      tmem_st16(s_tm + 16 * pc, v16);
      *reinterpret_cast<uint4*>(sb + sw128(i, 16 * pc)) = pack8(&v16[0]);
      *reinterpret_cast<uint4*>(sb + sw128(i, 16 * pc + 8)) = pack8(&v16[8]);
    }
    tmem_st_wait();
    fence_proxy_async_smem();
    tc_fence_before();
    named_bar(2, 256);
    // log-decays of the next chunk are fetched one chunk ahead (rows lane and 32 + lane)
    float pg0 = 0.0f, pg1 = 0.0f;
    auto fetch_g = [&](int c) {
      const int64_t tc = s_beg + 64 * c;
      const int Lc = (int)min((int64_t)64, s_end - tc);
      pg0 = lane < Lc ? __ldg(P.g + (tc + lane) * P.Hv + h) : 0.0f;
      pg1 = 32 + lane < Lc ? __ldg(P.g + (tc + 32 + lane) * P.Hv + h) : 0.0f;
    };
    if (nchunks > 0) fetch_g(0);
    TC_TRACE_DECL(leader || e == 64);

    // Exits are decided jointly (named_bar_and): a wait that ran out in any thread makes all 256
    // leave at the same barrier.
    for (int c = 0; c < nchunks; ++c) {
      const int st = c & 1, b = c & 1;
      const uint32_t par = c & 1;
      const int64_t t0 = s_beg + 64 * c;
      const int L = (int)min((int64_t)64, s_end - t0);
      const uint32_t kqa = sbase + OFF_KQ + st * KQ_STAGE;
      const uint32_t tpa = sbase + OFF_TP + b * TP_BUF;
      unsigned char* kq = smem + OFF_KQ + st * KQ_STAGE;
      unsigned char* vt = smem + OFF_V + st * V_STAGE;
      TC_TS(7);
      // in-chunk cumulative log-decay (inclusive scan over the chunk's 64 rows)
      float gl = pg0, gh = pg1;
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
      if (c + 1 < nchunks) fetch_g(c + 1);
      // this thread's row r: i for rows 0..63, i - 64 for rows 64..127
      const float g_row = __expf((ew & 1) ? gh : gl);           // Gamma_r
      const float d_row = __expf(glast - ((ew & 1) ? gh : gl)); // e^{gamma_63 - gamma_r}
      const float gC = __expf(glast);
      // the chunk's K, Q, V have landed (step 1 needs nothing from the prep warps)
      bool ok = mbar_wait(&bars[B_FULL0 + st], (c >> 1) & 1);
      TC_TS(0);
      // step 1: D_KS = [K; Q] S0^T
      if (leader && ok) {
        tc_fence_after();
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t a = kqa + (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u;
          const uint32_t bb = sbase + OFF_SB + (uint32_t)ks * 2048u;
          mma_bf16_ss(tmem + TM_KS, sdesc_sw128(a, 16, 1024), sdesc_sw128(bb, 16384, 1024), id_ks,
                      ks > 0);
        }
        mma_commit(&bars[B_M_KS]);
      }
      // S <- Gamma_L S in tensor memory while step 1 runs (step 5 then accumulates K^T D U onto it;
      // the previous chunk's step 5 has completed)
#pragma unroll
      for (int pc = 0; pc < 2; ++pc) {
        float v[32];
        tmem_ld32(s_tm + 32 * pc, v);
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) v[jj] *= gC;
        tmem_st16(s_tm + 32 * pc, *reinterpret_cast<float(*)[16]>(v));
        tmem_st16(s_tm + 32 * pc + 16, *reinterpret_cast<float(*)[16]>(v + 16));
      }
      tmem_st_wait();
      ok = ok && mbar_wait(&bars[B_M_KS], par);
      TC_TS(1);
      tc_fence_after();
      if (!ok) {
        // skip the work; the joint barrier below takes everyone out
      } else if (ew < 2) {
        // X = V - Gamma_r (K S0^T), rows r = i
        unsigned char* xu = smem + OFF_XU + hf * 8192;
        float ks[64];
        uint4 vraw[8];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          tmem_ld16(tmem + TM_KS + jb + 16 * q + lane_off, *reinterpret_cast<float(*)[16]>(ks + 16 * q));
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8)
          vraw[c8] = *reinterpret_cast<const uint4*>(vt + hf * 8192 + sw128(i, 8 * c8));
        tmem_ld_wait();
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          float vf[8];
          unpack8(vraw[c8], vf);
#pragma unroll
          for (int q = 0; q < 8; ++q) vf[q] = fmaf(-g_row, ks[8 * c8 + q], vf[q]);
          *reinterpret_cast<uint4*>(xu + sw128(i, 8 * c8)) = pack8(vf);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      if (!named_bar_and(2, 256, ok)) {
        fail(GDN_ERR_TIMEOUT);
        break;
      }
      TC_TS(2);
      // step 3: D_U = [T'; P] X  (needs this chunk's T' and P from the prep warps; prep_full also
      // means the prep's K K^T MMA has finished reading this stage's K)
      ok = mbar_wait(&bars[B_PREP_FULL0 + b], (c >> 1) & 1);
      if (leader && ok) {
        tc_fence_after();
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t a = tpa + (uint32_t)ks * 32u;
          const uint32_t bb = sbase + OFF_XU + (uint32_t)ks * 2048u;
          mma_bf16_ss(tmem + TM_U, sdesc_sw128(a, 16, 1024), sdesc_sw128(bb, 8192, 1024), id_u,
                      ks > 0);
        }
        mma_commit(&bars[B_M_U]);
      }
      ok = ok && mbar_wait(&bars[B_M_U], par);
      TC_TS(3);
      tc_fence_after();
      if (ok && ew < 2) {
        // U rows 0..63 -> bf16 operands: U itself (for P U; overwrites X, whose MMA has
        // completed) and e^{gamma_63 - gamma_s} U_s (for the state increment K^T diag(.) U; into
        // this stage's V buffer, which X has consumed)
        unsigned char* xu = smem + OFF_XU + hf * 8192;
        unsigned char* ud = vt + hf * 8192;
#pragma unroll
        for (int pc = 0; pc < 2; ++pc) {
          float uv[32];
          tmem_ld32(tmem + TM_U + jb + 32 * pc + lane_off, uv);
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4)
            *reinterpret_cast<uint4*>(xu + sw128(i, 8 * (4 * pc + c4))) = pack8(&uv[8 * c4]);
#pragma unroll
          for (int q = 0; q < 32; ++q) uv[q] *= d_row;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4)
            *reinterpret_cast<uint4*>(ud + sw128(i, 8 * (4 * pc + c4))) = pack8(&uv[8 * c4]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      if (!named_bar_and(2, 256, ok)) {
        fail(GDN_ERR_TIMEOUT);
        break;
      }
      TC_TS(4);
      // steps 3b and 5: D_U = [T'; P] U (rows 64..127 are P U; U itself is already in shared
      // memory);  D_S += K^T (D U)
      if (leader) {
        tc_fence_after();
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t a = tpa + (uint32_t)ks * 32u;
          const uint32_t bb = sbase + OFF_XU + (uint32_t)ks * 2048u;
          mma_bf16_ss(tmem + TM_U, sdesc_sw128(a, 16, 1024), sdesc_sw128(bb, 8192, 1024), id_u,
                      ks > 0);
        }
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t a = kqa + (uint32_t)ks * 2048u;
          const uint32_t bb = sbase + OFF_V + st * V_STAGE + (uint32_t)ks * 2048u;
          mma_bf16_ss(tmem + TM_S, sdesc_sw128(a, 16384, 1024), sdesc_sw128(bb, 8192, 1024), id_s,
                      1);
        }
        mma_commit(&bars[B_M_S]);
        mma_commit(&bars[B_PREP_EMPTY0 + b]);
        mma_commit(&bars[B_EMPTY0 + st]);
      }
      ok = mbar_wait(&bars[B_M_S], par);
      TC_TS(5);
      tc_fence_after();
      if (ok && ew >= 2) {
        const int r = i - 64;
        __nv_bfloat16* orow = P.out + ((t0 + r) * P.Hv + h) * 128 + jb;
#pragma unroll
        for (int pc = 0; pc < 2; ++pc) {
          // O = scale (Gamma_r (Q S0^T)_r + (P U)_r)
          float qs[32], pu[32];
          tmem_ld16(tmem + TM_KS + jb + 32 * pc + lane_off, *reinterpret_cast<float(*)[16]>(qs));
          tmem_ld16(tmem + TM_KS + jb + 32 * pc + 16 + lane_off,
                    *reinterpret_cast<float(*)[16]>(qs + 16));
          tmem_ld16(tmem + TM_U + jb + 32 * pc + lane_off, *reinterpret_cast<float(*)[16]>(pu));
          tmem_ld16(tmem + TM_U + jb + 32 * pc + 16 + lane_off,
                    *reinterpret_cast<float(*)[16]>(pu + 16));
          tmem_ld_wait();
          if (r < L) {
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
              float f[8];
#pragma unroll
              for (int q = 0; q < 8; ++q)
                f[q] = P.scale * fmaf(g_row, qs[8 * c4 + q], pu[8 * c4 + q]);
              *reinterpret_cast<uint4*>(orow + 8 * (4 * pc + c4)) = pack8(f);
            }
          }
        }
      }
      if (ok) {
#pragma unroll
        for (int pc = 0; pc < 2; ++pc) {
          float sv[32];
          tmem_ld32(s_tm + 32 * pc, sv);
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4)
            *reinterpret_cast<uint4*>(sb + sw128(i, 32 * pc + 8 * c4)) = pack8(&sv[8 * c4]);
        }
        fence_proxy_async_smem();
      }
      tc_fence_before();
      if (!named_bar_and(2, 256, ok)) {
        fail(GDN_ERR_TIMEOUT);
        break;
      }
      TC_TS(6);
    }
    TC_TRACE_FLUSH(leader ? 3 : 4);
    if (leader) {
      mma_commit(&bars[B_DRAIN_S]);
      mbar_wait(&bars[B_DRAIN_S], 0);
    }
    if (P.S_T && !*abort_flag) {
#pragma unroll
      for (int pc = 0; pc < 2; ++pc) {
        float sv[32];
        tmem_ld32(s_tm + 32 * pc, sv);
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) P.S_T[sbase_g + (size_t)(jb + 32 * pc + jj) * 128 + i] = sv[jj];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- host side ---------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [rows, heads, 128] bf16 with `tok_stride` elements between rows -> 3D map {128, heads, rows},
// box {64, 1, 64}, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int heads, int64_t rows, int64_t tok_stride) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {128, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {128 * 2, (cuuint64_t)tok_stride * 2};
  cuuint32_t box[3] = {64, 1, 64};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

namespace {
cudaError_t launch_chunk_tc_impl(const void* q, const void* k, const void* v, TokStrides ts,
                                 const float* g,
                                 const float* beta, float scale, const float* S0,
                                 const int32_t* cu, int N, int B, int64_t T, int Hk, int Hv,
                                 void* out, float* S_T, int* status, unsigned long long* trace,
                                 cudaStream_t s) {
  const int64_t rows = (int64_t)B * T;
  const int64_t ctas = (int64_t)N * Hv;
  if (ctas == 0) return cudaSuccess;
  if (ctas > 0x7fffffff) return cudaErrorInvalidConfiguration;
  CUtensorMap mq, mk, mv;
  const int64_t map_rows = rows > 0 ? rows : 1;
  if (!make_map(&mq, q, Hk, map_rows, ts.q) || !make_map(&mk, k, Hk, map_rows, ts.k) ||
      !make_map(&mv, v, Hv, map_rows, ts.v))
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
  chunk_tc_kernel<<<(unsigned)ctas, TC_THREADS, SMEM_BYTES, s>>>(mq, mk, mv, p);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_chunk_tc(const void* q, const void* k, const void* v, TokStrides ts,
                            const float* g,
                            const float* beta, float scale, const float* S0, const int32_t* cu,
                            int N, int B, int64_t T, int Hk, int Hv, void* out, float* S_T,
                            int* status, cudaStream_t s) {
  return launch_chunk_tc_impl(q, k, v, ts, g, beta, scale, S0, cu, N, B, T, Hk, Hv, out, S_T, status,
                              nullptr, s);
}

}  // namespace gdn
