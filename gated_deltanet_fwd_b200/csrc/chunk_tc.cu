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
//   DKS = [K; Gamma Q] S0^T   (128 x 128, K-dim 128)   -> K S0^T (for X) and Gamma Q S0^T
//   DU  = [T'; P] X           (128 x 128, K-dim 64)    -> U in rows 0..63
//   DKS += [T'; P] U          (accumulate)             -> rows 64..127 become Gamma Q S0^T + P U = O
//   DS  = K'^T U              (128 x 128, K-dim 64)    -> the state increment (K' = decayed K)
// Warp roles (512 threads):
//   warp 0      TMA producer: K, Q, V tiles of each chunk into a two-stage ring
//   warps 4-7   prep, running ahead of the state chain: issue D1, build the decay vectors, A (fp32)
//               and P, scale Q by Gamma in place, invert I + A (fp32 forward substitution on the
//               16 x 16 diagonal blocks, tf32 mma.sync for the off-diagonal block products), write T'
//   warps 8-15  state chain: hold S^T in fp32 registers (row i of S^T, 64 columns per thread),
//               issue the four chain MMAs from one elected thread, build X, convert U, decay K
//               into K', write O, update S and its bf16 operand copy.  Inside the chain the only
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
constexpr uint32_t OFF_DEC = OFF_MB + 4 * 16 * MS * 4; // 2 x {Gamma[64], Dec[64], GammaL, pad}
constexpr uint32_t DEC_BUF = 132 * 4;
constexpr uint32_t OFF_PV = OFF_DEC + 2 * DEC_BUF;     // prep: gamma*log2(e)[64], beta[64]
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

constexpr float kLog2e = 1.4426950408889634f;

struct TcParams {
  const float* g;
  const float* beta;
  const float* S0;
  const int32_t* cu;
  __nv_bfloat16* out;
  float* S_T;
  int* status;
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
    mbar_init(&bars[B_EMPTY0], 3);  // chain MMAs done + prep done + chain read V
    mbar_init(&bars[B_EMPTY1], 3);
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
    float* gl2 = reinterpret_cast<float*>(smem + OFF_PV);  // gamma * log2(e)
    float* bet = gl2 + 64;
    const uint32_t id_d1 = idesc_bf16(128, 64, 0, 0);
    for (int c = 0; c < nchunks; ++c) {
      const int st = c & 1, b = c & 1;
      const int64_t t0 = s_beg + 64 * c;
      const int L = (int)min((int64_t)64, s_end - t0);
      unsigned char* kq = smem + OFF_KQ + st * KQ_STAGE;
      unsigned char* tp = smem + OFF_TP + b * TP_BUF;
      float* dec = reinterpret_cast<float*>(smem + OFF_DEC + b * DEC_BUF);
      bool ok = true;
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
      // decay vectors while D1 runs (warp 0 of prep); rows >= L carry zero decay, zero beta
      if (pw == 0) {
        float x0 = lane < L ? __ldg(P.g + (t0 + lane) * P.Hv + h) : 0.0f;
        float x1 = 32 + lane < L ? __ldg(P.g + (t0 + 32 + lane) * P.Hv + h) : 0.0f;
        const float b0 = lane < L ? __ldg(P.beta + (t0 + lane) * P.Hv + h) : 0.0f;
        const float b1 = 32 + lane < L ? __ldg(P.beta + (t0 + 32 + lane) * P.Hv + h) : 0.0f;
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
        const float glast = __shfl_sync(0xffffffffu, x1, 31);
        gl2[lane] = x0 * kLog2e;
        gl2[32 + lane] = x1 * kLog2e;
        bet[lane] = b0;
        bet[32 + lane] = b1;
        // the chain's copy (buffer b) is free: the chain read it at the start of chunk c - 2,
        // before it issued the MMAs whose completion prep_empty[b] (waited below) reports
        dec[lane] = __expf(x0);
        dec[32 + lane] = __expf(x1);
        dec[64 + lane] = __expf(glast - x0);
        dec[96 + lane] = __expf(glast - x1);
        if (lane == 0) dec[128] = __expf(glast);
      }
      ok = ok && mbar_wait(&bars[B_PREP_EMPTY0 + b], ((c >> 1) & 1) ^ 1) &&
           mbar_wait(&bars[B_D1_FULL], c & 1);
      // one decision for all prep threads; also makes gl2 / bet visible to them
      if (!named_bar_and(1, 128, ok)) {
        fail(GDN_ERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      {
        // this thread's row of D1: rows 0..63 are K K^T, rows 64..127 are Q K^T
        float d[64];
        tmem_ld64(tmem + TM_D1 + ((uint32_t)(32 * pw) << 16), d);
        if (pw < 2) {
          const int r = 32 * pw + lane;
          const float gr = gl2[r], br = bet[r];
          float* arow = Af + r * AS;
#pragma unroll
          for (int s4 = 0; s4 < 16; ++s4) {
            const float4 gs = *reinterpret_cast<const float4*>(gl2 + 4 * s4);
            float4 a4;
            a4.x = (4 * s4 + 0 < r) ? br * ex2(gr - gs.x) * d[4 * s4 + 0] : 0.0f;
            a4.y = (4 * s4 + 1 < r) ? br * ex2(gr - gs.y) * d[4 * s4 + 1] : 0.0f;
            a4.z = (4 * s4 + 2 < r) ? br * ex2(gr - gs.z) * d[4 * s4 + 2] : 0.0f;
            a4.w = (4 * s4 + 3 < r) ? br * ex2(gr - gs.w) * d[4 * s4 + 3] : 0.0f;
            *reinterpret_cast<float4*>(arow + 4 * s4) = a4;
          }
        } else {
          const int r = 32 * (pw - 2) + lane;
          const float gr = gl2[r];
#pragma unroll
          for (int s8 = 0; s8 < 8; ++s8) {
            const float4 ga = *reinterpret_cast<const float4*>(gl2 + 8 * s8);
            const float4 gb = *reinterpret_cast<const float4*>(gl2 + 8 * s8 + 4);
            const float gsv[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
            float pv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              pv[e] = (8 * s8 + e <= r) ? ex2(gr - gsv[e]) * d[8 * s8 + e] : 0.0f;
            *reinterpret_cast<uint4*>(tp + sw128(64 + r, 8 * s8)) = pack8(pv);
          }
        }
      }
      // Gamma Q in place (D1 has consumed the unscaled Q)
      {
        const int r = p >> 1, hh = p & 1;
        const float gq = ex2(gl2[r]);
        unsigned char* qrow = kq + hh * 16384 + 8192;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          uint4* ptr = reinterpret_cast<uint4*>(qrow + sw128(r, 8 * c8));
          float f[8];
          unpack8(*ptr, f);
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] *= gq;
          *ptr = pack8(f);
        }
      }
      named_bar(1, 128);  // A complete
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
      // T' = T diag(beta) -> rows 0..63 of the [T'; P] tile (bf16, K-major); zero above the
      // diagonal (the solve leaves that part of Tf unwritten)
      {
        const int r = p >> 1, s0 = 32 * (p & 1);
        const float* trow = Tf + r * AS;
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          const int sb = s0 + 8 * c8;
          const float4 t0v = *reinterpret_cast<const float4*>(trow + sb);
          const float4 t1v = *reinterpret_cast<const float4*>(trow + sb + 4);
          const float4 b0v = *reinterpret_cast<const float4*>(bet + sb);
          const float4 b1v = *reinterpret_cast<const float4*>(bet + sb + 4);
          float tv[8] = {t0v.x * b0v.x, t0v.y * b0v.y, t0v.z * b0v.z, t0v.w * b0v.w,
                         t1v.x * b1v.x, t1v.y * b1v.y, t1v.z * b1v.z, t1v.w * b1v.w};
#pragma unroll
          for (int e = 0; e < 8; ++e)
            if (sb + e > r) tv[e] = 0.0f;
          *reinterpret_cast<uint4*>(tp + sw128(r, sb)) = pack8(tv);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar(1, 128);
      if (leader) {
        mbar_arrive(&bars[B_PREP_FULL0 + b]);
        mbar_arrive(&bars[B_EMPTY0 + st]);
      }
    }
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
    float sreg[64];
    const size_t sbase_g = ((size_t)n * P.Hv + h) * 128 * 128;
    if (P.S0) {
#pragma unroll
      for (int jj = 0; jj < 64; ++jj)
        sreg[jj] = __ldg(P.S0 + sbase_g + (size_t)(jb + jj) * 128 + i);
    } else {
#pragma unroll
      for (int jj = 0; jj < 64; ++jj) sreg[jj] = 0.0f;
    }
    auto write_sb = [&]() {
      unsigned char* sb = smem + OFF_SB + hf * 16384;
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8)
        *reinterpret_cast<uint4*>(sb + sw128(i, 8 * c8)) = pack8(&sreg[8 * c8]);
      fence_proxy_async_smem();
    };
    write_sb();
    named_bar(2, 256);

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
      // prep for this chunk done (T', P, Gamma Q, decay vectors); the TMA data has landed
      bool ok = mbar_wait(&bars[B_PREP_FULL0 + b], (c >> 1) & 1) &&
                mbar_wait(&bars[B_FULL0 + st], (c >> 1) & 1);
      const float* dec = reinterpret_cast<const float*>(smem + OFF_DEC + b * DEC_BUF);
      const float g_row = dec[i & 63];          // Gamma_r for r = i (rows 0..63)
      const float d_row = dec[64 + (i & 63)];   // e^{gamma_63 - gamma_s} for s = i - 64
      const float gC = dec[128];
      // step 1: D_KS = [K; Gamma Q] S0^T
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
      ok = ok && mbar_wait(&bars[B_M_KS], par);
      tc_fence_after();
      if (!ok) {
        // skip the work; the joint barrier below takes everyone out
      } else if (ew < 2) {
        // X = V - Gamma_r (K S0^T), rows r = i
        unsigned char* xu = smem + OFF_XU + hf * 8192;
#pragma unroll
        for (int pc = 0; pc < 2; ++pc) {
          float ks[32];
          tmem_ld32(tmem + TM_KS + jb + 32 * pc + lane_off, ks);
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const int c8 = 4 * pc + c4;
            float vf[8];
            unpack8(*reinterpret_cast<const uint4*>(vt + hf * 8192 + sw128(i, 8 * c8)), vf);
#pragma unroll
            for (int q = 0; q < 8; ++q) vf[q] = fmaf(-g_row, ks[8 * c4 + q], vf[q]);
            *reinterpret_cast<uint4*>(xu + sw128(i, 8 * c8)) = pack8(vf);
          }
        }
      } else {
        // K' = e^{gamma_63 - gamma_s} K in place, rows s = i - 64, dk half hf
        const int s = i - 64;
        unsigned char* krow = kq + hf * 16384;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          uint4* ptr = reinterpret_cast<uint4*>(krow + sw128(s, 8 * c8));
          float f[8];
          unpack8(*ptr, f);
#pragma unroll
          for (int q = 0; q < 8; ++q) f[q] *= d_row;
          *ptr = pack8(f);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      if (!named_bar_and(2, 256, ok)) {
        fail(GDN_ERR_TIMEOUT);
        break;
      }
      // step 3: D_U = [T'; P] X
      if (leader) {
        tc_fence_after();
        mbar_arrive(&bars[B_EMPTY0 + st]);  // V of this stage consumed
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t a = tpa + (uint32_t)ks * 32u;
          const uint32_t bb = sbase + OFF_XU + (uint32_t)ks * 2048u;
          mma_bf16_ss(tmem + TM_U, sdesc_sw128(a, 16, 1024), sdesc_sw128(bb, 8192, 1024), id_u,
                      ks > 0);
        }
        mma_commit(&bars[B_M_U]);
      }
      ok = mbar_wait(&bars[B_M_U], par);
      tc_fence_after();
      if (ok && ew < 2) {
        // U rows 0..63 -> bf16 operand (overwrites X: the MMA that read X has completed)
        unsigned char* xu = smem + OFF_XU + hf * 8192;
#pragma unroll
        for (int pc = 0; pc < 2; ++pc) {
          float uv[32];
          tmem_ld32(tmem + TM_U + jb + 32 * pc + lane_off, uv);
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4)
            *reinterpret_cast<uint4*>(xu + sw128(i, 8 * (4 * pc + c4))) = pack8(&uv[8 * c4]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      if (!named_bar_and(2, 256, ok)) {
        fail(GDN_ERR_TIMEOUT);
        break;
      }
      // steps 3b and 5: D_KS += [T'; P] U (rows 64..127 become O);  D_S = K'^T U
      if (leader) {
        tc_fence_after();
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t a = tpa + (uint32_t)ks * 32u;
          const uint32_t bb = sbase + OFF_XU + (uint32_t)ks * 2048u;
          mma_bf16_ss(tmem + TM_KS, sdesc_sw128(a, 16, 1024), sdesc_sw128(bb, 8192, 1024), id_u,
                      1);
        }
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t a = kqa + (uint32_t)ks * 2048u;
          const uint32_t bb = sbase + OFF_XU + (uint32_t)ks * 2048u;
          mma_bf16_ss(tmem + TM_S, sdesc_sw128(a, 16384, 1024), sdesc_sw128(bb, 8192, 1024), id_s,
                      ks > 0);
        }
        mma_commit(&bars[B_M_S]);
        mma_commit(&bars[B_PREP_EMPTY0 + b]);
        mma_commit(&bars[B_EMPTY0 + st]);
      }
      ok = mbar_wait(&bars[B_M_S], par);
      tc_fence_after();
      if (ok && ew >= 2) {
        const int r = i - 64;
        __nv_bfloat16* orow = P.out + ((t0 + r) * P.Hv + h) * 128 + jb;
#pragma unroll
        for (int pc = 0; pc < 2; ++pc) {
          float o[32];
          tmem_ld32(tmem + TM_KS + jb + 32 * pc + lane_off, o);
          if (r < L) {
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
              float f[8];
#pragma unroll
              for (int q = 0; q < 8; ++q) f[q] = P.scale * o[8 * c4 + q];
              *reinterpret_cast<uint4*>(orow + 8 * (4 * pc + c4)) = pack8(f);
            }
          }
        }
      }
      if (ok) {
#pragma unroll
        for (int pc = 0; pc < 2; ++pc) {
          float ds[32];
          tmem_ld32(tmem + TM_S + jb + 32 * pc + lane_off, ds);
#pragma unroll
          for (int jj = 0; jj < 32; ++jj)
            sreg[32 * pc + jj] = fmaf(gC, sreg[32 * pc + jj], ds[jj]);
        }
        write_sb();
      }
      tc_fence_before();
      if (!named_bar_and(2, 256, ok)) {
        fail(GDN_ERR_TIMEOUT);
        break;
      }
    }
    if (leader) {
      mma_commit(&bars[B_DRAIN_S]);
      mbar_wait(&bars[B_DRAIN_S], 0);
    }
    if (P.S_T && !*abort_flag) {
#pragma unroll
      for (int jj = 0; jj < 64; ++jj) P.S_T[sbase_g + (size_t)(jb + jj) * 128 + i] = sreg[jj];
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

// [rows, heads, 128] bf16 -> 3D map {128, heads, rows}, box {64, 1, 64}, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int heads, int64_t rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {128, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {128 * 2, (cuuint64_t)heads * 128 * 2};
  cuuint32_t box[3] = {64, 1, 64};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_chunk_tc(const void* q, const void* k, const void* v, const float* g,
                            const float* beta, float scale, const float* S0, const int32_t* cu,
                            int N, int B, int64_t T, int Hk, int Hv, void* out, float* S_T,
                            int* status, cudaStream_t s) {
  const int64_t rows = (int64_t)B * T;
  const int64_t ctas = (int64_t)N * Hv;
  if (ctas == 0) return cudaSuccess;
  if (ctas > 0x7fffffff) return cudaErrorInvalidConfiguration;
  CUtensorMap mq, mk, mv;
  const int64_t map_rows = rows > 0 ? rows : 1;
  if (!make_map(&mq, q, Hk, map_rows) || !make_map(&mk, k, Hk, map_rows) ||
      !make_map(&mv, v, Hv, map_rows))
    return cudaErrorInvalidValue;
  TcParams p;
  p.g = g;
  p.beta = beta;
  p.S0 = S0;
  p.cu = cu;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.S_T = S_T;
  p.status = status;
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

}  // namespace gdn
