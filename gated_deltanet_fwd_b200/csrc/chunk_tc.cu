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
//   warp 1      MMA issuer (one thread)
//   warps 4-7   prep, one chunk ahead of the state: reads K K^T / Q K^T from tensor memory, builds
//               A (fp32) and P, scales Q by Gamma in place, inverts I + A blockwise in fp32, writes T'
//   warps 8-15  state: hold S^T in fp32 registers (a row i of S^T and 64 of its columns per thread),
//               build X, convert U, decay K into K', write O, update S and its bf16 operand copy
// Every wait is bounded; a wait that runs out records GDN_ERR_TIMEOUT and the CTA winds down.
#include <mutex>

#include "gdn_internal.cuh"
#include "ptx.cuh"

namespace gdn {
namespace {

using namespace ptx;

constexpr int TC_THREADS = 512;
constexpr int AS = 68;  // fp32 row stride of the A and T scratch matrices (floats)

// shared-memory layout (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;          // 2 stages x [K;Q] A tile: 2 dk-halves x 128 rows x 128 B
constexpr uint32_t KQ_STAGE = 32768;
constexpr uint32_t OFF_V = 65536;       // 2 stages x V tile: 2 dv-halves x 64 rows x 128 B
constexpr uint32_t V_STAGE = 16384;
constexpr uint32_t OFF_SB = 98304;      // S^T bf16 (MN-major B operand): 2 x 128 rows x 128 B
constexpr uint32_t OFF_XU = 131072;     // X, then U (MN-major B operand): 2 x 64 rows x 128 B
constexpr uint32_t OFF_TP = 147456;     // 2 buffers x [T'; P] (K-major A): 128 rows x 128 B
constexpr uint32_t TP_BUF = 16384;
constexpr uint32_t OFF_AF = 180224;     // fp32 A [64][AS]
constexpr uint32_t OFF_TF = OFF_AF + 64 * AS * 4;   // fp32 T [64][AS]
constexpr uint32_t OFF_MB = OFF_TF + 64 * AS * 4;   // fp32 3 x [16][17] block products
constexpr uint32_t OFF_GB = OFF_MB + 3 * 16 * 17 * 4;  // prep: gamma[64], beta[64]
constexpr uint32_t OFF_BAR = OFF_GB + 2 * 64 * 4;   // mbarriers
constexpr uint32_t N_BARS = 20;
constexpr uint32_t SMEM_USED = OFF_BAR + N_BARS * 8 + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;   // slack for 1024-byte alignment

// tensor-memory columns
constexpr uint32_t TM_D1 = 0, TM_KS = 64, TM_U = 192, TM_S = 320;

// mbarrier indices
enum {
  B_FULL0 = 0, B_FULL1, B_EMPTY0, B_EMPTY1, B_D1_FULL, B_D1_EMPTY, B_Q_READY, B_PREP_FULL0,
  B_PREP_FULL1, B_PREP_EMPTY0, B_PREP_EMPTY1, B_S_READY, B_KS_FULL, B_X_READY, B_U_FULL,
  B_U_READY, B_S_FULL, B_DRAIN, B_COUNT
};
static_assert(B_COUNT <= (int)N_BARS, "barrier space");

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

// Inclusive in-chunk cumulative log-decay for rows l and 32 + l of the chunk (rows >= L count as
// zero decay).  Every lane returns gamma_l, gamma_{32+l} and gamma_63.
__device__ __forceinline__ void chunk_gamma(const float* g, int64_t t0, int L, int Hv, int h,
                                            int lane, float& gl, float& gh, float& glast) {
  float x0 = lane < L ? __ldg(g + (t0 + lane) * Hv + h) : 0.0f;
  float x1 = 32 + lane < L ? __ldg(g + (t0 + 32 + lane) * Hv + h) : 0.0f;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y0 = __shfl_up_sync(0xffffffffu, x0, o);
    const float y1 = __shfl_up_sync(0xffffffffu, x1, o);
    if (lane >= o) {
      x0 += y0;
      x1 += y1;
    }
  }
  const float tot0 = __shfl_sync(0xffffffffu, x0, 31);
  x1 += tot0;
  gl = x0;
  gh = x1;
  glast = __shfl_sync(0xffffffffu, x1, 31);
}

__global__ void __launch_bounds__(TC_THREADS, 1) chunk_tc_kernel(
    const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
    const __grid_constant__ CUtensorMap map_v, const TcParams P) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
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
  const bool bad_seq = P.cu && (s_beg < 0 || s_end < s_beg || s_end > P.T);
  if (bad_seq) {
    if (tid == 0) report(P.status, GDN_ERR_DEVICE_ARG);
    return;  // uniform across the CTA: nothing allocated yet
  }
  const int nchunks = (int)((s_end - s_beg + 63) / 64);

  if (tid == 0) {
    mbar_init(&bars[B_FULL0], 1);
    mbar_init(&bars[B_FULL1], 1);
    mbar_init(&bars[B_EMPTY0], 10);
    mbar_init(&bars[B_EMPTY1], 10);
    mbar_init(&bars[B_D1_FULL], 1);
    mbar_init(&bars[B_D1_EMPTY], 4);
    mbar_init(&bars[B_Q_READY], 1);
    // one "prep done" barrier per [T'; P] buffer: the prep warps may finish chunk c+1 before the
    // MMA thread waits for chunk c, and a single barrier would then complete two phases unseen
    mbar_init(&bars[B_PREP_FULL0], 1);
    mbar_init(&bars[B_PREP_FULL1], 1);
    mbar_init(&bars[B_PREP_EMPTY0], 1);
    mbar_init(&bars[B_PREP_EMPTY1], 1);
    mbar_init(&bars[B_S_READY], 8);
    mbar_init(&bars[B_KS_FULL], 1);
    mbar_init(&bars[B_X_READY], 8);
    mbar_init(&bars[B_U_FULL], 1);
    mbar_init(&bars[B_U_READY], 8);
    mbar_init(&bars[B_S_FULL], 1);
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
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer -------------
    if (lane == 0 && nchunks > 0) {
      const uint32_t id_d1 = idesc_bf16(128, 64, 0, 0);
      const uint32_t id_ks = idesc_bf16(128, 128, 0, 1);
      const uint32_t id_u = idesc_bf16(128, 128, 0, 1);
      const uint32_t id_s = idesc_bf16(128, 128, 1, 1);
      auto issue_d1 = [&](int c) {
        const uint32_t kq = sbase + OFF_KQ + (c & 1) * KQ_STAGE;
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t half = kq + (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u;
          mma_bf16_ss(tmem + TM_D1, sdesc_sw128(half, 16, 1024), sdesc_sw128(half, 16, 1024), id_d1,
                      ks > 0);
        }
        mma_commit(&bars[B_D1_FULL]);
      };
      bool ok = mbar_wait(&bars[B_FULL0], 0);
      if (!ok) fail(GDN_ERR_TIMEOUT);
      if (ok) {
        tc_fence_after();
        issue_d1(0);
      }
      for (int c = 0; ok && c < nchunks; ++c) {
        if (*abort_flag) break;
        const uint32_t par = c & 1;
        const uint32_t kq = sbase + OFF_KQ + (c & 1) * KQ_STAGE;
        const uint32_t tp = sbase + OFF_TP + (c & 1) * TP_BUF;
        // step 1: D_KS = [K; Gamma Q] S0^T
        if (!mbar_wait(&bars[B_S_READY], par) || !mbar_wait(&bars[B_Q_READY], par)) {
          fail(GDN_ERR_TIMEOUT);
          break;
        }
        tc_fence_after();
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t a = kq + (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u;
          const uint32_t b = sbase + OFF_SB + (uint32_t)ks * 2048u;
          mma_bf16_ss(tmem + TM_KS, sdesc_sw128(a, 16, 1024), sdesc_sw128(b, 16384, 1024), id_ks,
                      ks > 0);
        }
        mma_commit(&bars[B_KS_FULL]);
        // next chunk's K K^T / Q K^T while this chunk's state work proceeds
        if (c + 1 < nchunks) {
          if (!mbar_wait(&bars[B_FULL0 + ((c + 1) & 1)], ((c + 1) >> 1) & 1) ||
              !mbar_wait(&bars[B_D1_EMPTY], par)) {
            fail(GDN_ERR_TIMEOUT);
            break;
          }
          tc_fence_after();
          issue_d1(c + 1);
        }
        // step 3: D_U = [T'; P] X
        if (!mbar_wait(&bars[B_X_READY], par) ||
            !mbar_wait(&bars[B_PREP_FULL0 + (c & 1)], (c >> 1) & 1)) {
          fail(GDN_ERR_TIMEOUT);
          break;
        }
        tc_fence_after();
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t a = tp + (uint32_t)ks * 32u;
          const uint32_t b = sbase + OFF_XU + (uint32_t)ks * 2048u;
          mma_bf16_ss(tmem + TM_U, sdesc_sw128(a, 16, 1024), sdesc_sw128(b, 8192, 1024), id_u,
                      ks > 0);
        }
        mma_commit(&bars[B_U_FULL]);
        // steps 3b and 5: D_KS += [T'; P] U  (rows 64..127 become O);  D_S = K'^T U
        if (!mbar_wait(&bars[B_U_READY], par)) {
          fail(GDN_ERR_TIMEOUT);
          break;
        }
        tc_fence_after();
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t a = tp + (uint32_t)ks * 32u;
          const uint32_t b = sbase + OFF_XU + (uint32_t)ks * 2048u;
          mma_bf16_ss(tmem + TM_KS, sdesc_sw128(a, 16, 1024), sdesc_sw128(b, 8192, 1024), id_u, 1);
        }
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t a = kq + (uint32_t)ks * 2048u;
          const uint32_t b = sbase + OFF_XU + (uint32_t)ks * 2048u;
          mma_bf16_ss(tmem + TM_S, sdesc_sw128(a, 16384, 1024), sdesc_sw128(b, 8192, 1024), id_s,
                      ks > 0);
        }
        mma_commit(&bars[B_S_FULL]);
        mma_commit(&bars[B_PREP_EMPTY0 + (c & 1)]);
        mma_commit(&bars[B_EMPTY0 + (c & 1)]);
      }
      // drain: every MMA issued has completed before the CTA frees tensor memory
      mma_commit(&bars[B_DRAIN]);
      mbar_wait(&bars[B_DRAIN], 0);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ prep (128 threads) ------
    const int p = tid - 128, pw = warp - 4;
    float* Af = reinterpret_cast<float*>(smem + OFF_AF);
    float* Tf = reinterpret_cast<float*>(smem + OFF_TF);
    float* Mb = reinterpret_cast<float*>(smem + OFF_MB);
    float* gam_s = reinterpret_cast<float*>(smem + OFF_GB);
    float* bet_s = gam_s + 64;
    for (int c = 0; c < nchunks; ++c) {
      if (*abort_flag) break;
      const uint32_t par = c & 1;
      const int64_t t0 = s_beg + 64 * c;
      const int L = (int)min((int64_t)64, s_end - t0);
      unsigned char* kq = smem + OFF_KQ + (c & 1) * KQ_STAGE;
      unsigned char* tp = smem + OFF_TP + (c & 1) * TP_BUF;
      float gl, gh, glast;
      chunk_gamma(P.g, t0, L, P.Hv, h, lane, gl, gh, glast);
      if (pw == 0) {
        gam_s[lane] = gl;
        gam_s[32 + lane] = gh;
        bet_s[lane] = lane < L ? __ldg(P.beta + (t0 + lane) * P.Hv + h) : 0.0f;
        bet_s[32 + lane] = 32 + lane < L ? __ldg(P.beta + (t0 + 32 + lane) * P.Hv + h) : 0.0f;
      }
      named_bar(1, 128);
      bool ok = mbar_wait(&bars[B_D1_FULL], par) && mbar_wait(&bars[B_FULL0 + (c & 1)], (c >> 1) & 1) &&
                mbar_wait(&bars[B_PREP_EMPTY0 + (c & 1)], ((c >> 1) & 1) ^ 1);
      if (!ok) fail(GDN_ERR_TIMEOUT);
      if (*abort_flag) break;
      tc_fence_after();
      {
        // this thread's row of D1: rows 0..63 are K K^T, rows 64..127 are Q K^T
        float d[64];
        tmem_ld64(tmem + TM_D1 + ((uint32_t)(32 * pw) << 16), d);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_D1_EMPTY]);
        if (pw < 2) {
          const int r = 32 * pw + lane;
          const float gr = gam_s[r], br = bet_s[r];
          float* arow = Af + r * AS;
#pragma unroll
          for (int s4 = 0; s4 < 16; ++s4) {
            float4 a4;
            float* av = reinterpret_cast<float*>(&a4);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int s = 4 * s4 + e;
              av[e] = s < r ? br * __expf(gr - gam_s[s]) * d[s] : 0.0f;
            }
            *reinterpret_cast<float4*>(arow + 4 * s4) = a4;
          }
        } else {
          const int r = 32 * (pw - 2) + lane;
          const float gr = gam_s[r];
#pragma unroll
          for (int s8 = 0; s8 < 8; ++s8) {
            float pv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int s = 8 * s8 + e;
              pv[e] = s <= r ? __expf(gr - gam_s[s]) * d[s] : 0.0f;
            }
            *reinterpret_cast<uint4*>(tp + sw128(64 + r, 8 * s8)) = pack8(pv);
          }
        }
      }
      // Gamma Q in place (Q K^T above has consumed the unscaled Q)
      {
        const int r = p >> 1, hh = p & 1;
        const float gq = __expf(gam_s[r]);
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
      fence_proxy_async_smem();
      named_bar(1, 128);
      if (p == 0) {
        mbar_arrive(&bars[B_Q_READY]);
        mbar_arrive(&bars[B_EMPTY0 + (c & 1)]);
      }
      // T = (I + A)^{-1}, blockwise: 16 x 16 diagonal blocks by forward substitution, then the
      // off-diagonal blocks by distance, T_ij = -T_ii sum_{k=j}^{i-1} A_ik T_kj.
      if (p < 64) {
        const int b = p >> 4, jj = p & 15, col = 16 * b + jj;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          float acc = (r == jj) ? 1.0f : 0.0f;
          const float* arow = Af + (16 * b + r) * AS + 16 * b;
#pragma unroll
          for (int s = 0; s < r; ++s) acc = fmaf(-arow[s], x[s], acc);
          x[r] = acc;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Tf[(16 * b + r) * AS + col] = x[r];
      }
      named_bar(1, 128);
      for (int dist = 1; dist <= 3; ++dist) {
        const int nout = (4 - dist) * 256;
        for (int e = p; e < nout; e += 128) {
          const int blk = e >> 8, i = blk + dist, j = blk, r = (e >> 4) & 15, cc = e & 15;
          float acc = 0.0f;
          for (int kb = j; kb < i; ++kb) {
            const float* arow = Af + (16 * i + r) * AS + 16 * kb;
            const float* tcol = Tf + (16 * kb) * AS + 16 * j + cc;
#pragma unroll
            for (int s = 0; s < 16; ++s) acc = fmaf(arow[s], tcol[s * AS], acc);
          }
          Mb[(blk * 16 + r) * 17 + cc] = acc;
        }
        named_bar(1, 128);
        for (int e = p; e < nout; e += 128) {
          const int blk = e >> 8, i = blk + dist, j = blk, r = (e >> 4) & 15, cc = e & 15;
          const float* trow = Tf + (16 * i + r) * AS + 16 * i;
          float acc = 0.0f;
#pragma unroll
          for (int s = 0; s < 16; ++s)
            if (s <= r) acc = fmaf(trow[s], Mb[(blk * 16 + s) * 17 + cc], acc);
          Tf[(16 * i + r) * AS + 16 * j + cc] = -acc;
        }
        named_bar(1, 128);
      }
      // T' = T diag(beta) -> rows 0..63 of the [T'; P] tile (bf16, K-major)
      {
        const int r = p >> 1, s0 = 32 * (p & 1);
        const float* trow = Tf + r * AS;
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          float tv[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int s = s0 + 8 * c8 + e;
            tv[e] = s <= r ? trow[s] * bet_s[s] : 0.0f;
          }
          *reinterpret_cast<uint4*>(tp + sw128(r, s0 + 8 * c8)) = pack8(tv);
        }
      }
      fence_proxy_async_smem();
      named_bar(1, 128);
      if (p == 0) mbar_arrive(&bars[B_PREP_FULL0 + (c & 1)]);
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ state (256 threads) -----
    const int e = tid - 256, hf = e >> 7, ew = (e >> 5) & 3;
    const int i = 32 * ew + lane;  // tensor-memory lane = row of S^T (dk index)
    const int jb = 64 * hf;        // this thread's 64 value columns
    const uint32_t lane_off = (uint32_t)(32 * ew) << 16;
    float sreg[64];
    const size_t sbase_g = ((size_t)n * P.Hv + h) * 128 * 128;
    if (P.S0) {
#pragma unroll
      for (int jj = 0; jj < 64; ++jj) sreg[jj] = __ldg(P.S0 + sbase_g + (size_t)(jb + jj) * 128 + i);
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
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars[B_S_READY]);

    for (int c = 0; c < nchunks; ++c) {
      if (*abort_flag) break;
      const uint32_t par = c & 1;
      const int64_t t0 = s_beg + 64 * c;
      const int L = (int)min((int64_t)64, s_end - t0);
      unsigned char* kq = smem + OFF_KQ + (c & 1) * KQ_STAGE;
      unsigned char* vt = smem + OFF_V + (c & 1) * V_STAGE;
      float gl, gh, glast;
      chunk_gamma(P.g, t0, L, P.Hv, h, lane, gl, gh, glast);
      if (!mbar_wait(&bars[B_KS_FULL], par) || !mbar_wait(&bars[B_FULL0 + (c & 1)], (c >> 1) & 1)) {
        fail(GDN_ERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      if (ew < 2) {
        // X = V - Gamma_r (K S0^T), rows r = i
        const int r = i;
        const float gr = __expf(ew == 0 ? gl : gh);
        unsigned char* xu = smem + OFF_XU + hf * 8192;
#pragma unroll
        for (int pc = 0; pc < 2; ++pc) {
          float ks[32];
          tmem_ld32(tmem + TM_KS + jb + 32 * pc + lane_off, ks);
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const int c8 = 4 * pc + c4;
            float vf[8];
            unpack8(*reinterpret_cast<const uint4*>(vt + hf * 8192 + sw128(r, 8 * c8)), vf);
#pragma unroll
            for (int q = 0; q < 8; ++q) vf[q] = fmaf(-gr, ks[8 * c4 + q], vf[q]);
            *reinterpret_cast<uint4*>(xu + sw128(r, 8 * c8)) = pack8(vf);
          }
        }
      } else {
        // K' = e^{gamma_63 - gamma_s} K in place, rows s, dk half hf
        const int s = i - 64;
        const float dec = __expf(glast - (ew == 2 ? gl : gh));
        unsigned char* krow = kq + hf * 16384;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          uint4* ptr = reinterpret_cast<uint4*>(krow + sw128(s, 8 * c8));
          float f[8];
          unpack8(*ptr, f);
#pragma unroll
          for (int q = 0; q < 8; ++q) f[q] *= dec;
          *ptr = pack8(f);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars[B_X_READY]);
        mbar_arrive(&bars[B_EMPTY0 + (c & 1)]);
      }
      // U rows 0..63 -> bf16 operand (overwrites X: the MMA that read X has completed)
      if (!mbar_wait(&bars[B_U_FULL], par)) {
        fail(GDN_ERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      if (ew < 2) {
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
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_U_READY]);
      // outputs and the state carried to the next chunk
      if (!mbar_wait(&bars[B_S_FULL], par)) {
        fail(GDN_ERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      if (ew >= 2) {
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
      {
        const float gC = __expf(glast);
#pragma unroll
        for (int pc = 0; pc < 2; ++pc) {
          float ds[32];
          tmem_ld32(tmem + TM_S + jb + 32 * pc + lane_off, ds);
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) sreg[32 * pc + jj] = fmaf(gC, sreg[32 * pc + jj], ds[jj]);
        }
      }
      write_sb();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_S_READY]);
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
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
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
  cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  chunk_tc_kernel<<<(unsigned)ctas, TC_THREADS, SMEM_BYTES, s>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

}  // namespace gdn
