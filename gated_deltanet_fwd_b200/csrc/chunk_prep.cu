// chunk_prep.cu -- the state-independent half of the tensor-core prefill (bf16, dk = dv = 128,
// chunks of 64 tokens), fully parallel over (chunk, k-head).
//
// Method: the chunked parallel mode of "解密Qwen3-Next的Gated DeltaNet：如何用75%混合层实现长文本
// 高效推理" §2.2 applied to the gated delta rule.  Inside a chunk of L <= 64 tokens with in-chunk
// cumulative log-decays gamma_r, everything that does not depend on the state entering the chunk
// is fixed by the chunk's own keys, queries and gates:
//   A[r,s] = beta_r e^{gamma_r - gamma_s} k_r.k_s   (s < r),     T' = (I + A)^{-1} diag(beta)
//   P[r,s] = e^{gamma_r - gamma_s} q_r.k_s          (s <= r)
//   Gamma_r = e^{gamma_r},   d_s = e^{gamma_63 - gamma_s}
// so that, for a chunk entering with state S0, the corrected values are U = T'(V - diag(Gamma) K
// S0^T), the outputs scale (diag(Gamma) Q S0^T + P U) and the leaving state Gamma_63 S0 +
// U^T diag(d) K -- the chain kernel (chunk_chain.cu) evaluates those.  Only differences of
// cumulative log-decays are exponentiated, so nothing over- or underflows; rows past a sequence
// end read zero keys, queries, log-decay and beta, which makes their rows of T' and P zero.
//
// One CTA per (chunk slot, k-head): K and Q are loaded once and [K; Q] K^T is one tcgen05 MMA
// (M = 128, N = 64, K-dim 128, fp32 in tensor memory); the Hv/Hk v-heads that share the k-head
// then take their own gates: the decay masks are applied straight out of tensor memory, and
// I + A is inverted in fp32 by two warpgroups at once (one v-head each: forward substitution on
// the four 16 x 16 diagonal blocks, one column per lane, then the off-diagonal blocks by distance
// with tf32 mma.sync block products).  T', P, Gamma and d go to the workspace (layout in
// chunk_tm.cuh).
#include "chunk_tm.cuh"
#include "gdn_internal.cuh"
#include "ptx.cuh"

namespace gdn {
namespace {

using namespace ptx;

constexpr int PP_THREADS = 256;  // two warpgroups
constexpr int AS = 68;           // fp32 row stride of the A and T matrices
constexpr int MS = 20;           // fp32 row stride of the 16 x 16 block-product scratch
constexpr int PAIR = 2;          // v-heads solved side by side (one per warpgroup)

constexpr uint32_t PP_KQ = 0;                                 // [K; Q]: 2 halves x 128 x 128 B
constexpr uint32_t PP_A = 32768;                              // PAIR x fp32 [64][AS]
constexpr uint32_t PP_T = PP_A + PAIR * 64 * AS * 4;          // PAIR x fp32 [64][AS]
constexpr uint32_t PP_MB = PP_T + PAIR * 64 * AS * 4;         // PAIR x 4 x fp32 [16][MS]
constexpr uint32_t PP_GB = PP_MB + PAIR * 4 * 16 * MS * 4;    // PAIR x (gamma log2e [64], beta [64])
constexpr uint32_t PP_BAR = PP_GB + PAIR * 128 * 4;           // mbarrier, tensor-memory slot
constexpr uint32_t PP_SMEM = PP_BAR + 64 + 1024;              // + slack for 1024-byte alignment
// two CTAs per SM: the SM's 228 KB of shared memory less 1 KB the hardware reserves per CTA
static_assert(PP_SMEM <= 228 * 1024 / 2 - 1024, "two prep CTAs per SM");

constexpr float kLog2e = 1.4426950408889634f;

// Optional phase timing, compiled in only with -DGDN_PREP_TRACE: globaltimer stamps (ns) of every
// work item, 8 slots per item, written to PrepParams::trace.
#ifdef GDN_PREP_TRACE
#define PP_TS(k)                                                                   \
  do {                                                                             \
    if (P.trace && tid == 0) P.trace[(size_t)cur.it * 8 + (k)] = globaltimer_ns(); \
  } while (0)
#else
#define PP_TS(k) \
  do {           \
  } while (0)
#endif

struct PrepParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const float* g;
  const float* beta;
  const int32_t* cu;
  unsigned char* ws;  // workspace base
  int* status;
  int64_t q_stride, k_stride;  // elements between consecutive tokens
  int64_t T;
  int64_t gd_off;  // byte offset of the GD array
  int N, Hk, Hv;
  unsigned long long* trace;  // phase timing (trace builds only), else unused
  // fused gates: g and beta computed here from a, b (bf16) when a is set
  const __nv_bfloat16* a;
  const __nv_bfloat16* b;
  const float* A_log;
  const float* dt_bias;
};

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint4 pack8(const float* f) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

// T = (I + A)^{-1} for the unit lower-triangular I + A (A strictly lower, fp32 [64][AS]) by one
// warpgroup (w4 = warp within the group, bar = its named barrier).  Tf receives the lower triangle
// and the unit diagonal; above the diagonal it is left unwritten.
template <int bar>
__device__ __forceinline__ void solve64(const float* Af, float* Tf, float* Mb, int w4, int lane) {
  // diagonal 16 x 16 blocks: right-looking forward substitution, one column per lane
  if (w4 < 2) {
    const int blk = 2 * w4 + (lane >> 4), jj = lane & 15, col = 16 * blk + jj;
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
  named_bar(bar, 128);
  // off-diagonal blocks by distance:  T_ij = -T_ii sum_{k=j}^{i-1} A_ik T_kj
  if (w4 >= 1) {  // distance 1: block (w4, w4 - 1)
    const int i = w4, j = w4 - 1;
    float acc[2][4] = {};
    warp_mm16(Af + 16 * i * AS + 16 * j, AS, Tf + 16 * j * AS + 16 * j, AS, acc, lane);
    float* Mi = Mb + i * 16 * MS;
    warp_store16(Mi, MS, acc, 1.0f, lane);
    __syncwarp();
    float t2[2][4] = {};
    warp_mm16(Tf + 16 * i * AS + 16 * i, AS, Mi, MS, t2, lane);
    warp_store16(Tf + 16 * i * AS + 16 * j, AS, t2, -1.0f, lane);
  }
  named_bar(bar, 128);
  if (w4 >= 2) {  // distance 2: blocks (2,0), (3,1)
    const int i = w4, j = w4 - 2;
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
  } else if (w4 == 0) {  // meanwhile the known part of block (3,0): A_30 T_00 + A_31 T_10
    float acc[2][4] = {};
    warp_mm16(Af + 48 * AS + 0, AS, Tf + 0 * AS + 0, AS, acc, lane);
    warp_mm16(Af + 48 * AS + 16, AS, Tf + 16 * AS + 0, AS, acc, lane);
    warp_store16(Mb, MS, acc, 1.0f, lane);
  }
  named_bar(bar, 128);
  if (w4 == 3) {  // distance 3: block (3,0)
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
  named_bar(bar, 128);
}

__global__ void __launch_bounds__(PP_THREADS, 2) chunk_prep_kernel(const PrepParams P) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + PP_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + PP_BAR + 8);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = P.Hv / P.Hk;

  // ---- work items (slot, k-head), item = slot * Hk + hk, strided over the persistent CTAs
  struct Item {
    int64_t it, slot, t0, s_end;
    int hk, L;
  };
  // 1: `I` is a chunk; 0: past the last chunk (so is every later item); -1: malformed cu_seqlens
  // (reported; nothing may be read through it).  Uniform across the CTA.
  auto locate = [&](int64_t it, Item& I) -> int {
    I.it = it;
    I.slot = it / P.Hk;
    I.hk = (int)(it - I.slot * P.Hk);
    int n = -1;
    int64_t s_beg = 0;
    if (!P.cu) {
      const int64_t per = (P.T + tm::C - 1) / tm::C;
      if (per > 0 && I.slot < per * P.N) {
        n = (int)(I.slot / per);
        s_beg = (int64_t)n * P.T;
        I.s_end = s_beg + P.T;
        I.t0 = s_beg + (I.slot - (int64_t)n * per) * tm::C;
      }
    } else {
      int64_t base = 0;
      for (int m = 0; m < P.N; ++m) {
        const int64_t a = P.cu[m], b = P.cu[m + 1];
        if (a < 0 || b < a || b > P.T) {
          if (tid == 0) report(P.status, GDN_ERR_DEVICE_ARG);
          return -1;
        }
        const int64_t nch = (b - a + tm::C - 1) / tm::C;
        if (I.slot < base + nch) {
          n = m;
          I.s_end = b;
          I.t0 = a + (I.slot - base) * tm::C;
          break;
        }
        base += nch;
      }
    }
    if (n < 0) return 0;
    I.L = (int)min((int64_t)tm::C, I.s_end - I.t0);
    return 1;
  };
  // K and Q of an item into the 128-byte-swizzled [K; Q] operand, rows >= L zero-filled:
  // asynchronous per-thread copies (cp.async), waited for before the item's MMA
  auto issue_loads = [&](const Item& I) {
    constexpr int PER = 2 * 64 * 16 / PP_THREADS;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = tid + i * PP_THREADS;
      const int which = e >> 10, r = (e >> 4) & 63, ch = e & 15;
      const int half = ch >> 3, c8 = ch & 7;
      const __nv_bfloat16* src = (which ? P.q + (I.t0 + (r < I.L ? r : 0)) * P.q_stride
                                        : P.k + (I.t0 + (r < I.L ? r : 0)) * P.k_stride) +
                                 I.hk * tm::D + ch * 8;
      cp_async16_zfill(smem + PP_KQ + half * 16384 + which * 8192 + sw128(r, c8 * 8), src,
                       r < I.L ? 16u : 0u);
    }
  };

  Item cur;
  int st = locate(blockIdx.x, cur);
  if (st <= 0) return;  // nothing allocated yet
  PP_TS(0);
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 64);
    tmem_relinquish();
  }
  issue_loads(cur);
  // Once this thread's copies have landed: every thread's copies visible to the tensor core, then
  // D1 = [K; Q] K^T of the item in shared memory (rows 0..63 K K^T, rows 64..127 Q K^T; M = 128,
  // N = 64, K-dim 128) into tensor memory, completion signalled on `bar`.
  auto loads_then_mma = [&](uint32_t tmem) {
    cp_async_wait_all();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      const uint32_t id = idesc_bf16(128, 64, 0, 0);
      const uint64_t d0 = sdesc_sw128(sbase + PP_KQ, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t d = d0 + (uint64_t)(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4);
        mma_bf16_ss(tmem, d, d, id, ks > 0);
      }
      mma_commit(bar);
    }
  };
  // the tensor-memory address is visible after the barrier in the first call
  cp_async_wait_all();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  loads_then_mma(tmem);
  PP_TS(1);
  uint32_t mma_phase = 0;
  bool ok = true;
  while (st > 0 && ok) {
    const int64_t slot = cur.slot, t0 = cur.t0;
    const int hk = cur.hk, L = cur.L;
    Item nxt;
    const int nst = locate(cur.it + gridDim.x, nxt);
    float* gl2_all = reinterpret_cast<float*>(smem + PP_GB);
    const float* gxp = P.g;
    const float* bxp = P.beta;
  for (int h0 = 0; h0 < G; h0 += PAIR) {
    const int npair = min(PAIR, G - h0);
    // ---- cumulative log-decays (x log2 e) and betas of the pair's v-heads (warp gi: head gi)
    if (warp < npair) {
      const int h = hk * G + h0 + warp;
      float* gl2 = gl2_all + warp * 128;
      float x0 = 0.f, x1 = 0.f, b0 = 0.f, b1 = 0.f;
      if (P.a) {
        // the gates of the layer: beta = sigmoid(b), g = -exp(A_log) softplus(a + dt_bias)
        const float ea = expf(__ldg(P.A_log + h)), db = __ldg(P.dt_bias + h);
        if (lane < L) {
          x0 = -ea * softplusf_(__bfloat162float(P.a[(t0 + lane) * P.Hv + h]) + db);
          b0 = sigmoidf_(__bfloat162float(P.b[(t0 + lane) * P.Hv + h]));
        }
        if (32 + lane < L) {
          x1 = -ea * softplusf_(__bfloat162float(P.a[(t0 + 32 + lane) * P.Hv + h]) + db);
          b1 = sigmoidf_(__bfloat162float(P.b[(t0 + 32 + lane) * P.Hv + h]));
        }
      } else {
        if (lane < L) {
          x0 = gxp[(t0 + lane) * P.Hv + h];
          b0 = bxp[(t0 + lane) * P.Hv + h];
        }
        if (32 + lane < L) {
          x1 = gxp[(t0 + 32 + lane) * P.Hv + h];
          b1 = bxp[(t0 + 32 + lane) * P.Hv + h];
        }
      }
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
      gl2[64 + lane] = b0;
      gl2[96 + lane] = b1;
    }
    if (h0 == 0) {
      ok = mbar_wait(bar, mma_phase);
      mma_phase ^= 1;
      if (!ok) report(P.status, GDN_ERR_TIMEOUT);
    }
    tc_fence_before();
    if (!__syncthreads_and(ok)) break;
    tc_fence_after();
    // the MMA has read [K; Q]: the next item's K and Q may land there while this one is worked on
    if (h0 == 0 && nst > 0) issue_loads(nxt);
    PP_TS(2);
    // ---- decay masks straight out of tensor memory.  Thread: row R = 32 (warp & 3) + lane of
    // [K; Q], columns 32 (warp >> 2) .. + 31.  Rows 0..63 -> A (fp32, smem), 64..127 -> P (bf16,
    // workspace).  e^{gamma_r - gamma_s} = 2^{(gamma_r - gamma_s) log2 e}, never above 1.
    {
      const int R = 32 * (warp & 3) + lane, r = R & 63, cb = 32 * (warp >> 2);
      float d[32];
      tmem_ld16(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + cb, *reinterpret_cast<float(*)[16]>(d));
      tmem_ld16(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + cb + 16,
                *reinterpret_cast<float(*)[16]>(d + 16));
      tmem_ld_wait();
      for (int gi = 0; gi < npair; ++gi) {
        const int h = hk * G + h0 + gi;
        const float* gl2 = gl2_all + gi * 128;
        const float gr = gl2[r];
        const float br = R < 64 ? gl2[64 + r] : 1.0f;
        float v[32];
#pragma unroll
        for (int b16 = 0; b16 < 2; ++b16) {
          if (cb + 16 * b16 <= r) {
#pragma unroll
            for (int q = 16 * b16; q < 16 * b16 + 16; ++q) {
              const int s = cb + q;
              const bool keep = R < 64 ? (s < r) : (s <= r);
              v[q] = keep ? br * ex2f(gr - gl2[s]) * d[q] : 0.0f;
            }
          } else {  // the 16 columns lie above the diagonal
#pragma unroll
            for (int q = 16 * b16; q < 16 * b16 + 16; ++q) v[q] = 0.0f;
          }
        }
        if (R < 64) {
          float* Af = reinterpret_cast<float*>(smem + PP_A) + gi * 64 * AS;
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            *reinterpret_cast<float4*>(Af + r * AS + cb + 4 * q4) =
                make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
        } else {
          unsigned char* tp = P.ws + tm::tp_offset() + ((size_t)slot * P.Hv + h) * tm::TP_BYTES;
          uint4* dst = reinterpret_cast<uint4*>(tp + (size_t)(64 + r) * 128 + cb * 2);
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) dst[q8] = pack8(v + 8 * q8);
        }
      }
    }
    __syncthreads();  // A of every head of the pair complete
    // after the last pair's masks D1 is free: the next item's MMA runs during this item's solve
    if (h0 + PAIR >= G && nst > 0) loads_then_mma(tmem);
    PP_TS(3);
    // ---- T = (I + A)^{-1}: warpgroup gi solves head gi
    const int gi = warp >> 2, w4 = warp & 3, t4 = tid & 127;
    if (gi < npair) {
      const int h = hk * G + h0 + gi;
      const float* Af = reinterpret_cast<const float*>(smem + PP_A) + gi * 64 * AS;
      float* Tf = reinterpret_cast<float*>(smem + PP_T) + gi * 64 * AS;
      float* Mb = reinterpret_cast<float*>(smem + PP_MB) + gi * 4 * 16 * MS;
      const float* gl2 = gl2_all + gi * 128;
      if (gi == 0)
        solve64<1>(Af, Tf, Mb, w4, lane);
      else
        solve64<2>(Af, Tf, Mb, w4, lane);
      PP_TS(4);
      // T' = T diag(beta), zero above the diagonal -> rows 0..63 of the [T'; P] tile
      unsigned char* tp = P.ws + tm::tp_offset() + ((size_t)slot * P.Hv + h) * tm::TP_BYTES;
      const int r = t4 >> 1, s0 = 32 * (t4 & 1);
      float tv[32];
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        const int s = s0 + q;
        tv[q] = (s <= r) ? Tf[r * AS + s] * gl2[64 + s] : 0.0f;
      }
      uint4* dst = reinterpret_cast<uint4*>(tp + (size_t)r * 128 + s0 * 2);
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8) dst[q8] = pack8(tv + 8 * q8);
      // Gamma_r and d_s (gamma is constant past the sequence end, so gamma_63 is the chunk's total)
      if (t4 < 64) {
        float* gd = reinterpret_cast<float*>(P.ws + P.gd_off +
                                             ((size_t)slot * P.Hv + h) * tm::GD_BYTES);
        gd[t4] = ex2f(gl2[t4]);
        gd[64 + t4] = ex2f(gl2[63] - gl2[t4]);
      }
    }
    __syncthreads();  // gates / A / T buffers free for the next pair
    PP_TS(5);
  }
    cur = nxt;
    st = nst;
  }
  cp_async_wait_all();  // nothing lands in shared memory after the CTA ends
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

}  // namespace

unsigned long long* g_prep_trace = nullptr;  // trace builds: device buffer of 8 stamps per CTA

cudaError_t launch_chunk_prep(const void* q, const void* k, TokStrides ts, const float* g,
                              const float* beta, const int32_t* cu, int N, int B, int64_t T,
                              int Hk, int Hv, void* ws, int* status, cudaStream_t s,
                              const ChunkFusion& fuse) {
  const int64_t n_tok = (int64_t)B * T;
  const int64_t slots = tm::max_slots(N, n_tok);
  if (slots <= 0 || n_tok == 0) return cudaSuccess;
  if (slots > 0x7fffffff / 64) return cudaErrorInvalidConfiguration;
  PrepParams p;
  p.q = reinterpret_cast<const __nv_bfloat16*>(q);
  p.k = reinterpret_cast<const __nv_bfloat16*>(k);
  p.g = g;
  p.beta = beta;
  p.cu = cu;
  p.ws = reinterpret_cast<unsigned char*>(ws);
  p.status = status;
  p.q_stride = ts.q;
  p.k_stride = ts.k;
  p.T = T;
  p.gd_off = (int64_t)tm::gd_offset(N, n_tok, Hv);
  p.N = N;
  p.Hk = Hk;
  p.Hv = Hv;
  p.trace = g_prep_trace;
  p.a = fuse.a;
  p.b = fuse.b;
  p.A_log = fuse.A_log;
  p.dt_bias = fuse.dt_bias;
  static bool attr_set = false;  // idempotent attribute; a benign race between host threads
  static int sms = 0;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(chunk_prep_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, PP_SMEM);
    // all of the unified L1 / shared-memory space as shared memory: two CTAs per SM
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(chunk_prep_kernel,
                               cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    int dev = 0;
    if (e == cudaSuccess) e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  // persistent: two CTAs per SM, each taking every grid-th (slot, k-head) item
  const int64_t items = slots * Hk;
  const int64_t grid = items < 2 * (int64_t)sms ? items : 2 * (int64_t)sms;
  chunk_prep_kernel<<<(unsigned)grid, PP_THREADS, PP_SMEM, s>>>(p);
  return cudaGetLastError();
}

}  // namespace gdn

#ifdef GDN_PREP_TRACE
// Trace builds only: device buffer (8 stamps of 8 bytes per prep CTA) for the phase stamps.
extern "C" void gdn_debug_set_prep_trace(void* buf) {
  gdn::g_prep_trace = reinterpret_cast<unsigned long long*>(buf);
}
#endif
