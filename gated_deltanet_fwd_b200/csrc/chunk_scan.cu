// chunk_scan.cu -- the prefix step of the intra-sequence scan of the tensor-core prefill.
//
// Method: the state map of a stretch of tokens under the gated delta rule is affine,
// S_out = S_in M + B (M the product of the per-token transitions e^{g_t}(I - beta_t k_t k_t^T), B
// the state the stretch produces from a zero state), so a sequence split into segments can carry
// its state from segment to segment by composing those maps -- the state passing between calls of
// the chunked mode ("解密Qwen3-Next的Gated DeltaNet：如何用75%混合层实现长文本高效推理" §2.2, state
// carried through initial_state), applied inside one call.  After phase 1 of the chain kernel has
// produced SOUT (the state leaving segment 0) and BSEG / MSEG of every middle segment, this kernel
// walks each long sequence's segments in order:
//     SIN_1 = SOUT,     SIN_{k+1} = SIN_k M_k + B_k      (k = 1 .. nseg - 2)
// in fp32.  Rows of S are independent, so one CTA takes 16 rows of one (sequence, v-head).
// A one-thread planner kernel, run first, picks the segment length from the actual sequence
// lengths (or none, when the extra work of the middle segments would not pay).
#include "chunk_tm.cuh"
#include "gdn_internal.cuh"
#include "ptx.cuh"

namespace gdn {
namespace {

// four groups of 64 threads split the inner dimension (32 of its 128 terms each); a thread of a
// group: 4 rows x 8 columns of the block's 16 x 128 result
constexpr int PX_GROUPS = 4;
constexpr int PX_THREADS = 64 * PX_GROUPS;
constexpr int PX_ROWS = 16;
constexpr size_t PX_SMEM =
    (2 * (size_t)tm::D * tm::D + (size_t)PX_GROUPS * PX_ROWS * tm::D) * sizeof(float);

// M_k comes in by one bulk copy per step into alternating buffers, the next one while the current
// step computes; the running rows stay in shared memory.  Register blocking (4 rows per thread)
// keeps the inner product off the shared-memory port: each M element is read once per group and
// the groups cover disjoint rows of M, so the block reads M once per step.
__global__ void __launch_bounds__(PX_THREADS) scan_prefix_kernel(
    const int32_t* __restrict__ cu, int64_t T, int N, int Hv, const int64_t* __restrict__ plan,
    int64_t max_segs, float* __restrict__ st, int* status) {
  const int64_t lseg = *plan;
  extern __shared__ __align__(16) float px_smem[];
  float* Ms = px_smem;                     // two buffers of M (128 x 128)
  float* Sr = Ms + 2 * tm::D * tm::D;      // the block's 16 rows of the running state
  float* Pp = Sr + PX_ROWS * tm::D;         // partial sums of groups 1..3
  __shared__ uint64_t bars[3];             // M buffer 0, M buffer 1, first rows
  const int n = blockIdx.x, h = blockIdx.y, r0 = PX_ROWS * blockIdx.z;
  const int tid = threadIdx.x;
  // this sequence's segment count and the global index of its first segment
  int64_t nseg = 0, seg0 = 0;
  for (int m = 0; m <= n; ++m) {
    int64_t a, b;
    if (cu) {
      a = cu[m];
      b = cu[m + 1];
      if (a < 0 || b < a || b > T) {
        if (tid == 0 && blockIdx.y == 0 && blockIdx.z == 0) report(status, GDN_ERR_DEVICE_ARG);
        return;
      }
    } else {
      a = (int64_t)m * T;
      b = a + T;
    }
    const int64_t ns = tm::seg_count(b - a, lseg);
    if (m < n) seg0 += ns; else nseg = ns;
  }
  if (nseg < 2) return;  // one chain: nothing to compose
  const size_t hs = tm::STATE_FLOATS;
  const float* sout = st + ((size_t)n * Hv + h) * hs;
  const float* bseg = st + (size_t)N * Hv * hs;
  const float* mseg = bseg + (size_t)max_segs * Hv * hs;
  float* sin_ = const_cast<float*>(mseg) + (size_t)max_segs * Hv * hs;
  auto g_of = [&](int64_t k) { return ((size_t)(seg0 + k) * Hv + h) * hs; };

  if (tid == 0) {
    for (int i = 0; i < 3; ++i) ptx::mbar_init(&bars[i], 1);
    ptx::fence_barrier_init();
  }
  __syncthreads();
  auto fetch = [&](int i, float* dst, const float* src, uint32_t bytes) {
    ptx::mbar_arrive_expect_tx(&bars[i], bytes);
    ptx::bulk_load(dst, src, bytes, &bars[i]);
  };
  if (tid == 0) {
    fetch(2, Sr, sout + (size_t)r0 * tm::D, PX_ROWS * tm::D * 4);
    if (nseg > 2) fetch(0, Ms, mseg + g_of(1), tm::D * tm::D * 4);
  }
  // every request made is waited for before the CTA can leave (bounded waits)
  bool ok = ptx::mbar_wait(&bars[2], 0);
  const int kg = tid >> 6, tt = tid & 63;          // inner-dimension group, thread in the group
  const int rg = tt >> 4, c0 = 8 * (tt & 15);      // rows 4 rg .. 4 rg + 3, columns c0 .. c0 + 7
  constexpr int LK = tm::D / PX_GROUPS;            // inner terms per group
  for (int64_t k = 1; k < nseg; ++k) {
    if (__syncthreads_and(ok)) {
      for (int e = tid; e < PX_ROWS * tm::D / 4; e += PX_THREADS)
        reinterpret_cast<float4*>(sin_ + g_of(k) + (size_t)r0 * tm::D)[e] =
            reinterpret_cast<float4*>(Sr)[e];
    }
    if (k == nseg - 1) break;
    const int buf = (int)((k - 1) & 1);
    if (tid == 0 && k + 1 <= nseg - 2)  // the other buffer was released by the previous step
      fetch(buf ^ 1, Ms + (buf ^ 1) * tm::D * tm::D, mseg + g_of(k + 1), tm::D * tm::D * 4);
    float acc[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (kg == 0) {  // group 0 starts from B_k, the others from zero
        const float4* b4 = reinterpret_cast<const float4*>(bseg + g_of(k) +
                                                           (size_t)(r0 + 4 * rg + i) * tm::D + c0);
        const float4 x0 = b4[0], x1 = b4[1];
        acc[i][0] = x0.x; acc[i][1] = x0.y; acc[i][2] = x0.z; acc[i][3] = x0.w;
        acc[i][4] = x1.x; acc[i][5] = x1.y; acc[i][6] = x1.z; acc[i][7] = x1.w;
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[i][q] = 0.0f;
      }
    }
    const bool have = ptx::mbar_wait(&bars[buf], (uint32_t)((k - 1) >> 1) & 1);
    ok = ok && have;
    if (__syncthreads_and(ok)) {
      const float* M = Ms + buf * tm::D * tm::D;
#pragma unroll 4
      for (int l = LK * kg; l < LK * (kg + 1); ++l) {
        const float4 m0 = *reinterpret_cast<const float4*>(M + l * tm::D + c0);
        const float4 m1 = *reinterpret_cast<const float4*>(M + l * tm::D + c0 + 4);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float sv = Sr[(4 * rg + i) * tm::D + l];
          acc[i][0] = fmaf(sv, m0.x, acc[i][0]); acc[i][1] = fmaf(sv, m0.y, acc[i][1]);
          acc[i][2] = fmaf(sv, m0.z, acc[i][2]); acc[i][3] = fmaf(sv, m0.w, acc[i][3]);
          acc[i][4] = fmaf(sv, m1.x, acc[i][4]); acc[i][5] = fmaf(sv, m1.y, acc[i][5]);
          acc[i][6] = fmaf(sv, m1.z, acc[i][6]); acc[i][7] = fmaf(sv, m1.w, acc[i][7]);
        }
      }
      if (kg > 0) {
        float* pp = Pp + (size_t)(kg - 1) * PX_ROWS * tm::D;
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int q = 0; q < 8; ++q) pp[(4 * rg + i) * tm::D + c0 + q] = acc[i][q];
      }
    }
    __syncthreads();  // Sr and this M buffer have been read by every thread; partials written
    if (kg == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int e = (4 * rg + i) * tm::D + c0 + q;
          Sr[e] = acc[i][q] + (Pp[e] + Pp[PX_ROWS * tm::D + e]) + Pp[2 * PX_ROWS * tm::D + e];
        }
    }
  }
  if (!ok && tid == 0) report(status, GDN_ERR_TIMEOUT);
}

// Picks the segment length of the call from the sequences' actual lengths (one thread): for each
// candidate (no scan, L1, 2 L1, 4 L1) a makespan estimate of each phase on `sms` SMs with one chain
// per SM -- the longest unit, the total work spread evenly, and whole waves of the longest units --
// plus the prefix steps; the cheapest wins.  Costs are in chunk-steps of one chain.
__global__ void scan_plan_kernel(const int32_t* __restrict__ cu, int64_t T, int N, int Hv, int sms,
                                 int64_t L1, int64_t* plan, int* status) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  const int64_t C = tm::C;
  double best_cost = 0.0;
  int64_t best = 0;
  for (int cand = 0; cand < 4; ++cand) {
    const int64_t lseg = cand == 0 ? 0 : L1 << (cand - 1);
    // phase 1 and 3: longest unit, its count, and total chunk-steps (per v-head)
    int64_t max1 = 0, cnt1 = 0, tot1 = 0, max3 = 0, cnt3 = 0, tot3 = 0, maxseg = 0;
    auto add = [](int64_t len, int64_t& mx, int64_t& cnt, int64_t& tot, int64_t times) {
      if (times <= 0) return;
      if (len > mx) {
        mx = len;
        cnt = times;
      } else if (len == mx) {
        cnt += times;
      }
      tot += len * times;
    };
    for (int m = 0; m < N; ++m) {
      int64_t a, b;
      if (cu) {
        a = cu[m];
        b = cu[m + 1];
        if (a < 0 || b < a || b > T) {
          report(status, GDN_ERR_DEVICE_ARG);
          *plan = 0;
          return;
        }
      } else {
        a = (int64_t)m * T;
        b = a + T;
      }
      const int64_t len = b - a, nseg = tm::seg_count(len, lseg);
      if (nseg <= 1) {
        add((len + C - 1) / C, max1, cnt1, tot1, 1);
      } else {
        const int64_t lc = lseg / C, tail = (len - (nseg - 1) * lseg + C - 1) / C;
        add(lc, max1, cnt1, tot1, 1 + 2 * (nseg - 2));
        add(lc, max3, cnt3, tot3, nseg - 2);
        add(tail, max3, cnt3, tot3, 1);
        if (nseg > maxseg) maxseg = nseg;
      }
    }
    auto span = [&](int64_t mx, int64_t cnt, int64_t tot) {
      const double even = (double)tot * Hv / sms;
      const double waves = (double)((cnt * Hv + sms - 1) / sms) * mx;
      double c = (double)mx;
      if (even > c) c = even;
      if (waves > c) c = waves;
      return c;
    };
    double cost = span(max1, cnt1, tot1);
    if (maxseg > 0) cost += span(max3, cnt3, tot3) + 2.0 * (double)(maxseg - 2);
    if (cand == 0 || cost < best_cost) {
      best_cost = cost;
      best = lseg;
    }
  }
  *plan = best;
}

}  // namespace

cudaError_t launch_scan_plan(const int32_t* cu, int N, int B, int64_t T, int Hv, int sms,
                             int64_t L1, void* ws, int* status, cudaStream_t s) {
  (void)B;
  int64_t* plan = reinterpret_cast<int64_t*>(reinterpret_cast<unsigned char*>(ws) + tm::PLAN_OFF);
  scan_plan_kernel<<<1, 32, 0, s>>>(cu, T, N, Hv, sms, L1, plan, status);
  return cudaGetLastError();
}

cudaError_t launch_scan_prefix(const int32_t* cu, int N, int B, int64_t T, int Hv, int64_t lseg,
                               void* ws, int* status, cudaStream_t s) {
  const int64_t n_tok = (int64_t)B * T;
  if (N == 0 || lseg <= 0) return cudaSuccess;
  const int64_t* plan =
      reinterpret_cast<const int64_t*>(reinterpret_cast<unsigned char*>(ws) + tm::PLAN_OFF);
  if (N > 0x7fffffff || Hv > 65535) return cudaErrorInvalidConfiguration;
  float* st = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(ws) +
                                       tm::states_offset(N, n_tok, Hv));
  const size_t smem = PX_SMEM;
  static bool attr_set = false;  // idempotent attribute; a benign race between host threads
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(scan_prefix_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  scan_prefix_kernel<<<dim3((unsigned)N, (unsigned)Hv, tm::D / PX_ROWS), PX_THREADS, smem, s>>>(
      cu, T, N, Hv, plan, tm::max_segs(N, n_tok, lseg), st, status);
  return cudaGetLastError();
}

}  // namespace gdn
