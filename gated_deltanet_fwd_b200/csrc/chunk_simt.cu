// chunk_simt.cu -- chunk-parallel gated delta rule on CUDA cores (fp32 FFMA).
//
// Serves the all-fp32 mode and every shape the tensor-core path does not (dk, dv <= 128 in
// multiples of 16, chunk 16/32/64).  Source of the method: the chunked parallel mode
// (chunk_gated_delta_rule) of "解密Qwen3-Next的Gated DeltaNet：如何用75%混合层实现长文本高效推理"
// §2.2 -- parallel inside a chunk, state carried from chunk to chunk.
//
// Chunk form (exact re-association of the token recurrence).  For a chunk of L tokens with state
// S0 on entry, gamma_r = sum_{s<=r} g_s (inside the chunk), and u_r the per-token correction,
//     (I + A) U = diag(beta) (V - diag(e^gamma) K S0^T),   A[r,s] = beta_r e^{gamma_r-gamma_s} k_r.k_s (s<r)
//     O         = scale (diag(e^gamma) Q S0^T + (M o Q K^T) U),   M[r,s] = e^{gamma_r-gamma_s} (s<=r)
//     S_L       = e^{gamma_L} S0 + U^T diag(e^{gamma_L-gamma}) K
// The unit-lower triangular system is solved by forward substitution, one column of U per
// thread.  Only differences of in-chunk cumulative log-decays are exponentiated, so nothing
// under- or overflows whatever the decay.
//
// One block per (sequence, v-head, slice of <= 64 value rows); the state slice and the chunk's
// K, Q, V live in shared memory (rows padded by one float against bank conflicts).
#include "gdn_internal.cuh"

namespace gdn {

constexpr int SIMT_THREADS = 256;
constexpr int SIMT_DVS = 64;  // value rows per block

template <typename T>
__global__ void __launch_bounds__(SIMT_THREADS) chunk_simt_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, TokStrides ts,
    const float* __restrict__ g, const float* __restrict__ beta, float scale,
    const float* __restrict__ S0, const int32_t* __restrict__ cu, int N, int64_t Tlen, int Hk,
    int Hv, int dk, int dv, int C, T* __restrict__ out, float* __restrict__ S_T,
    int* __restrict__ status) {
  extern __shared__ float smem[];
  const int slices = (dv + SIMT_DVS - 1) / SIMT_DVS;
  const int bid = blockIdx.x;
  const int sl = bid % slices;
  const int h = (bid / slices) % Hv;
  const int n = bid / (slices * Hv);
  const int hk = h / (Hv / Hk);
  const int j0 = sl * SIMT_DVS;
  const int DVS = min(SIMT_DVS, dv - j0);
  const int tid = threadIdx.x;

  const int dkp = dk + 1, dvp = DVS + 1, cp = C + 1;
  float* Ss = smem;                 // [DVS][dk+1]
  float* Ks = Ss + SIMT_DVS * dkp;  // [C][dk+1]
  float* Qs = Ks + C * dkp;         // [C][dk+1]
  float* Vs = Qs + C * dkp;         // [C][DVS+1]  V -> right-hand side -> U
  float* Xs = Vs + C * (SIMT_DVS + 1);  // [C][DVS+1]  K S0^T, then Q S0^T
  float* As = Xs + C * (SIMT_DVS + 1);  // [C][C+1]    A, then M o Q K^T
  float* gam = As + C * cp;             // [C] cumulative log-decay
  float* bet = gam + C;                 // [C]
  float* dec = bet + C;                 // [C] e^{gamma_L - gamma_s}

  int64_t s_beg, s_end;
  if (cu) {
    s_beg = cu[n];
    s_end = cu[n + 1];
    if (s_beg < 0 || s_end < s_beg || s_end > Tlen) {
      report(status, GDN_ERR_DEVICE_ARG);
      return;
    }
  } else {
    s_beg = (int64_t)n * Tlen;
    s_end = s_beg + Tlen;
  }

  // state slice in
  const int64_t sbase = ((int64_t)n * Hv + h) * dv * dk;
  for (int e = tid; e < DVS * dk; e += SIMT_THREADS) {
    const int j = e / dk, i = e - j * dk;
    Ss[j * dkp + i] = S0 ? S0[sbase + (int64_t)(j0 + j) * dk + i] : 0.0f;
  }

  for (int64_t c_beg = s_beg; c_beg < s_end; c_beg += C) {
    const int L = (int)min((int64_t)C, s_end - c_beg);
    __syncthreads();  // previous chunk finished with every buffer
    // ---- load the chunk
    for (int e = tid; e < L * dk; e += SIMT_THREADS) {
      const int r = e / dk, i = e - r * dk;
      Ks[r * dkp + i] = to_f(k[(c_beg + r) * ts.k + hk * dk + i]);
      Qs[r * dkp + i] = to_f(q[(c_beg + r) * ts.q + hk * dk + i]);
    }
    for (int e = tid; e < L * DVS; e += SIMT_THREADS) {
      const int r = e / DVS, j = e - r * DVS;
      Vs[r * dvp + j] = to_f(v[(c_beg + r) * ts.v + h * dv + j0 + j]);
    }
    if (tid == 0) {
      float acc = 0.0f;
      for (int r = 0; r < L; ++r) {
        acc += g[(c_beg + r) * Hv + h];
        gam[r] = acc;
        bet[r] = beta[(c_beg + r) * Hv + h];
      }
      for (int r = 0; r < L; ++r) dec[r] = expf(acc - gam[r]);
    }
    __syncthreads();
    // ---- X = K S0^T ; A = strictly-lower beta_r e^{gamma_r - gamma_s} k_r.k_s
    for (int e = tid; e < L * DVS; e += SIMT_THREADS) {
      const int r = e / DVS, j = e - r * DVS;
      float acc = 0.0f;
      for (int i = 0; i < dk; ++i) acc = fmaf(Ss[j * dkp + i], Ks[r * dkp + i], acc);
      Xs[r * dvp + j] = acc;
    }
    for (int e = tid; e < L * L; e += SIMT_THREADS) {
      const int r = e / L, s = e - r * L;
      float val = 0.0f;
      if (s < r) {
        float acc = 0.0f;
        for (int i = 0; i < dk; ++i) acc = fmaf(Ks[r * dkp + i], Ks[s * dkp + i], acc);
        val = bet[r] * expf(gam[r] - gam[s]) * acc;
      }
      As[r * cp + s] = val;
    }
    __syncthreads();
    // ---- right-hand side beta_r (v_r - e^{gamma_r} (S0 k_r))
    for (int e = tid; e < L * DVS; e += SIMT_THREADS) {
      const int r = e / DVS, j = e - r * DVS;
      Vs[r * dvp + j] = bet[r] * (Vs[r * dvp + j] - expf(gam[r]) * Xs[r * dvp + j]);
    }
    __syncthreads();
    // ---- forward substitution (I + A) U = RHS, one column per thread
    if (tid < DVS) {
      const int j = tid;
      for (int r = 1; r < L; ++r) {
        float acc = Vs[r * dvp + j];
        for (int s = 0; s < r; ++s) acc = fmaf(-As[r * cp + s], Vs[s * dvp + j], acc);
        Vs[r * dvp + j] = acc;
      }
    }
    __syncthreads();
    // ---- X = Q S0^T ; A = M o Q K^T (lower incl. diagonal)
    for (int e = tid; e < L * DVS; e += SIMT_THREADS) {
      const int r = e / DVS, j = e - r * DVS;
      float acc = 0.0f;
      for (int i = 0; i < dk; ++i) acc = fmaf(Ss[j * dkp + i], Qs[r * dkp + i], acc);
      Xs[r * dvp + j] = acc;
    }
    for (int e = tid; e < L * L; e += SIMT_THREADS) {
      const int r = e / L, s = e - r * L;
      float val = 0.0f;
      if (s <= r) {
        float acc = 0.0f;
        for (int i = 0; i < dk; ++i) acc = fmaf(Qs[r * dkp + i], Ks[s * dkp + i], acc);
        val = expf(gam[r] - gam[s]) * acc;
      }
      As[r * cp + s] = val;
    }
    __syncthreads();
    // ---- outputs, and the state carried to the next chunk (independent: both read U)
    for (int e = tid; e < L * DVS; e += SIMT_THREADS) {
      const int r = e / DVS, j = e - r * DVS;
      float acc = expf(gam[r]) * Xs[r * dvp + j];
      for (int s = 0; s <= r; ++s) acc = fmaf(As[r * cp + s], Vs[s * dvp + j], acc);
      out[((c_beg + r) * Hv + h) * dv + j0 + j] = from_f<T>(scale * acc);
    }
    const float decL = expf(gam[L - 1]);
    for (int e = tid; e < DVS * dk; e += SIMT_THREADS) {
      const int j = e / dk, i = e - j * dk;
      float acc = decL * Ss[j * dkp + i];
      for (int s = 0; s < L; ++s) acc = fmaf(Vs[s * dvp + j] * dec[s], Ks[s * dkp + i], acc);
      Ss[j * dkp + i] = acc;
    }
  }
  __syncthreads();
  if (S_T) {
    for (int e = tid; e < DVS * dk; e += SIMT_THREADS) {
      const int j = e / dk, i = e - j * dk;
      S_T[sbase + (int64_t)(j0 + j) * dk + i] = Ss[j * dkp + i];
    }
  }
}

static size_t simt_smem_bytes(int dk, int C) {
  const size_t f = (size_t)SIMT_DVS * (dk + 1) + 2 * (size_t)C * (dk + 1) +
                   2 * (size_t)C * (SIMT_DVS + 1) + (size_t)C * (C + 1) + 3 * (size_t)C;
  return f * sizeof(float);
}

cudaError_t launch_chunk_simt(const void* q, const void* k, const void* v, TokStrides ts,
                              const float* g,
                              const float* beta, gdn_dtype dt, float scale, const float* S0,
                              const int32_t* cu, int N, int B, int64_t T, int Hk, int Hv, int dk,
                              int dv, int chunk, void* out, float* S_T, int* status,
                              cudaStream_t s) {
  (void)B;
  const int slices = (dv + SIMT_DVS - 1) / SIMT_DVS;
  const int64_t blocks = (int64_t)N * Hv * slices;
  if (blocks == 0) return cudaSuccess;
  const size_t smem = simt_smem_bytes(dk, chunk);
  cudaError_t e;
  if (dt == GDN_BF16) {
    e = cudaFuncSetAttribute(chunk_simt_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    chunk_simt_kernel<__nv_bfloat16><<<(unsigned)blocks, SIMT_THREADS, smem, s>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, ts, g, beta, scale,
        S0, cu, N, T, Hk, Hv, dk, dv, chunk, (__nv_bfloat16*)out, S_T, status);
  } else {
    e = cudaFuncSetAttribute(chunk_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    chunk_simt_kernel<float><<<(unsigned)blocks, SIMT_THREADS, smem, s>>>(
        (const float*)q, (const float*)k, (const float*)v, ts, g, beta, scale, S0, cu, N, T, Hk, Hv,
        dk, dv, chunk, (float*)out, S_T, status);
  }
  return cudaGetLastError();
}

}  // namespace gdn
