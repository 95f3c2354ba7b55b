/*
 * gdn_oracle.c -- plain, slow, fp64 CPU oracle for the gated delta rule.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's CPU-baseline leg
 * may load this file's library.  It shares no code, header, table or helper with the CUDA path.
 *
 * Sources (cited by page title and section):
 *   [P2] "解密Qwen3-Next的Gated DeltaNet：如何用75%混合层实现长文本高效推理" (jsqmd.com)
 *        §2.1 gate definitions, §2.2 chunk / recurrent call conventions, §3.2 zero-centred RMSNorm.
 *   [P3] "Qwen3.5 Gated DeltaNet 核心机制解析" (wanger-sjtu.github.io)
 *        flowchart (conv1d -> split -> gates -> "Delta Rule: State Update and Retrieval" ->
 *        RMSNormGated(core_attn_out, z)), and the prose sections on the conv layer, the core
 *        mechanism and the gated output norm.
 *   [P5] "Qwen3-Next大模型架构解析：混合注意力与MoE优化实践" (intelliparadigm.com)
 *        §2.2 Qwen3NextGatedDeltaNet forward sketch (gate formulas, mode dispatch).
 *
 * Every function below is the plain definition written out, one token at a time, with no
 * blocking, chunking or re-association.  Layouts (all row-major, innermost last):
 *   q, k      [B, T, Hk, dk]          v, out   [B, T, Hv, dv]
 *   g, beta   [B, T, Hv]              state    [N, Hv, dv, dk]   (row j = value index)
 *   mix, y    [B, T, C]               conv w   [C, K]            conv state [N, C, K-1]
 * With cu_seqlens (int32, N+1 entries) B must be 1 and sequence n is tokens
 * [cu_seqlens[n], cu_seqlens[n+1]); without it sequence n is batch row n (N == B).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- gates ---------------- */

/* softplus(x) = log(1 + e^x), evaluated as max(x,0) + log1p(e^{-|x|}) which is the same value
 * and never overflows. */
static double softplus(double x) { return (x > 0.0 ? x : 0.0) + log1p(exp(-fabs(x))); }

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/*
 * Gates, [P5] §2.2 ("beta = b.sigmoid(); g = -A_log.exp() * softplus(a + dt_bias)") and [P3]
 * flowchart (b -> Sigmoid -> beta; a -> Softplus + dt_bias; A_log -> Exp and Neg; Mul -> g).
 * [P2] §2.1 prints the same two expressions with the names swapped; the reading taken here is
 * the one of [P3]/[P5]: beta = sigmoid(b) is the write strength, g is the log-decay (e^g in (0,1)).
 * a, b: [n_tok, Hv]; A_log, dt_bias: [Hv]; g, beta: [n_tok, Hv].
 */
void oracle_gates(const double* a, const double* b, const double* A_log, const double* dt_bias,
                  int64_t n_tok, int Hv, double* g, double* beta) {
  for (int64_t t = 0; t < n_tok; ++t) {
    for (int h = 0; h < Hv; ++h) {
      int64_t i = t * Hv + h;
      beta[i] = sigmoid(b[i]);
      g[i] = -exp(A_log[h]) * softplus(a[i] + dt_bias[h]);
    }
  }
}

/* ---------------------------------------------------- causal depthwise conv1d + SiLU ------ */

static double silu(double x) { return x * sigmoid(x); }

/* Sequence boundaries: fills *start, *len for sequence n. */
static void seq_bounds(const int32_t* cu_seqlens, int64_t T, int n, int64_t* start,
                       int64_t* len) {
  if (cu_seqlens) {
    *start = cu_seqlens[n];
    *len = (int64_t)cu_seqlens[n + 1] - cu_seqlens[n];
  } else {
    *start = (int64_t)n * T; /* batch row n, flattened over [B, T] */
    *len = T;
  }
}

/*
 * Causal depthwise conv over time, then SiLU, then per-head L2 normalisation of the leading
 * n_l2norm_ch channels in groups of l2norm_group ([P3] conv-layer section and flowchart node
 * "conv1d: Depthwise Causal Conv" applied to the q|k|v mix before the split).
 *   pre[t, c] = bias[c] + sum_{i=0}^{K-1} w[c, i] * x[t - (K-1) + i, c]
 *   y[t, c]   = silu(pre[t, c])
 *   for a normalised group G containing c:  y[t, c] /= sqrt(sum_{c' in G} y[t, c']^2 + l2_eps)
 * Positions before a sequence's first token read conv_state_in[n, c, K-1+p] for p = -(K-1)..-1
 * (oldest first) or zero when conv_state_in is NULL.  The conv never crosses sequences.
 * conv_state_out (optional) receives, per sequence, the last K-1 inputs in the same layout.
 * x, y: [B, T, C]; w: [C, K]; bias: [C] or NULL.
 */
void oracle_causal_conv1d_silu(const double* x, const double* w, const double* bias, int B,
                               int64_t T, int C, int K, const int32_t* cu_seqlens, int N,
                               int n_l2norm_ch, int l2norm_group, double l2_eps,
                               const double* conv_state_in, double* conv_state_out, double* y) {
  (void)B;
  for (int n = 0; n < N; ++n) {
    int64_t start, len;
    seq_bounds(cu_seqlens, T, n, &start, &len);
    for (int64_t t = 0; t < len; ++t) {
      const int64_t row = start + t;
      for (int c = 0; c < C; ++c) {
        double acc = bias ? bias[c] : 0.0;
        for (int i = 0; i < K; ++i) {
          int64_t p = t - (K - 1) + i; /* position relative to the sequence start */
          double xv;
          if (p >= 0)
            xv = x[(start + p) * C + c];
          else
            xv = conv_state_in ? conv_state_in[((int64_t)n * C + c) * (K - 1) + (K - 1) + p]
                               : 0.0;
          acc += w[(int64_t)c * K + i] * xv;
        }
        y[row * C + c] = silu(acc);
      }
      for (int c0 = 0; c0 + l2norm_group <= n_l2norm_ch; c0 += l2norm_group) {
        double ss = 0.0;
        for (int c = c0; c < c0 + l2norm_group; ++c) ss += y[row * C + c] * y[row * C + c];
        double inv = 1.0 / sqrt(ss + l2_eps);
        for (int c = c0; c < c0 + l2norm_group; ++c) y[row * C + c] *= inv;
      }
    }
    if (conv_state_out) {
      for (int c = 0; c < C; ++c) {
        for (int j = 0; j < K - 1; ++j) {
          int64_t p = len - (K - 1) + j;
          double xv;
          if (p >= 0)
            xv = x[(start + p) * C + c];
          else
            xv = conv_state_in ? conv_state_in[((int64_t)n * C + c) * (K - 1) + (K - 1) + p]
                               : 0.0;
          conv_state_out[((int64_t)n * C + c) * (K - 1) + j] = xv;
        }
      }
    }
  }
}

/* ------------------------------------------------------------ the gated delta rule ------- */

typedef struct {
  const double *q, *k, *v, *g, *beta, *S0;
  const int32_t* cu_seqlens;
  double scale;
  int N, Hk, Hv, dk, dv;
  int64_t T;
  double *out, *S_final;
  int next_unit; /* shared work counter over (sequence, v-head) units */
  pthread_mutex_t lock;
} rule_job;

/*
 * One (sequence n, v-head h) chain, token by token.  The state update is the gated delta rule
 *     S_t = e^{g_t} S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,      o_t = scale * S_t q_t
 * -- a decay of the whole state by the forgetting gate g, then a correction of what the state
 * returns for the current key toward v with write strength beta ([P3] core-mechanism section:
 * g forgets, beta sets write strength, and the delta rule corrects the stored state according to
 * the current key; [P2] §2.1 table: element-wise precise deletion and selective update).
 * The product with (I - beta k k^T) is expanded as S - beta (S k) k^T; nothing else is reordered.
 * v-head h reads q/k head h / (Hv/Hk) (each k head is shared by Hv/Hk consecutive v heads).
 */
static void rule_unit(const rule_job* J, int n, int h) {
  const int dk = J->dk, dv = J->dv, Hk = J->Hk, Hv = J->Hv;
  const int hk = h / (Hv / Hk);
  double* S = (double*)malloc(sizeof(double) * (size_t)dv * dk);
  double* Sk = (double*)malloc(sizeof(double) * (size_t)dv);
  const size_t sbase = ((size_t)n * Hv + h) * (size_t)dv * dk;
  if (J->S0)
    memcpy(S, J->S0 + sbase, sizeof(double) * (size_t)dv * dk);
  else
    memset(S, 0, sizeof(double) * (size_t)dv * dk);

  int64_t start, len;
  seq_bounds(J->cu_seqlens, J->T, n, &start, &len);
  for (int64_t t = 0; t < len; ++t) {
    const int64_t row = start + t; /* flattened token index over [B, T] */
    const double* qt = J->q + (row * Hk + hk) * dk;
    const double* kt = J->k + (row * Hk + hk) * dk;
    const double* vt = J->v + (row * Hv + h) * dv;
    const double a = exp(J->g[row * Hv + h]);
    const double bt = J->beta[row * Hv + h];
    /* (S_{t-1} k_t) */
    for (int j = 0; j < dv; ++j) {
      double s = 0.0;
      for (int i = 0; i < dk; ++i) s += S[(size_t)j * dk + i] * kt[i];
      Sk[j] = s;
    }
    /* S_t = a (S_{t-1} - beta (S_{t-1} k) k^T) + beta v k^T */
    for (int j = 0; j < dv; ++j)
      for (int i = 0; i < dk; ++i)
        S[(size_t)j * dk + i] =
            a * (S[(size_t)j * dk + i] - bt * Sk[j] * kt[i]) + bt * vt[j] * kt[i];
    /* o_t = scale * S_t q_t */
    double* ot = J->out + (row * Hv + h) * dv;
    for (int j = 0; j < dv; ++j) {
      double s = 0.0;
      for (int i = 0; i < dk; ++i) s += S[(size_t)j * dk + i] * qt[i];
      ot[j] = J->scale * s;
    }
  }
  if (J->S_final) memcpy(J->S_final + sbase, S, sizeof(double) * (size_t)dv * dk);
  free(Sk);
  free(S);
}

static void* rule_worker(void* arg) {
  rule_job* J = (rule_job*)arg;
  const int units = J->N * J->Hv;
  for (;;) {
    pthread_mutex_lock(&J->lock);
    int u = J->next_unit++;
    pthread_mutex_unlock(&J->lock);
    if (u >= units) break;
    rule_unit(J, u / J->Hv, u % J->Hv);
  }
  return NULL;
}

/*
 * Whole-tensor gated delta rule ([P2] §2.2 chunk_gated_delta_rule / recurrent_gated_delta_rule:
 * (q, k, v, g, beta, initial_state) -> (out, final_state)).  Both modes compute this same
 * function; the chunked form is an exact re-association of it.
 * S0 may be NULL (zero initial state); S_final may be NULL.  (sequence, head) units are
 * independent and are spread over nthreads POSIX threads (<= 1 means the calling thread).
 * Returns 0, or -1 on an argument error.
 */
int oracle_gated_delta_rule(const double* q, const double* k, const double* v, const double* g,
                            const double* beta, double scale, const double* S0,
                            const int32_t* cu_seqlens, int N, int B, int64_t T, int Hk, int Hv,
                            int dk, int dv, double* out, double* S_final, int nthreads) {
  if (Hk <= 0 || Hv <= 0 || Hv % Hk != 0 || dk <= 0 || dv <= 0 || N <= 0) return -1;
  if (cu_seqlens ? B != 1 : N != B) return -1;
  rule_job J;
  J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta; J.S0 = S0; J.cu_seqlens = cu_seqlens;
  J.scale = scale; J.N = N; J.Hk = Hk; J.Hv = Hv; J.dk = dk; J.dv = dv; J.T = T;
  J.out = out; J.S_final = S_final; J.next_unit = 0;
  pthread_mutex_init(&J.lock, NULL);
  if (nthreads <= 1) {
    rule_worker(&J);
  } else {
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, rule_worker, &J);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
  }
  pthread_mutex_destroy(&J.lock);
  return 0;
}

/* ------------------------------------------------------------ gated RMSNorm ---------------- */

/*
 * Zero-centred RMSNorm ([P2] §3.2: weight initialised to zero and applied as (1 + w), normalised
 * in float with rsqrt(mean(x^2) + eps)) followed by the z gate ([P3] output section: the norm
 * fuses the z gate into the result, "like SwiGLU", i.e. a silu(z) factor after the norm).
 *   y[r, j] = x[r, j] / sqrt(mean_j x[r, :]^2 + eps) * (1 + w[j]) * silu(z[r, j])
 * x, z, y: [rows, dim]; w: [dim].
 */
void oracle_gated_rmsnorm(const double* x, const double* z, const double* w, double eps,
                          int64_t rows, int dim, double* y) {
  for (int64_t r = 0; r < rows; ++r) {
    const double* xr = x + r * dim;
    double ss = 0.0;
    for (int j = 0; j < dim; ++j) ss += xr[j] * xr[j];
    const double inv = 1.0 / sqrt(ss / dim + eps);
    for (int j = 0; j < dim; ++j) y[r * dim + j] = xr[j] * inv * (1.0 + w[j]) * silu(z[r * dim + j]);
  }
}
