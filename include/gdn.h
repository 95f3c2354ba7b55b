/*
 * gdn.h -- C ABI of libgdn, the B200 (sm_100a) library for the gated delta rule, the per-head core
 * of the Gated DeltaNet linear-attention layer of Qwen3-Next / Qwen3.5.
 *
 * Sources, by page title:
 *   [P2] "解密Qwen3-Next的Gated DeltaNet：如何用75%混合层实现长文本高效推理" (jsqmd.com)
 *   [P3] "Qwen3.5 Gated DeltaNet 核心机制解析" (wanger-sjtu.github.io)
 *   [P5] "Qwen3-Next大模型架构解析：混合注意力与MoE优化实践" (intelliparadigm.com)
 *
 * Per v-head, with beta_t = sigmoid(b_t) and g_t = -exp(A_log) * softplus(a_t + dt_bias), the
 * state S (dv x dk, fp32) evolves as
 *     S_t = exp(g_t) * S_{t-1} * (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,    o_t = scale * S_t q_t.
 *
 * Conventions shared by every call
 *   - All pointers are DEVICE pointers into memory the caller owns (allocated by any means).  The
 *     library allocates nothing and keeps no global state; calls on different streams are
 *     independent.  Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and returns after the launch.
 *   - Tensors are dense, row-major, innermost index last, with these layouts:
 *       q, k          [B, T, Hk, dk]         v, out, z    [B, T, Hv, dv]
 *       g, beta, a, b [B, T, Hv]             state        [N, Hv, dv, dk]  (row j = value index)
 *       mix, y (conv) [B, T, C]              conv weight  [C, K]           conv state [N, C, K-1]
 *   - Varlen: with cu_seqlens (int32 [N+1], non-decreasing, cu_seqlens[0] = 0, cu_seqlens[N] = T)
 *     B must be 1 and sequence n is tokens [cu_seqlens[n], cu_seqlens[n+1]).  Without it sequence
 *     n is batch row n and N == B.
 *   - Head sharing: v-head h reads q/k head h / (Hv / Hk); Hv must be a multiple of Hk.
 *   - gdn_dtype selects the element type of the activations q, k, v, out, a, b, x, z, y, mix;
 *     g, beta, A_log, dt_bias, weights and all states are always fp32.
 *   - Outputs must not overlap inputs unless a call says otherwise.
 *   - Errors: arguments are checked on the host before any launch.  A bad argument returns
 *     GDN_ERR_INVALID_ARG, a valid but unimplemented shape returns GDN_ERR_UNSUPPORTED, and a
 *     failed launch returns GDN_ERR_CUDA.  Nothing is launched when a check fails.  Faults a
 *     kernel detects (a bad cu_seqlens, a wait that ran out) never trap: they are recorded in a
 *     status word in the caller's workspace (gdn_chunk_fwd) and read with gdn_workspace_status.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GDN_OK = 0,
  GDN_ERR_INVALID_ARG = 1, /* null / misaligned pointer, bad size, inconsistent shape */
  GDN_ERR_UNSUPPORTED = 2, /* well-formed but outside what the kernels implement */
  GDN_ERR_CUDA = 3,        /* a CUDA runtime call or a kernel launch failed */
  GDN_ERR_TIMEOUT = 4,     /* a kernel's bounded wait ran out (device status word) */
  GDN_ERR_DEVICE_ARG = 5   /* a kernel found a bad device-side argument, e.g. cu_seqlens */
} gdn_status;

typedef enum { GDN_BF16 = 0, GDN_F32 = 1 } gdn_dtype;

/* Human-readable name of a status code (static storage; never NULL). */
const char* gdn_status_string(gdn_status status);

/*
 * gdn_gates -- the two gates of the layer ([P5] §2.2 forward sketch: "beta = b.sigmoid();
 * g = -A_log.exp() * softplus(a + dt_bias)"; [P3] flowchart: b -> Sigmoid -> beta and
 * a -> Softplus(+dt_bias), A_log -> Exp and Neg, Mul -> g).  [P2] §2.1 prints the same two
 * expressions with the names swapped; beta here is the write strength and exp(g) in (0,1) the decay.
 *     beta[t,h] = 1 / (1 + exp(-b[t,h]))
 *     g[t,h]    = -exp(A_log[h]) * log(1 + exp(a[t,h] + dt_bias[h]))
 * a, b     : [n_tok, Hv] of ab_dtype, n_tok = B*T (any token flattening).
 * A_log, dt_bias : [Hv] fp32.
 * g, beta  : [n_tok, Hv] fp32 outputs.
 * n_tok >= 0 (0 launches nothing), 1 <= Hv.
 */
gdn_status gdn_gates(const void* a, const void* b, gdn_dtype ab_dtype, const float* A_log,
                     const float* dt_bias, int64_t n_tok, int Hv, float* g, float* beta,
                     void* stream);

/*
 * gdn_causal_conv1d_silu -- depthwise causal conv over time on the q|k|v mix, SiLU, then the L2
 * normalisation of each q and k head ([P3] conv-layer section and flowchart: the QKV mix passes a
 * "Depthwise Causal Conv" before it is split into q, k, v).
 *     pre[t,c] = bias[c] + sum_{i<K} w[c,i] * x[t-(K-1)+i, c]     (cross-correlation; w[c,K-1]
 *                                                                  multiplies the current token)
 *     y[t,c]   = silu(pre[t,c]);  then for every group of l2norm_group channels inside the first
 *                n_l2norm_ch channels: y[t,G] /= sqrt(sum_G y[t,.]^2 + l2_eps)
 * Positions before a sequence start read conv_state_in[n, c, K-1+p] (p = -(K-1)..-1, oldest
 * first) or zero when conv_state_in is NULL; the conv never crosses sequences.
 * x, y           : [B, T, C] of dtype; x and y must not overlap.
 * w              : [C, K] fp32.  bias: [C] fp32 or NULL.
 * cu_seqlens     : int32 [N+1] or NULL (then N == B).
 * conv_state_in  : [N, C, K-1] fp32 or NULL.  conv_state_out: [N, C, K-1] fp32 or NULL, receives
 *                  the last K-1 inputs of each sequence (for a following decode).  The two must
 *                  not overlap.
 * Supported: 1 <= K <= 8; C a multiple of 8; n_l2norm_ch a multiple of l2norm_group; l2norm_group
 * in {0 (no normalisation), 32, 64, 128, 256}; x, y 16-byte aligned.
 */
gdn_status gdn_causal_conv1d_silu(const void* x, gdn_dtype dtype, const float* w,
                                  const float* bias, int B, int64_t T, int C, int K,
                                  const int32_t* cu_seqlens, int N, int n_l2norm_ch,
                                  int l2norm_group, float l2_eps, const float* conv_state_in,
                                  float* conv_state_out, void* y, void* stream);

/*
 * gdn_chunk_fwd -- chunk-parallel prefill, chunk_gated_delta_rule(q, k, v, g, beta,
 * initial_state) -> (out, final_state) of [P2] §2.2 (chunked parallel mode; state carried across
 * calls through initial_state) and [P3] "cache and state switching" (the training / prefill path).
 * Exactly the recurrence above, evaluated chunk by chunk in the WY/UT form: per chunk of `chunk`
 * tokens an intra-chunk triangular system gives the corrections, and the state is propagated
 * between chunks with the cumulative decay.
 * q, k           : [B, T, Hk, dk] dtype.   v, out: [B, T, Hv, dv] dtype.
 * g, beta        : [B, T, Hv] fp32 (log-decay and write strength, e.g. from gdn_gates).
 * scale          : multiplies S_t q_t (dk^-0.5 in Qwen3-Next).
 * initial_state  : [N, Hv, dv, dk] fp32 or NULL (zero state).
 * final_state    : [N, Hv, dv, dk] fp32 or NULL (not written).  May not overlap initial_state.
 * cu_seqlens     : int32 [N+1] or NULL (then N == B).  Each sequence is chunked from its own
 *                  start; its last chunk may be partial.
 * workspace      : device scratch, 256-byte aligned, at least 256 bytes; its first word is the
 *                  device status word (read it with gdn_workspace_status).  With at least
 *                  gdn_chunk_fwd_workspace_size() bytes the bf16 d = 128 chunk-64 shape takes the
 *                  fast two-kernel path, which keeps each chunk's state-independent operands
 *                  there (about 16.5 KB per chunk and v-head); with less it takes a path that
 *                  needs only the status word.  Contents on entry are ignored.  Concurrent calls
 *                  need separate workspaces.
 * Supported: dk, dv in {16, 32, ..., 128} (multiples of 16), chunk in {16, 32, 64}.  The tensor-core
 * path (tcgen05 + TMA) serves dtype GDN_BF16, dk = dv = 128, chunk = 64; every other supported
 * shape runs on the CUDA-core path.  All pointers 16-byte aligned.
 */
gdn_status gdn_chunk_fwd(const void* q, const void* k, const void* v, const float* g,
                         const float* beta, gdn_dtype dtype, float scale,
                         const float* initial_state, const int32_t* cu_seqlens, int N, int B,
                         int64_t T, int Hk, int Hv, int dk, int dv, int chunk, void* out,
                         float* final_state, void* workspace, size_t workspace_bytes,
                         void* stream);

/*
 * gdn_chunk_fwd_strided -- gdn_chunk_fwd on q, k, v whose tokens are not packed back to back,
 * e.g. q, k and v read straight out of the [q | k | v] output of gdn_causal_conv1d_silu (the
 * split after the conv in [P3]'s flowchart) without copying them apart.
 * q_tok_stride, k_tok_stride, v_tok_stride: elements between consecutive tokens (batch row b,
 * token t sits at token index b*T + t); within a token the heads stay contiguous (head h at
 * h*dk, resp. h*dv).  Each stride must be >= the token's heads (Hk*dk, resp. Hv*dv) and a
 * multiple of 8 elements.  Everything else as gdn_chunk_fwd, which is this call with the dense
 * strides Hk*dk, Hk*dk, Hv*dv.  out stays dense [B, T, Hv, dv].
 */
gdn_status gdn_chunk_fwd_strided(const void* q, int64_t q_tok_stride, const void* k,
                                 int64_t k_tok_stride, const void* v, int64_t v_tok_stride,
                                 const float* g, const float* beta, gdn_dtype dtype, float scale,
                                 const float* initial_state, const int32_t* cu_seqlens, int N,
                                 int B, int64_t T, int Hk, int Hv, int dk, int dv, int chunk,
                                 void* out, float* final_state, void* workspace,
                                 size_t workspace_bytes, void* stream);

/*
 * gdn_chunk_fwd_gated_norm -- the layer core after the conv in one call: the gates, the chunked
 * gated delta rule and the gated RMSNorm of its output, as in [P3]'s flowchart (split -> gates ->
 * delta rule -> RMSNormGated(core_attn_out, z)) and [P2] §3.2.  Results equal
 *     gdn_gates(a, b) -> gdn_chunk_fwd_strided(q, k, v, g, beta) -> gdn_gated_rmsnorm(., z)
 * except that g and beta are never written to memory: the gates are computed where the
 * per-chunk operands are prepared.  The delta-rule output is written to y and normalised there in
 * place by a second pass.
 * q, k, v, strides, scale, initial_state, cu_seqlens, N, B, T, Hk, Hv, final_state, workspace:
 *                  as gdn_chunk_fwd_strided.
 * a, b           : [B*T, Hv] bf16 gate pre-activations (as gdn_gates).
 * A_log, dt_bias : [Hv] fp32 (as gdn_gates).
 * z              : [B*T, Hv, dv] bf16, the output gate.   norm_w: [dv] fp32 (used as 1 + w).
 * y              : [B*T, Hv, dv] bf16, the gated RMSNorm of the delta-rule output.  Must not
 *                  overlap z, q, k or v.
 * Supported: bf16, dk = dv = 128, chunk = 64, with a workspace of gdn_chunk_fwd_workspace_size()
 * bytes (one too small for the intra-sequence scan's state arrays but holding the per-chunk
 * operands runs without the scan); anything else returns GDN_ERR_UNSUPPORTED -- use the three
 * unfused calls there.  z, y, norm_w 16-byte
 * aligned.  Device-detected faults land in the workspace status word as for gdn_chunk_fwd.
 */
gdn_status gdn_chunk_fwd_gated_norm(const void* q, int64_t q_tok_stride, const void* k,
                                    int64_t k_tok_stride, const void* v, int64_t v_tok_stride,
                                    const void* a, const void* b, const float* A_log,
                                    const float* dt_bias, const void* z, const float* norm_w,
                                    float norm_eps, gdn_dtype dtype, float scale,
                                    const float* initial_state, const int32_t* cu_seqlens, int N,
                                    int B, int64_t T, int Hk, int Hv, int dk, int dv, int chunk,
                                    void* y, float* final_state, void* workspace,
                                    size_t workspace_bytes, void* stream);

/*
 * gdn_chunk_fwd_noalloc -- gdn_chunk_fwd for callers that cannot allocate device memory.  The
 * pages have no counterpart: this is a library convenience.
 * Who needs it: code that receives device pointers from another runtime and may not allocate
 * during a call -- e.g. a plugin inside an inference engine that plans all device memory ahead
 * (cudaMalloc can synchronise the device and stall the engine's other streams), or a host with a
 * fixed device-memory budget that owns every buffer.  Such callers cannot supply a workspace.
 * Same arguments, layouts and results as gdn_chunk_fwd, without workspace / workspace_bytes: the
 * scratch is a fixed array of GDN_NOALLOC_SCRATCH_BYTES inside the library (a __device__
 * variable that every GPU which loads the library holds until the process exits).  Sizes whose
 * gdn_chunk_fwd_workspace_size() exceeds that maximum return GDN_ERR_UNSUPPORTED.  The call
 * allocates nothing (no cudaMalloc, cudaFree or allocating library routine).
 * Every call looks up the array's device address (cudaGetSymbolAddress) on the current device; the
 * first call on a device may load the library's device code there, so make that first call
 * before any stream capture.  cudaDeviceReset between calls is fine.  All calls on a device
 * share the one array and it keeps the last call's contents (the status word is cleared by each
 * call), so calls whose kernels overlap on the GPU -- on different streams, or from different host
 * threads -- race on it: serialise them.  Device-detected faults land in that shared status word
 * and are not reported separately; use gdn_chunk_fwd with a workspace to read them.
 */
#define GDN_NOALLOC_SCRATCH_BYTES (16 * 1024 * 1024)
gdn_status gdn_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* g,
                                 const float* beta, gdn_dtype dtype, float scale,
                                 const float* initial_state, const int32_t* cu_seqlens, int N,
                                 int B, int64_t T, int Hk, int Hv, int dk, int dv, int chunk,
                                 void* out, float* final_state, void* stream);

/* Bytes of workspace for gdn_chunk_fwd's fastest path at these sizes (always >= 256, a multiple of
 * 256): ceil(B*T / 64) + N chunk slots x Hv x 16896 bytes + 1024 for the bf16 d = 128 chunk-64
 * shape, 256 otherwise. */
size_t gdn_chunk_fwd_workspace_size(int N, int B, int64_t T, int Hk, int Hv, int dk, int dv,
                                    int chunk);

/*
 * gdn_workspace_status -- waits for `stream`, then reads the device status word a previous
 * gdn_chunk_fwd left in `workspace` into *device_status (GDN_OK when every kernel finished
 * cleanly).  Returns GDN_ERR_CUDA if the copy or the wait failed.  A debugging aid: it blocks.
 */
gdn_status gdn_workspace_status(const void* workspace, void* stream, int* device_status);

/*
 * gdn_recurrent_step -- one-token decode, recurrent_gated_delta_rule(q, k, v, g, beta,
 * initial_state=cached_state) -> (out, new_state) of [P2] §2.2 (recurrent inference mode) and
 * [P3] (the path taken when the cache is valid and L = 1).  One token per sequence:
 *     a = exp(g);  S <- a*S;  u = beta*(v - S k);  S <- S + u k^T;  o = scale * S q
 * q, k   : [N, Hk, dk] dtype.   v, out: [N, Hv, dv] dtype.   g, beta: [N, Hv] fp32.
 * state  : [N, Hv, dv, dk] fp32, read and updated IN PLACE.
 * Supported: dk = 128 with dv a multiple of 8 up to 256 (rows are spread over warps), all
 *            pointers 16-byte aligned.  N = 0 launches nothing.
 */
gdn_status gdn_recurrent_step(const void* q, const void* k, const void* v, const float* g,
                              const float* beta, gdn_dtype dtype, float scale, float* state,
                              int N, int Hk, int Hv, int dk, int dv, void* out, void* stream);

/*
 * gdn_decode_layer_step -- one decode token of the whole layer core in one launch ([P3] "cache and
 * state switching": the decode path advances the conv_states cache (the conv's last K-1 inputs)
 * and the recurrent_states cache (the delta-rule state) by one token; the flowchart's order conv ->
 * split -> gates -> delta rule -> RMSNormGated(core_attn_out, z); [P2] §2.2 recurrent mode and
 * §3.2 norm).  Per sequence it equals
 *     gdn_causal_conv1d_silu on the one new token with conv_state_in as history (q and k heads
 *     L2-normalised with l2_eps) -> gdn_gates(a, b) -> gdn_recurrent_step -> gdn_gated_rmsnorm(., z)
 * except that q, k and v stay fp32 between the conv and the delta rule.
 * mix            : [N, C] dtype, C = 2*Hk*dk + Hv*dv: the new token's [q | k | v] mix before the
 *                  conv (channel order as gdn_causal_conv1d_silu's).
 * a, b           : [N, Hv] dtype.   z: [N, Hv, dv] dtype.
 * conv_w         : [C, K] fp32.  conv_bias: [C] fp32 or NULL.
 * conv_state_in  : [N, C, K-1] fp32, the previous K-1 inputs of each channel, oldest first.
 * conv_state_out : [N, C, K-1] fp32, receives them advanced by this token.  Must not overlap
 *                  conv_state_in (ping-pong two buffers).  Both may be NULL when K = 1.
 * A_log, dt_bias : [Hv] fp32.   norm_w: [dv] fp32 (zero-centred, used as 1 + w).
 * state          : [N, Hv, dv, dk] fp32, read and updated IN PLACE.
 * y              : [N, Hv, dv] dtype, the gated RMSNorm of the core output (must not overlap the
 *                  inputs).
 * Supported: dk = dv = 128, 1 <= K <= 8; mix, z, y, state 16-byte aligned.  N = 0 launches nothing.
 */
gdn_status gdn_decode_layer_step(const void* mix, const void* a, const void* b, const void* z,
                                 gdn_dtype dtype, const float* conv_w, const float* conv_bias,
                                 int K, const float* conv_state_in, float* conv_state_out,
                                 const float* A_log, const float* dt_bias, const float* norm_w,
                                 float l2_eps, float norm_eps, float scale, float* state, int N,
                                 int Hk, int Hv, int dk, int dv, void* y, void* stream);

/*
 * gdn_gated_rmsnorm -- zero-centred RMSNorm gated by z ([P2] §3.2: weight stored zero-centred and
 * used as (1 + w), normalisation in fp32 with rsqrt(mean(x^2) + eps); [P3] output section: the norm
 * of core_attn_out fuses the z gate in, "like SwiGLU").
 *     y[r,j] = x[r,j] * rsqrt(mean_j x[r,.]^2 + eps) * (1 + w[j]) * silu(z[r,j])
 * x, z, y : [n_rows, dim] dtype (e.g. n_rows = B*T*Hv, dim = dv).   w: [dim] fp32.
 * Supported: dim in {8, 16, 32, 64, 128, 256}; x, z, y 16-byte aligned.  n_rows = 0 launches
 * nothing.  y may alias x (in place) but not z.
 */
gdn_status gdn_gated_rmsnorm(const void* x, const void* z, gdn_dtype dtype, const float* w,
                             float eps, int64_t n_rows, int dim, void* y, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
