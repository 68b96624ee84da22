/*
 * gdn.h -- C ABI of libgdn.so, the Gated DeltaNet token mixer on NVIDIA B200 (sm_100a).
 *
 * The method: "Qwen3.8-Flash-Next 技术总结 -- Qwen4 架构的探路者", section 2.1
 * "Gated DeltaNet".  Per sequence and V head the recurrent state S_t is a dk x dv
 * matrix (row index = key dimension) updated token by token as
 *
 *     S_t = alpha_t S_{t-1} + beta_t k_t (v_t - alpha_t S_{t-1}^T k_t)^T
 *         = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
 *
 * (the two equal forms the page gives), with alpha_t the forget gate and beta_t
 * the write strength.  The page names no read-out; this library returns
 * o_t = S_t^T q_t, taken with the state after token t's update, unscaled.
 * The same section gives the model's head layout -- 48 V heads that share 16
 * QK heads, head dim 128 -- and says the recurrence is evaluated chunk by chunk
 * with the WY representation; gdn_chunk_fwd is that chunkwise evaluation,
 * gdn_decode_step the one-token update.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layouts are dense and row-major; "[a, b, c]" lists dimensions outermost first.
 *   q, k      [B, T, Hqk, dk]   (decode: [B, Hqk, dk])    dtype given by `dtype`
 *   v, o      [B, T, Hv,  dv]   (decode: [B, Hv,  dv])    dtype given by `dtype`
 *   alpha     [B, T, Hv]        (decode: [B, Hv])         float; alpha itself, not log alpha
 *   beta      [B, T, Hv]        (decode: [B, Hv])         float
 *   S0, S     [B, Hv, dk, dv]                             float (fp32 state)
 * V head h reads q and k of QK head h / (Hv / Hqk) (contiguous groups of
 * Hv / Hqk V heads share one QK head).  Gates are per token and V head.
 * alpha is expected in (0, 1] (1 = no forgetting); the kernels clamp log alpha
 * below at -87, so alpha = 0 acts as alpha = exp(-87).  beta may be any real.
 *
 * Ownership: every pointer is a DEVICE pointer to memory the caller owns; the
 * library keeps no reference after the call returns and allocates no device
 * memory.  Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 * default stream).  Input buffers must not be modified until the work on
 * `stream` completes.
 *
 * Errors: argument checks run synchronously on the host before any launch and
 * return GDN_ERR_INVALID_ARG (bad pointer, size or alignment) or
 * GDN_ERR_UNSUPPORTED (a shape this build does not implement).  A failed launch
 * returns GDN_ERR_CUDA (the CUDA error is also returned by gdn_last_cuda_error()).
 * Kernels never trap.  Every pointer must be 16-byte aligned.
 */
#ifndef GDN_H
#define GDN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,
    GDN_ERR_UNSUPPORTED = 2,
    GDN_ERR_CUDA = 3,
    GDN_ERR_TIMEOUT = 4   /* a bounded wait inside a kernel gave up (see gdn_device_status) */
} gdn_status;

typedef enum {
    GDN_F32 = 0,   /* q, k, v, o are float  (fp32 arithmetic end to end)          */
    GDN_BF16 = 1   /* q, k, v, o are bfloat16; state, gates and accumulation fp32 */
} gdn_dtype;

/*
 * gdn_chunk_fwd -- prefill: runs T tokens of every (sequence, V head) from S0.
 *
 * Defines: section 2.1 "Gated DeltaNet" of the page above (the update rule and
 * the chunkwise WY evaluation it attributes to the Gated DeltaNet paper).
 *
 * In:  q, k, v, alpha, beta  as in the layout table, T tokens per sequence.
 *      S0       initial state [B, Hv, dk, dv]; NULL means all zeros.
 * Out: o        [B, T, Hv, dv], o_t = S_t^T q_t.
 *      S_final  state after token T-1, [B, Hv, dk, dv]; NULL skips it.  It may
 *               be the same buffer as S0 (in-place update); any other overlap
 *               of outputs with inputs is undefined.
 * Sizes: B >= 0, T >= 0 (T == 0 copies S0, or zeros, to S_final), Hqk >= 1,
 *      Hv >= 1 with Hv % Hqk == 0, dk == dv == 128 and chunk == 64
 *      (else GDN_ERR_UNSUPPORTED).
 * dtype: GDN_F32 evaluates the chunk form in fp32 on CUDA cores; GDN_BF16 runs
 *      the contractions on the tensor cores with fp32 accumulation and an fp32
 *      state.
 */
gdn_status gdn_chunk_fwd(const void *q, const void *k, const void *v,
                         const float *alpha, const float *beta, const float *S0,
                         void *o, float *S_final,
                         int B, int T, int Hqk, int Hv, int dk, int dv, int chunk,
                         gdn_dtype dtype, void *stream);

/*
 * gdn_chunk_fwd_varlen -- prefill of N sequences of different lengths packed
 * back to back (continuous batching of prompts of any lengths in one call).
 *
 * Defines: gdn_chunk_fwd applied to each sequence on its own.  Use: continuous
 * batching in serving ("通义千问Qwen3.8-Flash-Next开源：四大架构升级与部署优化全解析",
 * section "性能表现与开源生态支持").
 *
 * In:  q, k [T_total, Hqk, dk]; v [T_total, Hv, dv]; alpha, beta [T_total, Hv];
 *      cu_seqlens [N + 1] int32 (device): sequence n is token rows
 *      cu_seqlens[n] .. cu_seqlens[n+1] - 1 (cu_seqlens[0] = 0, nondecreasing,
 *      cu_seqlens[N] = T_total; offsets are clamped into [0, T_total], so a
 *      malformed table gives wrong results, never an out-of-bounds access);
 *      S0 [N, Hv, dk, dv] or NULL (zeros).
 * Out: o [T_total, Hv, dv]; S_final [N, Hv, dk, dv] or NULL (may be S0).  An
 *      empty sequence copies its S0 (or zeros) to S_final.
 * Sizes, dtypes, alignment and kernel choice as for gdn_chunk_fwd, with
 *      N in place of B (N <= 65535); cu_seqlens must be 4-byte aligned.
 */
gdn_status gdn_chunk_fwd_varlen(const void *q, const void *k, const void *v,
                                const float *alpha, const float *beta, const float *S0,
                                void *o, float *S_final, const int *cu_seqlens,
                                int N, int T_total, int Hqk, int Hv, int dk, int dv, int chunk,
                                gdn_dtype dtype, void *stream);

/*
 * gdn_chunk_fwd_split -- gdn_chunk_fwd with each sequence cut into segments that
 * run side by side (long sequences, or few sequences x heads for the GPU).
 *
 * Defines: the same function as gdn_chunk_fwd.  The update of section 2.1
 * "Gated DeltaNet" (page above) is affine in the state, so a segment's end state
 * is M S_start + D and its outputs are o^0_t + S_start^T r_t.  Here:
 *   - D and o^0 come from a run from a zero start;
 *   - M and the rows r_t come from a run from S = I with v = 0;
 *   - one launch runs these for every segment at once;
 *   - a short fp32 walk over the segments then gives each S_start, and a
 *     tensor-core pass adds R S_start to the outputs (with two segments,
 *     S_start = D of the first, and one launch does both the pass and the
 *     final state).
 * The serial chain is one segment long.  Use: long contexts at small batch
 * ("Qwen3.8-Flash-Next 技术总结 -- Qwen4 架构的探路者", section 2.1 and the model
 * card's 262,144-token native context).
 *
 * Arguments as gdn_chunk_fwd, plus:
 *   segments   1..16, or 0 for the most segments whose CTAs all fit on the device
 *              at once (B*Hv*(2*segments-1) CTAs).  Segments are whole chunks.
 *   workspace  device scratch of at least gdn_chunk_fwd_split_workspace(...)
 *              bytes, 256-byte aligned, owned by the caller; its contents on
 *              entry do not matter, and calls sharing it must not overlap.
 * Only GDN_BF16 on the tensor cores splits; otherwise, or when one segment
 * covers the sequence, the call is gdn_chunk_fwd (workspace unused, may be
 * NULL).  A too small or misaligned workspace returns GDN_ERR_INVALID_ARG.
 * Rounding differs from gdn_chunk_fwd (outputs of later segments are a sum
 * of two bf16-rounded terms) within the bf16 tolerance of the method.
 */
size_t gdn_chunk_fwd_split_workspace(int B, int T, int Hv, int dk, int dv, int segments);
gdn_status gdn_chunk_fwd_split(const void *q, const void *k, const void *v,
                               const float *alpha, const float *beta, const float *S0,
                               void *o, float *S_final,
                               int B, int T, int Hqk, int Hv, int dk, int dv, int chunk,
                               int segments, gdn_dtype dtype, void *workspace,
                               size_t workspace_bytes, void *stream);

/*
 * gdn_chunk_fwd_pipelined -- gdn_chunk_fwd with the state-independent part of
 * every chunk prepared on SMs of its own and streamed to the SMs that carry the
 * states (one cooperative launch).
 *
 * Defines: the same function as gdn_chunk_fwd (section 2.1 "Gated DeltaNet" of
 * the page above, chunkwise WY evaluation).  Of each chunk's WY work, the gates,
 * the grams, the masked decay products, the triangular inverse (I + A)^-1 and
 * the scaled inverses do not depend on the state; "prep" CTAs compute them (the
 * grams once per QK head group) and pass them through a ring in the workspace
 * to "chain" CTAs, which keep each (sequence, V head)'s fp32 state in tensor
 * memory and run the state-dependent products chunk after chunk.  With few
 * sequences x heads (long prompts at small batch) most SMs prepare and the
 * chains run at the speed of their own products; with many, chains and prep
 * share the SMs.
 *
 * Arguments as gdn_chunk_fwd, plus:
 *   opts       NULL for the defaults, or:
 *                chain_ctas         CTAs that carry states (0 = automatic: all
 *                                   B*Hv heads at once when that is at most half
 *                                   of the SMs, else about 60% of them); rounded
 *                                   down to a multiple of Hv/Hqk
 *                wait_limit_cycles  SM clocks any wait inside the kernel may take
 *                                   before it gives up (0 = 2^32, about 2 s); a
 *                                   wait that gives up makes every CTA stop and
 *                                   is reported by gdn_device_status (the
 *                                   outputs are then undefined)
 *   workspace  device scratch of at least gdn_chunk_fwd_pipelined_workspace(...)
 *              bytes (for this device), 256-byte aligned, owned by the caller;
 *              its contents on entry do not matter; calls sharing it must not
 *              overlap.
 * Only GDN_BF16 takes this path; GDN_F32 (and B == 0 or T == 0) is
 * gdn_chunk_fwd, workspace unused.  Needs all its CTAs resident at once (one per
 * SM); if other work on the device prevents that, the launch waits for it, and a
 * device too small returns GDN_ERR_CUDA.  The results agree with
 * gdn_chunk_fwd's tensor-core kernel to a few bf16 ulp.  The products are the
 * same, but the diagonal decay scalings are rounded to bf16 at other points.
 * Every reduction runs in a fixed order, so repeated calls on the same inputs
 * return the same bits.  The workspace holds a 16-slot ring of 49 KB per chain
 * CTA plus one cache line of flags per chain CTA: 37 MB for B=1 with 48 V heads.
 */
typedef struct {
    int chain_ctas;
    long long wait_limit_cycles;
} gdn_pipeline_options;

size_t gdn_chunk_fwd_pipelined_workspace(int B, int Hqk, int Hv, int dk, int dv);
gdn_status gdn_chunk_fwd_pipelined(const void *q, const void *k, const void *v,
                                   const float *alpha, const float *beta, const float *S0,
                                   void *o, float *S_final,
                                   int B, int T, int Hqk, int Hv, int dk, int dv, int chunk,
                                   gdn_dtype dtype, const gdn_pipeline_options *opts,
                                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdn_device_status -- waits for `stream`, then reports and clears the device
 * error words of the tensor-core prefill kernels.  Returns GDN_ERR_TIMEOUT if a
 * bounded wait inside any of them gave up since the last call (on any stream:
 * the words are per library, not per call), GDN_ERR_CUDA if the stream reports
 * an error, else GDN_OK.  The kernels never trap or hang: a wait that gives up
 * ends its launch early, leaves its outputs undefined and the device usable.
 * This call synchronises, so call it where a check is wanted (tests, after a
 * batch), not on every step.
 */
gdn_status gdn_device_status(void *stream);

/*
 * gdn_chunk_fwd_split_noalloc -- gdn_chunk_fwd_split for callers that cannot
 * allocate device memory: its scratch is a static device array inside the
 * library (48 MiB, 256-byte aligned) instead of a caller workspace.
 *
 * The pages have no counterpart of this entry point; it is a deployment
 * variant of gdn_chunk_fwd_split, which defines what it computes.
 *
 * Arguments and results as gdn_chunk_fwd_split without workspace and
 * workspace_bytes.
 * - A GDN_BF16 problem whose split scratch (gdn_chunk_fwd_split_workspace,
 *   under the calling thread's kernel choice) is over 48 MiB returns
 *   GDN_ERR_UNSUPPORTED.
 * - Every call looks up the array's address in the current device's context
 *   (cudaGetSymbolAddress); the current device must be the one that holds the
 *   data.  A failed lookup returns GDN_ERR_CUDA.
 * - With lazy module loading (CUDA_MODULE_LOADING=LAZY, the default of recent
 *   CUDA), the module that holds the array is loaded, and its 48 MiB reserved,
 *   by the first call on each device (or by the first use of any kernel of the
 *   library).  A caller with a fixed memory plan makes one call as a warm-up
 *   before the plan is fixed, and before any stream capture.  After that no
 *   call changes the device's free memory.
 * - Every call shares the one array, so calls that overlap on the GPU (on
 *   different streams, or from different threads) race.
 * - Nothing in the array has to start at zero.
 * - The call allocates nothing.
 */
gdn_status gdn_chunk_fwd_split_noalloc(const void *q, const void *k, const void *v,
                                       const float *alpha, const float *beta, const float *S0,
                                       void *o, float *S_final,
                                       int B, int T, int Hqk, int Hv, int dk, int dv, int chunk,
                                       int segments, gdn_dtype dtype, void *stream);

/*
 * gdn_decode_step -- one token for each of B sequences (autoregressive decode).
 *
 * Defines: the first form of the update in section 2.1 "Gated DeltaNet",
 * applied once: p = S^T k, u = beta (v - alpha p), S' = alpha S + k u^T,
 * o = S'^T q (evaluated as alpha S^T q + (k . q) u, which is equal).
 *
 * In:  q, k [B, Hqk, dk]; v [B, Hv, dv]; alpha, beta [B, Hv]; S [B, Hv, dk, dv].
 * Out: o [B, Hv, dv]; S_new [B, Hv, dk, dv] -- may be the same buffer as S
 *      (in-place update, the normal use); any other overlap is undefined.
 * Sizes: B >= 0 (0 is a no-op), Hqk >= 1, Hv % Hqk == 0, dk == dv == 128.
 */
gdn_status gdn_decode_step(const void *q, const void *k, const void *v,
                           const float *alpha, const float *beta, const float *S,
                           void *o, float *S_new,
                           int B, int Hqk, int Hv, int dk, int dv,
                           gdn_dtype dtype, void *stream);

/*
 * gdn_decode_tokens -- n tokens per sequence in one call (multi-token decode and
 * verification of speculative drafts), with the state after every token kept
 * for rollback.
 *
 * Defines: the update of gdn_decode_step applied to tokens 0 .. n-1 in order.
 * Use: "Qwen3.8-Flash-Next 技术总结 -- Qwen4 架构的探路者", section 2.5 (MTP):
 * the multi-token prediction head drafts several tokens per step for
 * speculative decoding, and the backbone checks them in one pass.  If only
 * the first m drafts are accepted, the state to continue from is S_steps[:, m-1].
 *
 * In:  q, k [B, n, Hqk, dk]; v [B, n, Hv, dv]; alpha, beta [B, n, Hv];
 *      S [B, Hv, dk, dv].
 * Out: o [B, n, Hv, dv], o_t read after token t's update;
 *      S_new [B, Hv, dk, dv], the state after token n-1 (may be S itself);
 *      S_steps [B, n, Hv, dk, dv] or NULL, the state after every token
 *      (it must not overlap S or S_new).
 * Sizes: B >= 0, 1 <= n <= 64 (n > 64: GDN_ERR_UNSUPPORTED), heads as for
 *      gdn_decode_step.  n == 1 with S_steps == NULL is gdn_decode_step.
 */
gdn_status gdn_decode_tokens(const void *q, const void *k, const void *v,
                             const float *alpha, const float *beta, const float *S,
                             void *o, float *S_new, float *S_steps,
                             int B, int n, int Hqk, int Hv, int dk, int dv,
                             gdn_dtype dtype, void *stream);

/*
 * gdn_decode_step_slots -- one decode token for B sequences whose states live
 * in a shared pool, updated in place (continuous batching: the sequences of a
 * step are any subset of the pool, in any order).
 *
 * Defines: the update of gdn_decode_step, with sequence b's state at
 * state_pool[slots[b]].  Use: continuous batching in serving
 * ("通义千问Qwen3.8-Flash-Next开源：四大架构升级与部署优化全解析", section
 * "性能表现与开源生态支持").
 *
 * In:  q, k [B, Hqk, dk]; v [B, Hv, dv]; alpha, beta [B, Hv];
 *      slots [B] int32 (device); state_pool [n_slots, Hv, dk, dv] fp32.
 * Out: o [B, Hv, dv]; state_pool[slots[b]] updated in place.
 * A slot outside [0, n_slots) marks a padding entry: sequence b is skipped, its
 * o row is left as it was and no state changes.  Two entries with the same slot
 * race (undefined result).  slots must be 4-byte aligned; the other pointers
 * 16-byte aligned.
 */
gdn_status gdn_decode_step_slots(const void *q, const void *k, const void *v,
                                 const float *alpha, const float *beta,
                                 float *state_pool, const int *slots, void *o,
                                 int B, int n_slots, int Hqk, int Hv, int dk, int dv,
                                 gdn_dtype dtype, void *stream);

/*
 * Prefill kernel selection (library-specific: the page describes the method,
 * not how its evaluation is split over the GPU).
 *
 *   GDN_PREFILL_AUTO   default: GDN_BF16 runs on the tensor cores
 *                      (GDN_PREFILL_TC), GDN_F32 on the CUDA-core kernel
 *   GDN_PREFILL_SIMT   CUDA-core chunk kernel, both dtypes
 *   GDN_PREFILL_TC     tensor cores, one CTA per (sequence, V head)
 * All variants compute the same function, each to its dtype's rounding (the
 * tensor-core kernel with bf16 operands, the CUDA-core kernel in fp32).  The TC
 * variant takes GDN_BF16 only: with another choice gdn_chunk_fwd returns
 * GDN_ERR_UNSUPPORTED, as it does when the tensor-map encoder is missing.
 *
 * gdn_set_prefill_kernel sets the choice for the later gdn_chunk_fwd,
 * gdn_chunk_fwd_varlen and gdn_chunk_fwd_split calls of the CALLING THREAD only
 * (a per-thread setting; other threads keep their own, AUTO unless they set
 * one); it returns GDN_ERR_INVALID_ARG for a value outside the enum.
 * gdn_get_prefill_kernel returns the calling thread's current choice.
 */
typedef enum {
    GDN_PREFILL_AUTO = 0,
    GDN_PREFILL_SIMT = 1,
    GDN_PREFILL_TC = 2
} gdn_prefill_kernel;

gdn_status gdn_set_prefill_kernel(gdn_prefill_kernel kernel);
gdn_prefill_kernel gdn_get_prefill_kernel(void);

/*
 * The kernel (a gdn_prefill_kernel value, never GDN_PREFILL_AUTO) that
 * gdn_chunk_fwd runs for B sequences of Hv V heads in `dtype` under the calling
 * thread's current choice, on its current CUDA device; -1 if that call would
 * return GDN_ERR_UNSUPPORTED (a forced TC kernel with GDN_F32) or the arguments
 * are invalid.  No kernel is launched.
 */
int gdn_prefill_kernel_for(int B, int Hv, gdn_dtype dtype);

/*
 * gdn_bwd -- gradients of the chunked / token forward with respect to every input
 * (training).
 *
 * Defines: the derivative of L = sum_t <dO_t, o_t> + <dS_final, S_T> through the
 * recurrence of "Qwen3.8-Flash-Next 技术总结 -- Qwen4 架构的探路者", section 2.1
 * "Gated DeltaNet" (the pages give the forward only and say that the chunkwise
 * form is what makes training efficient; the gradients are the chain rule
 * applied to it).  Walking t down with G = dL/dS_t:
 *   G += q_t dO_t^T;  x = G^T k_t;  w = S_{t-1}^T k_t;  r = v_t - alpha_t w
 *   dq_t += S_t dO_t;  dk_t += beta_t G r - alpha_t beta_t S_{t-1} x;  dv_t = beta_t x
 *   dbeta_t = x . r;  dalpha_t = <G, S_{t-1}> - beta_t x . w
 *   G <- alpha_t (G - beta_t k_t x^T);   dS0 = G at the end.
 * dq and dk of a QK head sum over the V heads that read it.  The forward states
 * are recomputed inside the call (from checkpoints every 16 tokens kept in the
 * workspace); the gradients do not depend on how the forward was evaluated.
 *
 * In:  q, k [B, T, Hqk, dk]; v [B, T, Hv, dv]; dO [B, T, Hv, dv], all of dtype;
 *      alpha, beta [B, T, Hv] fp32; S0, dS_final [B, Hv, dk, dv] fp32 or NULL
 *      (zeros).
 * Out (fp32, overwritten): dq, dk [B, T, Hqk, dk]; dv [B, T, Hv, dv];
 *      dalpha, dbeta [B, T, Hv]; dS0 [B, Hv, dk, dv].  Outputs must not overlap
 *      inputs or each other.
 * workspace: device scratch of at least gdn_bwd_workspace(B, T, Hv, dk, dv)
 *      bytes (B * Hv * (ceil(T/16) + 16) * 64 KiB), 256-byte aligned, owned by
 *      the caller; contents on entry do not matter; calls sharing it must not
 *      overlap.  May be NULL when that size is 0 (T == 0).
 * Sizes and errors as gdn_chunk_fwd (heads, dtype; B <= 65535); pointers other
 * than the workspace 16-byte aligned.  dq, dk, dalpha, dbeta are accumulated
 * with fp32 atomic adds, so their last bits may differ between calls.
 */
size_t gdn_bwd_workspace(int B, int T, int Hv, int dk, int dv);
gdn_status gdn_bwd(const void *q, const void *k, const void *v, const float *alpha,
                   const float *beta, const float *S0, const void *dO, const float *dS_final,
                   float *dq, float *dk, float *dv, float *dalpha, float *dbeta, float *dS0,
                   int B, int T, int Hqk, int Hv, int dk_, int dv_, gdn_dtype dtype,
                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdn_bwd_chunk -- the same gradients as gdn_bwd, computed in the chunkwise (WY)
 * form on tensor cores; bf16 q, k, v, dO only.
 *
 * Defines: the chain rule through the chunk equations of the WY evaluation of
 * section 2.1 "Gated DeltaNet" of "Qwen3.8-Flash-Next 技术总结 -- Qwen4 架构的探路者"
 * (the pages name the WY representation as what makes the layer trainable in
 * parallel).  Per chunk of 64 tokens, from the chunk's start state S, with
 * b = cumsum(log alpha), gamma = exp(b), Gam = exp(b_r - b_i) (i <= r),
 * g = exp(b_63 - b), T = (I + strict_lower(diag(beta)(Gam o K K^T)))^-1:
 *   W = T diag(beta gamma) K, U = T diag(beta) V - W S, O = diag(gamma) Q S + (Gam o Q K^T) U,
 *   S' = gamma_63 S + K^T diag(g) U;
 * serially from the last chunk, dU = diag(g) K dS' + (Gam o Q K^T)^T dO and
 * dS = gamma_63 dS' + Q^T diag(gamma) dO - W^T dU; every other gradient per
 * chunk from S, dS', U and dU.  Four launches: preparation (per chunk and QK
 * head), forward state chain and gradient chain (per V head and 64 value
 * columns), per-chunk gradients (per chunk and QK head).  Operands are bf16 (the
 * start states, U, W, T, dU and dS' included), accumulation fp32; each output is
 * within 2e-2 of max|ref| of the exact gradients (the forward's bf16 bar), and
 * bitwise the same from call to call (no atomics).
 *
 * In / Out: as gdn_bwd, dtype GDN_BF16 (GDN_F32 -> GDN_ERR_UNSUPPORTED).
 * workspace: device scratch of at least gdn_bwd_chunk_workspace(B, T, Hv, dk, dv)
 *      bytes (about 128 KiB per chunk of 64 tokens and V head), 256-byte
 *      aligned, owned by the caller; contents on entry do not matter; calls
 *      sharing it must not overlap.  May be NULL when that size is 0 (T == 0).
 * Sizes and errors as gdn_bwd; ceil(T / 64) <= 2^31 - 1 and Hqk <= 65535.
 */
size_t gdn_bwd_chunk_workspace(int B, int T, int Hv, int dk, int dv);
gdn_status gdn_bwd_chunk(const void *q, const void *k, const void *v, const float *alpha,
                         const float *beta, const float *S0, const void *dO, const float *dS_final,
                         float *dq, float *dk, float *dv, float *dalpha, float *dbeta, float *dS0,
                         int B, int T, int Hqk, int Hv, int dk_, int dv_, gdn_dtype dtype,
                         void *workspace, size_t workspace_bytes, void *stream);

/* Static, NUL-terminated name of a status code. */
const char *gdn_status_string(gdn_status status);

/* The cudaError_t value behind the calling thread's last GDN_ERR_CUDA (0 if none). */
int gdn_last_cuda_error(void);

/* Library version as MAJOR * 10000 + MINOR * 100 + PATCH. */
int gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
