/*
 * svd.h -- C ABI of libsvd.so: fused speculative verify-and-distill for B200 (sm_100a).
 *
 * The operations restate the hot path of AdaFlash (arXiv 2607.19223) as the Pith review page
 * "AdaFlash: Adaptive Speculative Decoding via On-Policy Distilled Diffusion Drafters" and the
 * Pith verdict record describe it:
 *   - a small length head on pooled drafter hidden states predicts the block's acceptance rate
 *     bhat and sets the verification length b_k ("What carries the argument"; Referee Report,
 *     minor comment 2, their section 3.2; free parameter gamma in the Axiom & Free-Parameter
 *     Ledger);
 *   - only the first b_k drafts are verified against the target (verdict record,
 *     skeptic_critique.load_bearing_attack), by the standard speculative-decoding acceptance
 *     rule (Axiom ledger: Leviathan et al. 2023): greedy, or accept when u < min(1, p/q) with a
 *     residual resample from max(0, p - q);
 *   - the drafter is distilled from the same verification logits with a convex mix of
 *     hard-label cross-entropy and reverse-KL with entry-wise clipping ("What carries the
 *     argument"; Axiom ledger alpha, delta and temperature; Referee major comment 2).
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller, row-major and contiguous.
 *     bf16 tensors are passed as their 16-bit patterns (uint16_t).  The library never frees or
 *     retains them beyond the call's stream work.
 *   - Every call is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream) and
 *     never synchronizes.  Argument errors are returned before anything is launched.  Launch
 *     failures return SVD_ERR_CUDA.  Errors found on the device (a draft token outside [0,V), a
 *     bounded wait that ran out) are recorded in the workspace status word and read with
 *     svd_get_device_error().
 *   - The library allocates no device memory.  Scratch lives in the caller's workspace `ws` of
 *     at least svd_workspace_bytes() bytes, 256-byte aligned.  The workspace must be all zero
 *     before its first use (cudaMemset, torch.zeros, or svd_workspace_reset); every call that
 *     completes leaves it zero again, apart from the device status word.  After a device error
 *     reset it.  Calls that share a workspace must not overlap on the GPU; calls on different
 *     workspaces are independent and may run concurrently on different streams.
 *   - Limits: 1 <= k <= 32, kt in {k, k+1}, 1 <= V <= 327680, b_k in [1, k].  The fast path
 *     needs V % 8 == 0 and 16-byte aligned logit / gradient pointers; other shapes take a
 *     slower path with plain loads and stores.
 *   - Positions are 0-based: sequence b verifies draft rows i = 0 .. b_k-1.
 */
#ifndef SVD_H
#define SVD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum svd_status {
    SVD_OK = 0,
    SVD_ERR_INVALID_ARG = 1,   /* bad size, null required pointer, k/kt/b_k out of range */
    SVD_ERR_ALIGNMENT = 2,     /* workspace not 256-byte aligned */
    SVD_ERR_WORKSPACE = 3,     /* workspace smaller than svd_workspace_bytes() */
    SVD_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
    SVD_ERR_TIMEOUT = 5,       /* device: a bounded wait ran out (status word only) */
    SVD_ERR_UNSUPPORTED = 6,   /* shape outside the supported range (e.g. V too large) */
    SVD_ERR_TOKEN_RANGE = 7    /* device: a caller draft token outside [0, V) (status word) */
} svd_status;

typedef enum svd_mode {
    SVD_GREEDY = 0,            /* accept x_i iff x_i == argmax T_i (lowest id on ties) */
    SVD_STOCHASTIC = 1         /* accept iff u_i < min(1, p_i(x_i) / q_i(x_i)) */
} svd_mode;

typedef enum svd_bk_round {
    SVD_BK_CEIL = 0,           /* b_k = clamp(ceil(gamma * bhat * k), 1, k)  (default reading) */
    SVD_BK_FLOOR = 1           /* b_k = clamp(floor(gamma * bhat * k), 1, k) (referee's quote)  */
} svd_bk_round;

/* Per-row diagnostics, optional output of shape [B, kt].  Rows that were not processed hold
 * -1 in the integer fields and NaN in the float fields (loss 0). */
typedef struct svd_row_info {
    int32_t draft_token;    /* x_i: caller token or argmax of the draft row; -1 if unverified */
    int32_t target_argmax;  /* argmax of the target row (verified rows and the bonus row)     */
    int32_t accepted;       /* 1 / 0 acceptance decision; -1 if the row was not verified      */
    int32_t sample_token;   /* greedy: the target argmax of the row.  Stochastic: the drawn
                             * correction / bonus token on the row it was drawn from (the
                             * first rejected row, else the bonus row); -1 on other rows     */
    float ratio;            /* p_i(x_i) / q_i(x_i) in stochastic mode, NaN otherwise           */
    float lse_draft;        /* log sum_v exp(D_i,v / tau), NaN if not computed                */
    float lse_target;       /* log sum_v exp(T_i,v / tau), NaN if not computed                */
    float loss;             /* row loss L_i of the distillation objective (0 if not computed) */
} svd_row_info;

/* Workspace size in bytes for a batch of B sequences, blocks of k drafts, kt target rows per
 * sequence and a length head with M hidden units (M = 0 if svd_length_head is not used). */
size_t svd_workspace_bytes(int B, int k, int kt, int M);

/* Zero the whole workspace on `stream` (one cudaMemsetAsync). */
svd_status svd_workspace_reset(void* ws, size_t ws_bytes, void* stream);

/* a1 -- adaptive length head (Pith review "What carries the argument"; Axiom ledger, "maps a
 * pooled representation to a single scalar ... linearly converted"; Referee minor comment 2).
 *   hidden_m = relu( sum_j W1[m,j] h[b,j] + b1[m] ),  z_b = sum_m w2[m] hidden_m + b2,
 *   bhat_b = sigmoid(z_b),  b_k = clamp(round(gamma * bhat_b * k), 1, k) with round = ceil or
 *   floor per `rnd`.
 * h [B,H] bf16 (pooled drafter hidden states), W1 [M,H] bf16 (nn.Linear layout), b1 [M] fp32
 * or NULL, w2 [M] bf16, b2 scalar.  Outputs bhat_out [B] fp32 (may be NULL), bk_out [B] int32.
 * fp32 accumulation on tensor cores.  Uses the workspace (per-tile partial sums, a ticket). */
svd_status svd_length_head(const uint16_t* h, const uint16_t* W1, const float* b1,
                           const uint16_t* w2, float b2, int B, int H, int M, int k,
                           float gamma, svd_bk_round rnd, float* bhat_out, int32_t* bk_out,
                           void* ws, size_t ws_bytes, void* stream);

/* a2 + a3 + a4 -- truncated verification (verdict record, load_bearing_attack; acceptance rule
 * of the Axiom ledger).  D [B,k,V] draft logits, T [B,kt,V] target logits (bf16); draft_tok
 * [B,k] int32 (NULL in greedy mode means x_i = argmax D_i; required in stochastic mode); bk [B]
 * verification lengths.  For each sequence: a = first i < b_k that is rejected, else b_k;
 * emitted = x_0..x_{a-1}, then the correction token at row a if a < b_k (greedy: argmax T_a;
 * stochastic: residual sample from max(0, p_a - q_a)), else the bonus token from row b_k if
 * b_k < kt (greedy: argmax; stochastic: sample from p).  Philox4x32-10 uniforms: key = seed,
 * counter = (position, sequence, step); word 0 = accept uniform, word 1 = resample uniform.
 * Outputs: accept_len [B], emitted [B,k+1] (-1 padded), n_emitted [B], row_info [B,kt] or NULL. */
svd_status svd_verify(const uint16_t* D, const uint16_t* T, const int32_t* draft_tok,
                      const int32_t* bk, int B, int k, int kt, int V, svd_mode mode,
                      float temperature, uint64_t seed, uint64_t step, int32_t* accept_len,
                      int32_t* emitted, int32_t* n_emitted, svd_row_info* row_info, void* ws,
                      size_t ws_bytes, void* stream);

/* a5 -- distillation loss and its gradient w.r.t. the draft logits (Pith review "What carries
 * the argument"; Axiom ledger alpha/delta/temperature; Referee major comment 2).  For rows
 * i < b_k, with q = softmax(D_i/tau), p = softmax(T_i/tau), y = argmax T_i:
 *   d_v = q_v (log q_v - log p_v),  K_c = sum_v min(d_v, c),  L_i = lambda (-log q_y) + (1-lambda) K_c
 *   dL/dD_u = (grad_scale/tau) [lambda (q_u - [u=y]) + (1-lambda) q_u (m_u (s_u+1) - S)],
 *   s_u = log q_u - log p_u, m_u = [d_u <= c], S = sum_v m_v q_v (s_v + 1).
 * Rows i >= b_k get L_i = 0 and a zero gradient row.  clip_c may be +INFINITY (plain
 * reverse-KL).  Outputs: loss_rows [B,k] fp32 or NULL, loss_total [1] fp32 (sum of all row
 * losses, unscaled), dlogits [B,k,V] bf16 (dlogits_fp32 = 0) or fp32 (dlogits_fp32 = 1). */
svd_status svd_distill_loss_grad(const uint16_t* D, const uint16_t* T, const int32_t* bk,
                                 int B, int k, int kt, int V, float lambda, float clip_c,
                                 float temperature, float grad_scale, float* loss_rows,
                                 float* loss_total, void* dlogits, int dlogits_fp32, void* ws,
                                 size_t ws_bytes, void* stream);

/* Arguments of the fused call.  Set h = NULL to skip the length head and use bk_in. */
typedef struct svd_verify_distill_args {
    /* length head (a1) */
    const uint16_t* h;       /* [B,H] bf16 or NULL                      */
    const uint16_t* W1;      /* [M,H] bf16                              */
    const float* b1;         /* [M] fp32 or NULL                        */
    const uint16_t* w2;      /* [M] bf16                                */
    float b2;
    int H, M;
    float gamma;
    svd_bk_round rnd;
    const int32_t* bk_in;    /* [B] used when h == NULL                 */
    /* logits */
    const uint16_t* D;       /* [B,k,V] bf16                            */
    const uint16_t* T;       /* [B,kt,V] bf16                           */
    const int32_t* draft_tok;/* [B,k] or NULL (greedy)                  */
    int B, k, kt, V;
    /* verification (a2-a4) */
    svd_mode mode;
    float temperature;
    uint64_t seed, step;
    /* distillation (a5) */
    float lambda, clip_c, grad_scale;
    int dlogits_fp32;
    /* outputs */
    float* bhat;             /* [B] or NULL                             */
    int32_t* bk;             /* [B] verification lengths used (required)*/
    int32_t* accept_len;     /* [B]                                     */
    int32_t* emitted;        /* [B,k+1]                                 */
    int32_t* n_emitted;      /* [B]                                     */
    float* loss_rows;        /* [B,k] or NULL                           */
    float* loss_total;       /* [1]                                     */
    void* dlogits;           /* [B,k,V] bf16 / fp32                     */
    svd_row_info* row_info;  /* [B,kt] or NULL                          */
    /* Length-head labels.  The head's online update fits bhat to an acceptance label a*; under
     * truncated verification only a/b_k is observable (Pith verdict record, load_bearing_attack),
     * and its proposed test (concrete_test; the review page's falsifier) verifies all k drafts to
     * obtain the full-block label a/k.  full_k = 1 runs that variant: b_k (the head's choice, or
     * bk_in) is still computed and written to `bk`, but every sequence verifies and distills all
     * k rows; accept_len, emitted, n_emitted, the losses and the gradient are those of the
     * full-k pass.  Acceptance is a prefix scan and each decision depends only on its own row,
     * so min(a, b_k) is exactly the acceptance truncated verification would have seen. */
    int full_k;              /* 0 or 1                                                        */
    float* label_proxy;      /* [B] or NULL: a / b_k as truncated verification observes it;
                              * with full_k = 1, min(a, b_k) / b_k                            */
    float* label_full;       /* [B] or NULL: a / k with full_k = 1; NaN with full_k = 0         */
    /* [B,M] fp32 or NULL: the head's pre-activations W1 h + b1, written when the head runs.  With
     * `bhat`, they are the forward an online update of the head on the same hidden states and
     * served weights needs (svd_head_update_args.preact), so that update need not recompute it. */
    float* head_preact;
} svd_verify_distill_args;

/* a1 .. a5 in one call: the length head (unless h == NULL), then one persistent pass over the
 * logits that verifies, samples and writes the loss and gradient.  Same semantics as calling
 * svd_length_head, svd_verify and svd_distill_loss_grad in turn, with each logit row read
 * from HBM once. */
svd_status svd_verify_distill(const svd_verify_distill_args* args, void* ws, size_t ws_bytes,
                              void* stream);

/* Largest workspace svd_verify_distill_noalloc can stand in for (4 MiB per device). */
#define SVD_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)

/* svd_verify_distill without a caller workspace, for callers that cannot allocate device
 * memory: a C host program with no device allocator, or a runtime that has claimed nearly all
 * HBM for its own pools and forbids cudaMalloc on its path (cudaMalloc may synchronise the
 * device and fails once the memory is claimed).  The paper has no counterpart: it is a
 * deployment variant of the fused call above, with identical arguments, kernels and results.
 *
 * Scratch: a file-scope device array of SVD_NOALLOC_SCRATCH_BYTES in the library, one per
 * device.  Nothing is allocated, by the library or by anything it calls.
 *   - Set-up: the first call in each CUDA context (the runtime's primary context of a device,
 *     or a driver-API context the caller made current) looks up the array's address in that
 *     context and caches it under the context's unique id; a context destroyed and created
 *     again (cudaDeviceReset) is a new context and is looked up again.  `stream` must belong
 *     to the current context.  Make the first call in a context before any stream capture
 *     begins.
 *   - Checks: every argument is checked before the scratch is touched; a rejected call
 *     enqueues nothing.
 *   - Zeroing: every call clears the svd_workspace_bytes(B, k, kt, M) bytes it uses with one
 *     cudaMemsetAsync on `stream`, so nothing needs to start at zero and an earlier device
 *     error leaves nothing behind.
 *   - Size limit: calls whose svd_workspace_bytes(B, k, kt, M) exceeds
 *     SVD_NOALLOC_SCRATCH_BYTES return SVD_ERR_WORKSPACE before anything is launched.
 *   - Concurrency: all calls in one context share the one array.  Calls that overlap on the
 *     GPU (different streams, or host threads enqueuing without ordering) race on it and give
 *     undefined results; order them on one stream or with events.
 *   - Device errors: if `status_out` (a caller-owned DEVICE pointer to one uint32_t) is not
 *     NULL, the call's device status word (SVD_OK, SVD_ERR_TOKEN_RANGE or SVD_ERR_TIMEOUT) is
 *     copied there on `stream` after the kernels.  It is written only when the call returns
 *     SVD_OK; after any other return code its contents are unchanged.
 * Other return codes as for svd_verify_distill. */
svd_status svd_verify_distill_noalloc(const svd_verify_distill_args* args, uint32_t* status_out,
                                      void* stream);

/* Length-head online update: one step of AdamW on the head's parameters for the loss
 *   l = (1/B) sum_b (bhat_b - a*_b)^2
 * (Pith verdict record, skeptic_critique.load_bearing_attack: l_len = (bhat - a*)^2 trains the
 * head online; Pith review page, Axiom & Free-Parameter Ledger: length-head learning rate 2e-4).
 * a* is the caller's label per sequence, e.g. label_proxy or label_full of svd_verify_distill.
 * The forward runs on the served bf16 weights W1, w2 with the fp32 b1 and b2 (the same head as
 * svd_length_head); the gradient goes to fp32 master weights W1m, w2m (b1, b2 are their own
 * masters), AdamW (decoupled weight decay, in the order of torch.optim.AdamW) updates them, and
 * W1, w2 are refreshed as their round-to-nearest-even bf16 copies.  No gradient flows into h.
 * The AdamW moments must be zero before step 1; `step` counts from 1.  All pointers are device
 * memory; every parameter and moment is updated in place on `stream`. */
typedef struct svd_head_update_args {
    const uint16_t* h;       /* [B,H] bf16 pooled hidden states                          */
    const float* label;      /* [B] fp32 acceptance labels a*                            */
    int B, H, M;
    float* W1m;              /* [M,H] fp32 master of W1                                  */
    float* b1;               /* [M] fp32                                                 */
    float* w2m;              /* [M] fp32 master of w2                                    */
    float* b2;               /* [1] fp32                                                 */
    uint16_t* W1;            /* [M,H] bf16 served copy (read by the forward, refreshed)  */
    uint16_t* w2;            /* [M] bf16 served copy                                     */
    float *mW1, *vW1, *mb1, *vb1, *mw2, *vw2, *mb2, *vb2;   /* AdamW moments, same shapes */
    int step;                /* 1, 2, ...                                                */
    float lr, beta1, beta2, eps, weight_decay;
    float* loss;             /* [1] out: l before the step                               */
    float* bhat;             /* [B] out: the forward's bhat before the step (an input when
                              * preact is given)                                         */
    /* [B,M] fp32 or NULL: pre-activations W1 h + b1 of a forward already run on these hidden
     * states with the current served weights (svd_verify_distill_args.head_preact, with that
     * call's bhat passed in `bhat`).  Then the update skips its own forward: one kernel instead
     * of two.  The caller guarantees that no step has changed the weights since that forward. */
    const float* preact;
} svd_head_update_args;

/* Workspace: svd_workspace_bytes(B, 1, 1, M) bytes. */
svd_status svd_length_head_update(const svd_head_update_args* args, void* ws, size_t ws_bytes,
                                  void* stream);

/* Speedup reporter for one verification step (Pith review page, Referee Report minor comment 1,
 * their Eq. 1: E[tau] = (1 - Acc^(k+1)) / (1 - Acc), eta = E[tau] / (rho*k + 1), which assumes
 * i.i.d. acceptance; the measured values are reported beside the model).  Inputs are the
 * step's outputs per sequence: accept_len a_b, bk n_b (rows verified) and n_emitted e_b, with
 * 0 <= a_b <= n_b <= k.  `rho` is the drafter-to-target cost ratio of the speedup formula.
 * Writes out [8 + k] fp64 (device):
 *   out[0] measured E[tau] = mean e_b (tokens per target verification)
 *   out[1] Acc = sum a_b / sum min(a_b + 1, n_b) (accepted / decisions taken)
 *   out[2] model E[tau] from Acc; out[3] eta = out[2] / (rho*k + 1); out[4] = out[0] / (rho*k + 1)
 *   out[5] mean n_b, out[6] mean a_b, out[7] B
 *   out[8 + i] acceptance at position i given an accepted prefix and a verified row:
 *              #{a_b > i} / #{a_b >= i and n_b > i} (NaN if no sequence reached row i). */
svd_status svd_speedup_report(const int32_t* accept_len, const int32_t* bk,
                              const int32_t* n_emitted, int B, int k, double rho, double* out,
                              void* stream);

/* Reads and clears the device status word of `ws` (synchronizes `stream`).  Returns SVD_OK,
 * SVD_ERR_TOKEN_RANGE or SVD_ERR_TIMEOUT as recorded by kernels that used this workspace, or
 * SVD_ERR_CUDA if the read itself failed. */
svd_status svd_get_device_error(void* ws, void* stream);

/* Human-readable name of a status code (static storage). */
const char* svd_status_string(svd_status s);

/* Test hook for the bounded-wait path: launches one block that waits on a barrier nothing will
 * complete, with a limit of `limit_ns` nanoseconds; the wait gives up, records SVD_ERR_TIMEOUT
 * in the status word of `ws` and the kernel returns normally.  Nothing hangs or faults. */
svd_status svd_selftest_wait_timeout(void* ws, size_t ws_bytes, uint64_t limit_ns,
                                     void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SVD_H */
