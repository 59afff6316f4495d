/* svd_vocab.h -- C ABI of the vocab-sharded verify-and-distill pass.
 *
 * The same computation as svd_verify_distill (include/svd.h) when every logit row is split
 * over P ranks by vocabulary id, as a tensor-parallel LM head leaves it: rank r holds ids
 * [v0, v0 + Vl) of every draft and target row.  Truncated verification (Pith verdict record,
 * skeptic_critique.load_bearing_attack: only the first b_k drafts are verified), greedy or
 * speculative sampling (acceptance u < min(1, p/q), residual resampling from max(0, p - q),
 * a bonus draw from p: Pith review page, Axiom & Free-Parameter Ledger), and the lambda-mixed
 * CE + entry-wise clipped reverse-KL loss with its gradient (Pith review page, "What carries
 * the argument"; Referee report major comment 2) -- with the readings of svd.h.
 *
 * A row's result depends on row-global quantities (maxima, log-sum-exps, the clip sums, the
 * sample's mass interval), so each rank reduces its slice to a fixed-size record and the
 * ranks exchange those records.  One step on each rank is:
 *
 *   svd_vs_stats    (this rank's slice)          -> send1            [B*kt records, 48 B]
 *   all-gather      send1 of every rank          -> recv1            [P][B*kt records]
 *   svd_vs_resolve  (recv1, this rank's slice)   -> send2, workspace [B*kt records, 32 B]
 *   all-gather      send2 of every rank          -> recv2            [P][B*kt records]
 *   svd_vs_finish   (recv2, this rank's slice)   -> outputs
 *   stochastic mode only: element-wise max over ranks of `emitted` (and of row_info's
 *   sample_token column), since only the rank whose slice holds the correction / bonus token
 *   writes it and every other rank writes -1 there.
 *
 * The all-gathers are the caller's (NCCL over NVLink from torch.distributed in the Python
 * package): the library calls no collective and no kernel waits for another rank.  Every rank
 * combines the gathered records in rank order with the same code, so all decisions (b_k
 * prefix, acceptance, clip candidates, which rank owns the sample) are identical on every
 * rank.  Rank r's record must sit at index r of recv1 / recv2 (the layout of an all-gather).
 *
 * Conventions as in svd.h: bf16 as uint16_t bits, device pointers, rows contiguous, every
 * call enqueues on `stream` and never synchronizes, argument errors are returned before any
 * launch, device errors (a draft token outside [0, V)) go to the workspace status word and are
 * read with svd_get_device_error(ws).  The workspace must be zero before its first use.
 * Limits: 1 <= k <= 32, kt in {k, k+1}, 1 <= Vl, 0 <= v0, v0 + Vl <= V < 2^31, 1 <= P <= 64.
 * The slices of the P ranks must tile [0, V) (not checkable by one rank).  The fast path needs
 * Vl % 8 == 0 and 16-byte aligned D, T and dlogits; other slices take plain loads and stores.
 */
#ifndef SVD_VOCAB_H
#define SVD_VOCAB_H

#include "svd.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct svd_vs_args {
    const uint16_t* D;          /* [B, k, Vl] this rank's slice of the draft logits            */
    const uint16_t* T;          /* [B, kt, Vl] this rank's slice of the target logits          */
    const int32_t* draft_tok;   /* [B, k] global token ids, or NULL (greedy only): x = argmax
                                 * of the draft row over all V ids, lowest id on ties          */
    const int32_t* bk;          /* [B] b_k in [1, k], identical on every rank (clamped)        */
    int B, k, kt;
    int V;                      /* full vocabulary size                                        */
    int v0, Vl;                 /* this rank's ids: [v0, v0 + Vl)                              */
    int P, rank;                /* number of ranks, this rank                                  */
    svd_mode mode;
    float temperature;          /* tau > 0                                                     */
    uint64_t seed, step;        /* Philox key and step counter (stochastic mode)               */
    int distill;                /* 1: loss and gradient as well, 0: verification only          */
    float lambda, clip_c, grad_scale;
    void* dlogits;              /* [B, k, Vl] this rank's gradient slice, bf16 or fp32; rows
                                 * i >= b_k are zero (distill only)                            */
    int dlogits_fp32;
    float* loss_rows;           /* [B, k] or NULL; identical on every rank                     */
    float* loss_total;          /* [1] (distill only); identical on every rank                 */
    int32_t* accept_len;        /* [B], identical on every rank                                */
    int32_t* emitted;           /* [B, k+1], -1 padded; greedy: identical on every rank;
                                 * stochastic: the correction / bonus token only on its owner  */
    int32_t* n_emitted;         /* [B], identical on every rank                                */
    svd_row_info* row_info;     /* [B, kt] or NULL; stochastic sample_token as `emitted`       */
} svd_vs_args;

/* Bytes of one rank's exchange record buffer: which = 1 (send1) or 2 (send2).  The gathered
 * buffers recv1 / recv2 are P times that.  0 for bad arguments. */
size_t svd_vs_exchange_bytes(int B, int kt, int which);

/* Workspace bytes of one rank (256-byte aligned base, zero before first use). */
size_t svd_vs_workspace_bytes(int B, int k, int kt);

/* Step 1: partial statistics of this rank's slice of every processed row (the b_k verified
 * rows and the bonus row) into send1. */
svd_status svd_vs_stats(const svd_vs_args* a, void* send1, void* ws, size_t ws_bytes,
                        void* stream);

/* Step 2: combines the gathered records recv1 (every rank's send1, rank order) into the
 * row-global statistics and decisions (kept in the workspace; accept_len, n_emitted, emitted
 * and row_info written), then reduces this rank's slice of the rows that need it (clip
 * candidates, the correction / bonus row's sample masses) into send2. */
svd_status svd_vs_resolve(const svd_vs_args* a, const void* recv1, void* send2, void* ws,
                          size_t ws_bytes, void* stream);

/* Step 3: combines recv2 (every rank's send2, rank order); writes this rank's gradient slice,
 * the loss rows and total, and, on the rank whose slice holds it, the sampled token. */
svd_status svd_vs_finish(const svd_vs_args* a, const void* recv2, void* ws, size_t ws_bytes,
                         void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SVD_VOCAB_H */
