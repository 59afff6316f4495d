// svd_internal.h -- kernel parameter blocks, workspace layout and launch entry points shared by
// the C ABI layer (svd_api.cu) and the kernels (length_head.cu, verify_distill.cu).
#pragma once

#include <cstddef>
#include <cstdint>

#include "../../include/svd.h"

namespace svd {

// ------------------------------------------------------------------------------------------
// Workspace layout (all sections 256-byte aligned).  Everything except the status word is
// returned to zero by the kernel that used it.
// ------------------------------------------------------------------------------------------
struct WsHeader {
    uint32_t status;       // first device-side error (svd_status), sticky until read
    uint32_t head_ticket;  // length head: CTAs finished
    uint32_t loss_ticket;  // finalize pass: CTAs finished
    uint32_t item_ticket;  // row pass: next loaded row to hand out (reset by the finalize pass)
    uint32_t zero_ticket;  // row pass: next zero-gradient unit to hand out (reset likewise)
    uint32_t head_unit;    // row pass with the length head inside: next head unit to hand out
    uint32_t head_done;    // ... and the 16-sequence tiles whose b_k are written (both reset
                           // by the finalize pass)
    uint32_t update_ticket;  // length-head update: backward CTAs finished
    uint32_t pad[56];
};
static_assert(sizeof(WsHeader) == 256, "header is one 256-byte line");

constexpr int kHeadTileM = 64;   // hidden units per length-head CTA
constexpr int kHeadTileB = 16;   // sequences per length-head CTA

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// K splits of the length-head contraction: enough CTAs to cover the SMs twice over.
// K splits of the length head.  head_ws_splits: the splits the workspace holds partials for --
// enough work units to fill the GPU (about two per SM) and, when the head has at most 32 output
// tiles, at least 11, so that hidden sizes up to 11 x kHeadSplitCols columns split into pieces
// the fused pass stages in one chunk of its large-vocabulary staging area (kHeadSplitCols
// columns of 16 + 64 rows fit its 64 KB); at most kHeadMaxSplit.  head_nsplit: the splits a call
// uses, within that.
constexpr int kHeadMaxSplit = 16;
constexpr int kHeadSplitCols = 400;
__host__ __device__ inline int head_ws_splits(int B, int M) {
    if (B <= 0 || M <= 0) return 0;
    const int tiles = ((B + kHeadTileB - 1) / kHeadTileB) * ((M + kHeadTileM - 1) / kHeadTileM);
    int n = (296 + tiles - 1) / tiles;
    if (tiles <= 32 && n < 11) n = 11;
    return n < 1 ? 1 : (n > kHeadMaxSplit ? kHeadMaxSplit : n);
}
__host__ __device__ inline int head_nsplit(int B, int M, int H) {
    if (B <= 0 || M <= 0) return 0;
    const int tiles = ((B + kHeadTileB - 1) / kHeadTileB) * ((M + kHeadTileM - 1) / kHeadTileM);
    int n = (296 + tiles - 1) / tiles;
    const int nk = (H + kHeadSplitCols - 1) / kHeadSplitCols;
    if (nk > n) n = nk;
    const int cap = head_ws_splits(B, M);
    return n < 1 ? 1 : (n > cap ? cap : n);
}

struct WsLayout {
    size_t rec, seq_loss, zpart, part, tile_ticket, u, e, total;
};

__host__ __device__ inline WsLayout ws_layout(int B, int k, int kt, int M) {
    (void)k;
    WsLayout L;
    size_t off = sizeof(WsHeader);
    L.rec = off;
    off = align256(off + sizeof(svd_row_info) * (size_t)B * (size_t)kt);
    L.seq_loss = off;
    off = align256(off + sizeof(float) * (size_t)B);
    const int mt = M > 0 ? (M + kHeadTileM - 1) / kHeadTileM : 0;
    const int bt = (B + kHeadTileB - 1) / kHeadTileB;
    L.zpart = off;
    off = align256(off + sizeof(float) * (size_t)mt * (size_t)B);
    L.part = off;
    off = align256(off + sizeof(float) * (size_t)head_ws_splits(B, M) * (size_t)B * (size_t)(M > 0 ? M : 0));
    L.tile_ticket = off;   // output-tile tickets [bt * mt], then sequence-tile tickets [bt]
    off = align256(off + sizeof(uint32_t) * ((size_t)bt * (size_t)mt + (size_t)bt));
    // length-head update: pre-activations W1 h + b1 and backward terms, [B, M] fp32 each
    const size_t bm = (size_t)B * (size_t)(M > 0 ? M : 0);
    L.u = off;
    off = align256(off + sizeof(float) * bm);
    L.e = off;   // backward terms: the w2 and b1 gradients [2, M] (at least)
    off = align256(off + sizeof(float) * (bm > 2 * (size_t)(M > 0 ? M : 0) ? bm : 2 * (size_t)(M > 0 ? M : 0)));
    L.total = off;
    return L;
}

// ------------------------------------------------------------------------------------------
// length head
// ------------------------------------------------------------------------------------------
struct HeadParams {
    const uint16_t* h;
    const uint16_t* W1;
    const float* b1;
    const uint16_t* w2;
    float b2;
    int B, H, M, k;
    float gamma;
    int rnd;
    float* bhat;
    int32_t* bk;             // or null (no verification length wanted)
    const float* b2_dev;     // or null: b2 from device memory instead of the scalar
    float* u_out;            // or null: [B, M] pre-activations W1 h + b1
    WsHeader* hdr;
    float* zpart;            // [ceil(M/64), B] per-tile logits
    float* part;             // [nsplit, B, M] split partials of W1 h
    uint32_t* tile_ticket;   // [ceil(B/16) * ceil(M/64)] + [ceil(B/16)]
    int nsplit, ks;          // K splits and columns per split
};

// ------------------------------------------------------------------------------------------
// row pass (verify + distill)
// ------------------------------------------------------------------------------------------
// Batches up to this size keep b_k and the prefixes of loaded and zero-gradient rows per
// sequence in the row pass's shared memory (compact lists handed out dynamically); the length
// head runs inside the row pass only for such batches.
constexpr int kRowCompactMaxB = 4096;

enum : int {
    kFlagVerify = 1,
    kFlagDistill = 2,
    kFlagStochastic = 4,
};

struct RowParams {
    const uint16_t* D;
    const uint16_t* T;
    const int32_t* draft;
    const int32_t* bk;
    int B, k, kt, V;
    int chunk;         // logit elements per CTA of a row cluster (multiple of 8)
    int flags;
    int aligned;       // 1: TMA bulk staging and vector stores; 0: plain loads / stores
    float tau, inv_tau, k2;  // k2 = log2(e) / tau
    uint64_t seed, step;
    float lambda, clip_c, grad_scale;
    int dl_fp32;
    void* dlogits;
    float* loss_rows;
    float* loss_total;
    int32_t* accept_len;
    int32_t* emitted;
    int32_t* n_emitted;
    svd_row_info* row_info;
    WsHeader* hdr;
    svd_row_info* rec;
    float* seq_loss;
    uint64_t wait_limit_ns;
    int bk_const;                // > 0: every sequence verifies this many rows (full-k mode)
    const int32_t* bk_trunc;     // the truncated choice of b_k, for the labels
    float* label_proxy;          // [B] or null
    float* label_full;           // [B] or null
    // length head computed inside the row pass (b_k written to `bk` before rows past 0 start)
    int head_fused;
    HeadParams head;
};

// Launchers (return cudaError_t as int; 0 = success).
int launch_length_head(const HeadParams& p, void* stream);
int launch_row_pass(const RowParams& p, void* stream);
// stochastic mode, after the finalize pass: each sequence's correction / bonus draw
int launch_sample_fix(const RowParams& p, void* stream);
int launch_wait_timeout_selftest(WsHeader* hdr, uint64_t limit_ns, void* stream);
struct HeadUpdateParams {
    const uint16_t* h;
    const float* label;
    const float* bhat;
    const float* u;          // [B, M] pre-activations of the forward
    float* e;                // workspace: [M] the new w2 masters, until the last CTA copies them
    uint32_t* ticket;        // backward CTAs finished (back to zero after the step)
    int B, H, M;
    float *W1m, *b1, *w2m, *b2;
    uint16_t *W1, *w2;
    float *mW1, *vW1, *mb1, *vb1, *mw2, *vw2, *mb2, *vb2;
    float lr, beta1, beta2, eps, wd;
    float step_size, rsqrt_bc2;   // lr / (1 - beta1^step), 1 / sqrt(1 - beta2^step)
    float* loss;
};
int launch_head_update(const HeadUpdateParams& p, void* stream);
int launch_speedup_report(const int32_t* accept_len, const int32_t* bk, const int32_t* n_emitted,
                          int B, int k, double rho, double* out, void* stream);

// Cluster geometry chosen for a vocabulary size.
struct RowGeometry {
    int variant;   // 0: 128 threads x 2 vectors per lane; 1: 256 x 10
    int threads;
    int cluster;   // CTAs per row
    int chunk;     // elements per CTA
    size_t smem;   // dynamic shared memory per CTA
};
bool row_geometry(int V, RowGeometry* g);

// Argument checks of svd_verify_distill that need no workspace (SVD_OK when the call may go on).
svd_status check_verify_distill_args(const svd_verify_distill_args* a);

}  // namespace svd
