// svd_api.cu -- the C ABI: argument validation, workspace carving and launch sequencing on the
// caller's stream.  No device memory is allocated and no host synchronisation happens here
// (except in svd_get_device_error, which reads the status word back).
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>

#include "svd_internal.h"

using namespace svd;

namespace {

constexpr int kMaxK = 32;
constexpr int kMaxV = 327680;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

svd_status check_ws(void* ws, size_t ws_bytes, int B, int k, int kt, int M) {
    if (ws == nullptr) return SVD_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return SVD_ERR_ALIGNMENT;
    if (ws_bytes < ws_layout(B, k, kt, M).total) return SVD_ERR_WORKSPACE;
    return SVD_OK;
}

svd_status check_shape(int B, int k, int kt, int V) {
    if (B < 0 || k < 1 || k > kMaxK || (kt != k && kt != k + 1) || V < 1) return SVD_ERR_INVALID_ARG;
    if (V > kMaxV) return SVD_ERR_UNSUPPORTED;
    return SVD_OK;
}

struct WsPtrs {
    WsHeader* hdr;
    svd_row_info* rec;
    float* seq_loss;
    float* zpart;
    float* part;
    uint32_t* tile_ticket;
};

WsPtrs carve(void* ws, int B, int k, int kt, int M) {
    const WsLayout L = ws_layout(B, k, kt, M);
    char* base = static_cast<char*>(ws);
    WsPtrs w;
    w.hdr = reinterpret_cast<WsHeader*>(base);
    w.rec = reinterpret_cast<svd_row_info*>(base + L.rec);
    w.seq_loss = reinterpret_cast<float*>(base + L.seq_loss);
    w.zpart = reinterpret_cast<float*>(base + L.zpart);
    w.part = reinterpret_cast<float*>(base + L.part);
    w.tile_ticket = reinterpret_cast<uint32_t*>(base + L.tile_ticket);
    return w;
}

svd_status from_cuda(int err) { return err == 0 ? SVD_OK : SVD_ERR_CUDA; }

// Bound on any device-side wait: 1 s of wall-clock time (a staging copy lands in microseconds).
constexpr uint64_t kWaitLimitNs = 1000000000ull;

HeadParams head_params(const uint16_t* h, const uint16_t* W1, const float* b1, const uint16_t* w2,
                       float b2, int B, int H, int M, int k, float gamma, svd_bk_round rnd,
                       float* bhat_out, int32_t* bk_out, const WsPtrs& w) {
    HeadParams p;
    p.h = h; p.W1 = W1; p.b1 = b1; p.w2 = w2; p.b2 = b2;
    p.B = B; p.H = H; p.M = M; p.k = k;
    p.gamma = gamma; p.rnd = static_cast<int>(rnd);
    p.bhat = bhat_out; p.bk = bk_out; p.b2_dev = nullptr; p.u_out = nullptr;
    p.hdr = w.hdr; p.zpart = w.zpart; p.part = w.part; p.tile_ticket = w.tile_ticket;
    p.nsplit = head_nsplit(B, M, H);
    const int per = (H + p.nsplit - 1) / p.nsplit;
    p.ks = (per + 15) & ~15;
    return p;
}

svd_status run_head(const uint16_t* h, const uint16_t* W1, const float* b1, const uint16_t* w2,
                    float b2, int B, int H, int M, int k, float gamma, svd_bk_round rnd,
                    float* bhat_out, int32_t* bk_out, const WsPtrs& w, void* stream) {
    const HeadParams p = head_params(h, W1, b1, w2, b2, B, H, M, k, gamma, rnd, bhat_out, bk_out, w);
    return from_cuda(launch_length_head(p, stream));
}

svd_status run_rows(const uint16_t* D, const uint16_t* T, const int32_t* draft, const int32_t* bk,
                    int B, int k, int kt, int V, int flags, float temperature, uint64_t seed,
                    uint64_t step, float lambda, float clip_c, float grad_scale, int dl_fp32,
                    void* dlogits, float* loss_rows, float* loss_total, int32_t* accept_len,
                    int32_t* emitted, int32_t* n_emitted, svd_row_info* row_info, const WsPtrs& w,
                    void* stream, int bk_const = 0, float* label_proxy = nullptr,
                    float* label_full = nullptr, const HeadParams* head = nullptr) {
    RowParams p;
    std::memset(&p, 0, sizeof p);
    p.D = D; p.T = T; p.draft = draft; p.bk = bk;
    p.B = B; p.k = k; p.kt = kt; p.V = V;
    p.flags = flags;
    const bool distill = (flags & kFlagDistill) != 0;
    p.aligned = (V % 8 == 0) && aligned16(D) && aligned16(T) && (!distill || aligned16(dlogits)) ? 1 : 0;
    p.tau = temperature;
    p.inv_tau = 1.0f / temperature;
    p.k2 = 1.4426950408889634f / temperature;
    p.seed = seed; p.step = step;
    p.lambda = lambda; p.clip_c = clip_c; p.grad_scale = grad_scale;
    p.dl_fp32 = dl_fp32;
    p.dlogits = dlogits; p.loss_rows = loss_rows; p.loss_total = loss_total;
    p.accept_len = accept_len; p.emitted = emitted; p.n_emitted = n_emitted;
    p.row_info = row_info;
    p.hdr = w.hdr; p.rec = w.rec; p.seq_loss = w.seq_loss;
    p.wait_limit_ns = kWaitLimitNs;
    p.bk_const = bk_const;
    p.bk_trunc = bk;
    p.label_proxy = label_proxy;
    p.label_full = label_full;
    p.head_fused = head != nullptr ? 1 : 0;
    if (head) p.head = *head;
    return from_cuda(launch_row_pass(p, stream));
}

bool bad_float(float x) { return !std::isfinite(x); }

}  // namespace

namespace svd {

// Every argument check of svd_verify_distill that needs no workspace, in one place, so that
// callers which bring their own scratch can reject a call before touching it.
svd_status check_verify_distill_args(const svd_verify_distill_args* a) {
    if (!a) return SVD_ERR_INVALID_ARG;
    svd_status s = check_shape(a->B, a->k, a->kt, a->V);
    if (s != SVD_OK) return s;
    if (a->mode != SVD_GREEDY && a->mode != SVD_STOCHASTIC) return SVD_ERR_INVALID_ARG;
    if (bad_float(a->temperature) || !(a->temperature > 0.f)) return SVD_ERR_INVALID_ARG;
    if (bad_float(a->lambda) || a->lambda < 0.f || a->lambda > 1.f) return SVD_ERR_INVALID_ARG;
    if (std::isnan(a->clip_c) || a->clip_c < 0.f || bad_float(a->grad_scale)) return SVD_ERR_INVALID_ARG;
    if (a->dlogits_fp32 != 0 && a->dlogits_fp32 != 1) return SVD_ERR_INVALID_ARG;
    if (a->full_k != 0 && a->full_k != 1) return SVD_ERR_INVALID_ARG;
    if (a->h != nullptr) {
        if (a->H < 1 || a->M < 1 || !a->W1 || !a->w2) return SVD_ERR_INVALID_ARG;
        if (a->rnd != SVD_BK_CEIL && a->rnd != SVD_BK_FLOOR) return SVD_ERR_INVALID_ARG;
        if (bad_float(a->b2) || bad_float(a->gamma) || !(a->gamma > 0.f)) return SVD_ERR_INVALID_ARG;
    } else if (!a->bk_in && a->B > 0) {
        return SVD_ERR_INVALID_ARG;
    }
    if (a->B == 0) return SVD_OK;
    if (!a->D || !a->T || !a->bk || !a->accept_len || !a->emitted || !a->n_emitted ||
        !a->loss_total || !a->dlogits)
        return SVD_ERR_INVALID_ARG;
    if (a->mode == SVD_STOCHASTIC && !a->draft_tok) return SVD_ERR_INVALID_ARG;
    return SVD_OK;
}

}  // namespace svd

extern "C" {

size_t svd_workspace_bytes(int B, int k, int kt, int M) {
    if (B < 0 || k < 1 || kt < k || M < 0) return 0;
    return ws_layout(B, k, kt, M).total;
}

svd_status svd_workspace_reset(void* ws, size_t ws_bytes, void* stream) {
    if (ws == nullptr) return SVD_ERR_INVALID_ARG;
    return from_cuda(static_cast<int>(
        cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream))));
}

svd_status svd_length_head(const uint16_t* h, const uint16_t* W1, const float* b1,
                           const uint16_t* w2, float b2, int B, int H, int M, int k,
                           float gamma, svd_bk_round rnd, float* bhat_out, int32_t* bk_out,
                           void* ws, size_t ws_bytes, void* stream) {
    if (B < 0 || H < 1 || M < 1 || k < 1 || k > kMaxK) return SVD_ERR_INVALID_ARG;
    if (rnd != SVD_BK_CEIL && rnd != SVD_BK_FLOOR) return SVD_ERR_INVALID_ARG;
    if (bad_float(b2) || bad_float(gamma) || !(gamma > 0.f)) return SVD_ERR_INVALID_ARG;
    if (B == 0) return SVD_OK;
    if (!h || !W1 || !w2 || !bk_out) return SVD_ERR_INVALID_ARG;
    svd_status s = check_ws(ws, ws_bytes, B, k, k, M);
    if (s != SVD_OK) return s;
    return run_head(h, W1, b1, w2, b2, B, H, M, k, gamma, rnd, bhat_out, bk_out,
                    carve(ws, B, k, k, M), stream);
}

svd_status svd_verify(const uint16_t* D, const uint16_t* T, const int32_t* draft_tok,
                      const int32_t* bk, int B, int k, int kt, int V, svd_mode mode,
                      float temperature, uint64_t seed, uint64_t step, int32_t* accept_len,
                      int32_t* emitted, int32_t* n_emitted, svd_row_info* row_info, void* ws,
                      size_t ws_bytes, void* stream) {
    svd_status s = check_shape(B, k, kt, V);
    if (s != SVD_OK) return s;
    if (mode != SVD_GREEDY && mode != SVD_STOCHASTIC) return SVD_ERR_INVALID_ARG;
    if (bad_float(temperature) || !(temperature > 0.f)) return SVD_ERR_INVALID_ARG;
    if (B == 0) return SVD_OK;
    if (!D || !T || !bk || !accept_len || !emitted || !n_emitted) return SVD_ERR_INVALID_ARG;
    if (mode == SVD_STOCHASTIC && !draft_tok) return SVD_ERR_INVALID_ARG;
    s = check_ws(ws, ws_bytes, B, k, kt, 0);
    if (s != SVD_OK) return s;
    const int flags = kFlagVerify | (mode == SVD_STOCHASTIC ? kFlagStochastic : 0);
    return run_rows(D, T, draft_tok, bk, B, k, kt, V, flags, temperature, seed, step, 0.f, 0.f,
                    0.f, 0, nullptr, nullptr, nullptr, accept_len, emitted, n_emitted, row_info,
                    carve(ws, B, k, kt, 0), stream);
}

svd_status svd_distill_loss_grad(const uint16_t* D, const uint16_t* T, const int32_t* bk,
                                 int B, int k, int kt, int V, float lambda, float clip_c,
                                 float temperature, float grad_scale, float* loss_rows,
                                 float* loss_total, void* dlogits, int dlogits_fp32, void* ws,
                                 size_t ws_bytes, void* stream) {
    svd_status s = check_shape(B, k, kt, V);
    if (s != SVD_OK) return s;
    if (bad_float(lambda) || lambda < 0.f || lambda > 1.f) return SVD_ERR_INVALID_ARG;
    if (std::isnan(clip_c) || clip_c < 0.f) return SVD_ERR_INVALID_ARG;
    if (bad_float(temperature) || !(temperature > 0.f) || bad_float(grad_scale))
        return SVD_ERR_INVALID_ARG;
    if (dlogits_fp32 != 0 && dlogits_fp32 != 1) return SVD_ERR_INVALID_ARG;
    if (B == 0) return SVD_OK;
    if (!D || !T || !bk || !loss_total || !dlogits) return SVD_ERR_INVALID_ARG;
    s = check_ws(ws, ws_bytes, B, k, kt, 0);
    if (s != SVD_OK) return s;
    return run_rows(D, T, nullptr, bk, B, k, kt, V, kFlagDistill, temperature, 0, 0, lambda,
                    clip_c, grad_scale, dlogits_fp32, dlogits, loss_rows, loss_total, nullptr,
                    nullptr, nullptr, nullptr, carve(ws, B, k, kt, 0), stream);
}

svd_status svd_verify_distill(const svd_verify_distill_args* a, void* ws, size_t ws_bytes,
                              void* stream) {
    svd_status s = svd::check_verify_distill_args(a);
    if (s != SVD_OK || a->B == 0) return s;
    const bool head = a->h != nullptr;
    const int M = head ? a->M : 0;
    s = check_ws(ws, ws_bytes, a->B, a->k, a->kt, M);
    if (s != SVD_OK) return s;
    const WsPtrs w = carve(ws, a->B, a->k, a->kt, M);
    const int32_t* bk = a->bk;
    // The length head runs inside the row pass (one launch less on the critical path) when its
    // operands suit the tensor-core fragments read straight from L2 and the batch keeps its
    // lists in shared memory; otherwise it runs as its own kernel first.
    const bool fuse_head = head && a->B <= kRowCompactMaxB && a->H % 16 == 0 && aligned16(a->h) &&
                           aligned16(a->W1);
    HeadParams hp;
    if (head) {
        hp = head_params(a->h, a->W1, a->b1, a->w2, a->b2, a->B, a->H, a->M, a->k, a->gamma,
                         a->rnd, a->bhat, a->bk, w);
        hp.u_out = a->head_preact;
        if (!fuse_head) {
            s = from_cuda(launch_length_head(hp, stream));
            if (s != SVD_OK) return s;
        }
    } else if (a->bk != a->bk_in) {
        if (cudaMemcpyAsync(a->bk, a->bk_in, sizeof(int32_t) * a->B, cudaMemcpyDeviceToDevice,
                            static_cast<cudaStream_t>(stream)) != cudaSuccess)
            return SVD_ERR_CUDA;
    }
    const int flags = kFlagVerify | kFlagDistill | (a->mode == SVD_STOCHASTIC ? kFlagStochastic : 0);
    return run_rows(a->D, a->T, a->draft_tok, bk, a->B, a->k, a->kt, a->V, flags, a->temperature,
                    a->seed, a->step, a->lambda, a->clip_c, a->grad_scale, a->dlogits_fp32,
                    a->dlogits, a->loss_rows, a->loss_total, a->accept_len, a->emitted,
                    a->n_emitted, a->row_info, w, stream, a->full_k ? a->k : 0, a->label_proxy,
                    a->label_full, fuse_head ? &hp : nullptr);
}

svd_status svd_length_head_update(const svd_head_update_args* a, void* ws, size_t ws_bytes,
                                  void* stream) {
    if (!a) return SVD_ERR_INVALID_ARG;
    if (a->B < 1 || a->H < 1 || a->M < 1 || a->step < 1) return SVD_ERR_INVALID_ARG;
    if (!a->h || !a->label || !a->W1m || !a->b1 || !a->w2m || !a->b2 || !a->W1 || !a->w2 ||
        !a->mW1 || !a->vW1 || !a->mb1 || !a->vb1 || !a->mw2 || !a->vw2 || !a->mb2 || !a->vb2 ||
        !a->loss || !a->bhat)
        return SVD_ERR_INVALID_ARG;
    if (bad_float(a->lr) || a->lr < 0.f || bad_float(a->weight_decay) || a->weight_decay < 0.f ||
        !(a->beta1 >= 0.f && a->beta1 < 1.f) || !(a->beta2 >= 0.f && a->beta2 < 1.f) ||
        bad_float(a->eps) || !(a->eps > 0.f))
        return SVD_ERR_INVALID_ARG;
    svd_status s = check_ws(ws, ws_bytes, a->B, 1, 1, a->M);
    if (s != SVD_OK) return s;
    const WsLayout L = ws_layout(a->B, 1, 1, a->M);
    const WsPtrs w = carve(ws, a->B, 1, 1, a->M);
    char* base = static_cast<char*>(ws);
    float* u = reinterpret_cast<float*>(base + L.u);
    float* e = reinterpret_cast<float*>(base + L.e);
    // forward on the served weights, keeping the pre-activations -- unless the caller passes
    // those of a forward already run (then bhat is that forward's, an input)
    const bool have_fwd = a->preact != nullptr;
    if (have_fwd) u = const_cast<float*>(a->preact);
    HeadParams hp;
    hp.h = a->h; hp.W1 = a->W1; hp.b1 = a->b1; hp.w2 = a->w2; hp.b2 = 0.f;
    hp.B = a->B; hp.H = a->H; hp.M = a->M; hp.k = 1;
    hp.gamma = 1.f; hp.rnd = 0;
    hp.bhat = a->bhat; hp.bk = nullptr; hp.b2_dev = a->b2; hp.u_out = u;
    hp.hdr = w.hdr; hp.zpart = w.zpart; hp.part = w.part; hp.tile_ticket = w.tile_ticket;
    hp.nsplit = head_nsplit(a->B, a->M, a->H);
    const int per = (a->H + hp.nsplit - 1) / hp.nsplit;
    hp.ks = (per + 15) & ~15;
    if (!have_fwd) {
        s = from_cuda(launch_length_head(hp, stream));
        if (s != SVD_OK) return s;
    }
    HeadUpdateParams p;
    p.h = a->h; p.label = a->label; p.bhat = a->bhat; p.u = u; p.e = e;
    p.ticket = &w.hdr->update_ticket;
    p.B = a->B; p.H = a->H; p.M = a->M;
    p.W1m = a->W1m; p.b1 = a->b1; p.w2m = a->w2m; p.b2 = a->b2; p.W1 = a->W1; p.w2 = a->w2;
    p.mW1 = a->mW1; p.vW1 = a->vW1; p.mb1 = a->mb1; p.vb1 = a->vb1;
    p.mw2 = a->mw2; p.vw2 = a->vw2; p.mb2 = a->mb2; p.vb2 = a->vb2;
    p.lr = a->lr; p.beta1 = a->beta1; p.beta2 = a->beta2; p.eps = a->eps; p.wd = a->weight_decay;
    p.step_size = static_cast<float>(a->lr / (1.0 - std::pow(static_cast<double>(a->beta1), a->step)));
    p.rsqrt_bc2 = static_cast<float>(1.0 / std::sqrt(1.0 - std::pow(static_cast<double>(a->beta2), a->step)));
    p.loss = a->loss;
    return from_cuda(launch_head_update(p, stream));
}

svd_status svd_speedup_report(const int32_t* accept_len, const int32_t* bk,
                              const int32_t* n_emitted, int B, int k, double rho, double* out,
                              void* stream) {
    if (B < 1 || k < 1 || k > kMaxK || !std::isfinite(rho) || rho < 0.0) return SVD_ERR_INVALID_ARG;
    if (!accept_len || !bk || !n_emitted || !out) return SVD_ERR_INVALID_ARG;
    return from_cuda(launch_speedup_report(accept_len, bk, n_emitted, B, k, rho, out, stream));
}

svd_status svd_get_device_error(void* ws, void* stream) {
    if (ws == nullptr) return SVD_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t code = 0;
    if (cudaMemcpyAsync(&code, ws, sizeof code, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return SVD_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return SVD_ERR_CUDA;
    if (code != 0) {
        if (cudaMemsetAsync(ws, 0, sizeof code, st) != cudaSuccess) return SVD_ERR_CUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return SVD_ERR_CUDA;
    }
    return static_cast<svd_status>(code);
}

const char* svd_status_string(svd_status s) {
    switch (s) {
        case SVD_OK: return "SVD_OK";
        case SVD_ERR_INVALID_ARG: return "SVD_ERR_INVALID_ARG";
        case SVD_ERR_ALIGNMENT: return "SVD_ERR_ALIGNMENT";
        case SVD_ERR_WORKSPACE: return "SVD_ERR_WORKSPACE";
        case SVD_ERR_CUDA: return "SVD_ERR_CUDA";
        case SVD_ERR_TIMEOUT: return "SVD_ERR_TIMEOUT";
        case SVD_ERR_UNSUPPORTED: return "SVD_ERR_UNSUPPORTED";
        case SVD_ERR_TOKEN_RANGE: return "SVD_ERR_TOKEN_RANGE";
    }
    return "SVD_ERR_UNKNOWN";
}

svd_status svd_selftest_wait_timeout(void* ws, size_t ws_bytes, uint64_t limit_ns, void* stream) {
    if (ws == nullptr || ws_bytes < sizeof(WsHeader)) return SVD_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return SVD_ERR_ALIGNMENT;
    if (limit_ns > 10000000000ull) return SVD_ERR_INVALID_ARG;  // at most 10 s
    return from_cuda(launch_wait_timeout_selftest(static_cast<WsHeader*>(ws), limit_ns, stream));
}

}  // extern "C"
