// vocab_shard.cu -- the verify-and-distill pass over logit rows split by vocabulary id across
// ranks (the C ABI of include/svd_vocab.h).
//
// What a row computes is the fused pass's (truncated verification: Pith verdict record,
// skeptic_critique.load_bearing_attack; acceptance u < min(1, p/q), residual resampling from
// max(0, p - q) and the bonus draw from p: Pith review page, Axiom & Free-Parameter Ledger;
// the lambda-mixed CE + entry-wise clipped reverse-KL loss and its gradient: Pith review page,
// "What carries the argument" and Referee report major comment 2).  Here rank r holds ids
// [v0, v0 + Vl) of every row, and the row-global quantities travel as fixed-size records:
//
//   stats    one CTA per row: a single streaming pass over the slice gives the maxima and
//            their lowest ids, sum 2^(x k2 - round(m k2)) of D and T (online rescaling when a
//            thread's maximum grows), sum e_v (D_v - T_v) (the reverse-KL moment), max(D - T),
//            and D, T at the caller's token and D at the local target argmax.      -> Rec1
//   resolve  one CTA per sequence, one warp per row: every rank combines the P records of
//            each row (identical arithmetic on every rank), takes the acceptance decisions and
//            the b_k prefix, and keeps the row state in the workspace.  Then one CTA per row
//            that needs it re-reads the slice for the clip sums (only vectors whose largest q
//            can reach the clip bound) and the 2^-48 fixed-point sample masses.      -> Rec2
//   finish   one CTA per row: the gradient slice from the combined sums, the loss rows (the
//            last CTA adds them up), and on the rank whose mass interval holds the Philox
//            target, the sample search.
//
// Per-element arithmetic (q_v, p_v, s_v, d_v, the fixed-point masses) is the fused pass's
// (svd_device.cuh), so every rank rounds an element the same way wherever it is recomputed.
#include <cuda_runtime.h>

#include <cmath>

#include "svd_vocab.h"
#include "svd_device.cuh"
#include "svd_internal.h"

namespace svd {
namespace {

constexpr int kVsThreads = 256;
constexpr int kVsWarps = kVsThreads / 32;
constexpr int kVsUnroll = 4;                 // 16-byte vectors in flight per thread and tensor
constexpr uint32_t kNoId = 0xffffffffu;
constexpr uint16_t kSentinel = 0xFF7Fu;      // lowest finite bf16: pads a ragged slice tail

// Every kernel here is launched as a programmatic dependent of whatever precedes it on the
// stream (launch_dependent below) and reads nothing before that grid has finished: the launch
// latency overlaps the preceding kernel's tail (this rank's previous pass, or the all-gather).
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}


__device__ __forceinline__ float neg_inf() { return -__int_as_float(0x7f800000); }
__device__ __forceinline__ float quiet_nan() { return __int_as_float(0x7fc00000); }

// One rank's partial statistics of one row (exchange 1).  Sums are taken relative to
// round(m k2) of the maximum they travel with.
struct alignas(16) Rec1 {
    float mD, sD, sDd, dmax;    // draft: max, sum 2^(D k2 - round(mD k2)), same times (D - T), max(D - T)
    float mT, sT;               // target: max, sum 2^(T k2 - round(mT k2))
    uint32_t argD, argT;        // global ids of the first maxima in this slice
    float Dx, Tx;               // D and T at the caller's token if this slice holds it, else 0
    float Dy;                   // D at argT (the target argmax of this slice)
    uint32_t pad;
};
// One rank's clip sums and sample masses of one row (exchange 2).
struct alignas(16) Rec2 {
    float clip_d, clip_q, n_clip, pad;   // sum of d_v, q_v and count over entries with d_v > c
    unsigned long long mass;             // sample weights (residual, or p for a bonus row)
    unsigned long long pmass;            // p alone (the fallback when the residual is empty)
};
static_assert(sizeof(Rec1) == 48 && sizeof(Rec2) == 32, "exchange records");

constexpr uint32_t kRowVerified = 1, kRowBonus = 2, kRowClip = 4, kRowSample = 8;

// Row-global state after exchange 1 (identical on every rank).
struct alignas(16) RowState {
    float lseD, lseT, L2D, L2T;
    float dl, rkl, qthr, Dy;
    float u1, ratio;
    int32_t x, y;
    int32_t acc;
    uint32_t flags;
    float pad0, pad1;
};
struct alignas(16) SeqState {
    int32_t n, a, fix_row, pad;
};

struct VsLayout {
    size_t rows, seqs, lrow, total;
};
VsLayout vs_layout(int B, int k, int kt) {
    VsLayout L;
    size_t off = sizeof(WsHeader);
    L.rows = off;
    off = align256(off + sizeof(RowState) * static_cast<size_t>(B) * kt);
    L.seqs = off;
    off = align256(off + sizeof(SeqState) * static_cast<size_t>(B));
    L.lrow = off;
    off = align256(off + sizeof(float) * static_cast<size_t>(B) * k);
    L.total = off;
    return L;
}

struct VsParams {
    const uint16_t* D;
    const uint16_t* T;
    const int32_t* draft;
    const int32_t* bk;
    int B, k, kt, V, v0, Vl, P, rank;
    int stoch, distill, dl_fp32;
    float itau, k2, lambda, cc, grad_scale;
    uint64_t seed, step;
    Rec1* send1;
    const Rec1* recv1;
    Rec2* send2;
    const Rec2* recv2;
    WsHeader* hdr;
    RowState* rows;
    SeqState* seqs;
    float* lrow;
    void* dlogits;
    float* loss_rows;
    float* loss_total;
    int32_t* accept_len;
    int32_t* emitted;
    int32_t* n_emitted;
    svd_row_info* row_info;
};

// A programmatic dependent launch of one of the kernels below (see grid_dependency_wait).
template <typename Kernel>
cudaError_t launch_dependent(Kernel kernel, unsigned grid, unsigned block, cudaStream_t st,
                             const VsParams& p) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(block, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    return cudaLaunchKernelEx(&cfg, kernel, p);
}


__device__ __forceinline__ int vs_bk(const VsParams& p, int b) {
    const int n = __ldg(p.bk + b);
    return n < 1 ? 1 : (n > p.k ? p.k : n);
}

// Vector g (ids 8g .. 8g+7 of the slice) of a row; ids past the slice read as the sentinel.
template <bool ALIGNED>
__device__ __forceinline__ uint4 load_vec(const uint16_t* row, int g, int Vl) {
    if constexpr (ALIGNED) {
        return __ldg(reinterpret_cast<const uint4*>(row) + g);
    } else {
        uint32_t w[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const int id = g * 8 + 2 * h;
            const uint32_t lo = id < Vl ? __ldg(row + id) : kSentinel;
            const uint32_t hi = id + 1 < Vl ? __ldg(row + id + 1) : kSentinel;
            w[h] = lo | (hi << 16);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
}

__device__ __forceinline__ float bf16_at(const uint16_t* row, int id) {
    return __uint_as_float(static_cast<uint32_t>(__ldg(row + id)) << 16);
}

// Block reduction helpers (kVsThreads threads): fixed order, identical on every call.
__device__ __forceinline__ float block_sum(float v, float* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_sum(v);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kVsWarps; ++w) s += red[w];
    return s;
}
__device__ __forceinline__ unsigned long long block_sum_u64(unsigned long long v,
                                                            unsigned long long* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_sum_u64(v);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    unsigned long long s = 0ull;
#pragma unroll
    for (int w = 0; w < kVsWarps; ++w) s += red[w];
    return s;
}

// ------------------------------------------------------------------------------------------
// stats: one CTA per row
// ------------------------------------------------------------------------------------------
struct Partial {         // one thread's (then one warp's) running statistics of one tensor
    float m, s, sd;      // maximum, sum relative to round(m k2), moment (draft only)
    uint32_t pos;        // slice position of the first maximum
};

__device__ __forceinline__ void absorb(Partial& a, const uint4& v, int g, float k2, bool exps,
                                       const float (*xt)[8], float* dmax) {
    const float mv = max8_bf16(v);
    if (mv > a.m) {
        if (exps) {
            const float f = rescale(a.m, mv, k2);
            a.s *= f;
            a.sd *= f;
        }
        a.m = mv;
        a.pos = static_cast<uint32_t>(g * 8 + first_pos(v, mv));
    }
    if (!exps) return;
    float x[8];
    unpack8(v, x);
    const float A = __fmul_rn(a.m, k2);
    float s = 0.f, sd = 0.f;
#pragma unroll
    for (int l = 0; l < 8; ++l) {
        const float e = fast_exp2(__fmaf_rn(x[l], k2, -A));
        s += e;
        if (xt) {
            const float d = __fsub_rn(x[l], (*xt)[l]);
            sd = fmaf(e, d, sd);
            *dmax = fmaxf(*dmax, d);
        }
    }
    a.s += s;
    a.sd += sd;
}

// Warp, then block, combination of partials; result valid in thread 0.
__device__ __forceinline__ Partial combine_block(Partial a, float k2, bool exps, Partial* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float wm = redux_max_f32(a.m);
    Partial w;
    w.m = wm;
    w.pos = redux_min_u32(a.m == wm ? a.pos : kNoId);
    w.s = w.sd = 0.f;
    if (exps) {
        const float f = rescale(a.m, wm, k2);
        w.s = warp_sum(a.s * f);
        w.sd = warp_sum(a.sd * f);
    }
    __syncthreads();
    if (lane == 0) red[warp] = w;
    __syncthreads();
    Partial r;
    r.m = neg_inf();
    r.pos = kNoId;
    r.s = r.sd = 0.f;
    if (threadIdx.x == 0) {
        for (int q = 0; q < kVsWarps; ++q) r.m = fmaxf(r.m, red[q].m);
        for (int q = 0; q < kVsWarps; ++q) {
            if (red[q].m == r.m) r.pos = min(r.pos, red[q].pos);
            if (exps) {
                const float f = rescale(red[q].m, r.m, k2);
                r.s += red[q].s * f;
                r.sd += red[q].sd * f;
            }
        }
    }
    return r;
}

template <bool ALIGNED>
__global__ void __launch_bounds__(kVsThreads) vs_stats_kernel(const VsParams p) {
    __shared__ Partial redT[kVsWarps], redD[kVsWarps];
    __shared__ float sdm[kVsWarps];
    grid_dependency_wait();
    const int row = blockIdx.x, t = threadIdx.x;
    const int b = row / p.kt, i = row % p.kt;
    const int n = vs_bk(p, b);
    const bool verified = i < n, bonus = i == n && n < p.kt;
    Rec1 rec;
    rec.mD = rec.mT = rec.dmax = neg_inf();
    rec.sD = rec.sDd = rec.sT = 0.f;
    rec.argD = rec.argT = kNoId;
    rec.Dx = rec.Tx = rec.Dy = 0.f;
    rec.pad = 0u;
    if (!verified && !bonus) {
        if (t == 0) p.send1[row] = rec;
        return;
    }
    const bool exps = (p.distill && verified) || p.stoch;
    const uint16_t* Trow = p.T + (static_cast<size_t>(b) * p.kt + i) * p.Vl;
    const uint16_t* Drow = p.D + (static_cast<size_t>(b) * p.k + i) * p.Vl;
    const int nvec = (p.Vl + 7) >> 3;
    Partial aT{neg_inf(), 0.f, 0.f, kNoId}, aD{neg_inf(), 0.f, 0.f, kNoId};
    float dmax = neg_inf();
    // The thread's vectors g = t, t + 256, ... in order, two at a time, with the next two
    // already loading while these are absorbed (two register buffers, A and B, in turn).
    constexpr int kG = kVsUnroll / 2;
    constexpr int kStep = kVsThreads * kG;
    uint4 tA[kG], dA[kG], tB[kG], dB[kG];
    auto load_group = [&](uint4 (&tv)[kG], uint4 (&dv)[kG], int g0) {
#pragma unroll
        for (int u = 0; u < kG; ++u) {
            const int g = g0 + u * kVsThreads;
            if (g < nvec) {
                tv[u] = load_vec<ALIGNED>(Trow, g, p.Vl);
                if (verified) dv[u] = load_vec<ALIGNED>(Drow, g, p.Vl);
            }
        }
    };
    auto absorb_group = [&](const uint4 (&tv)[kG], const uint4 (&dv)[kG], int g0) {
#pragma unroll
        for (int u = 0; u < kG; ++u) {
            const int g = g0 + u * kVsThreads;
            if (g >= nvec) break;
            absorb(aT, tv[u], g, p.k2, exps, nullptr, nullptr);
            if (verified) {
                float xt[8];
                unpack8(tv[u], xt);
                absorb(aD, dv[u], g, p.k2, exps, &xt, &dmax);
            }
        }
    };
    int g0 = t;
    if (g0 < nvec) load_group(tA, dA, g0);
    while (g0 < nvec) {
        if (g0 + kStep < nvec) load_group(tB, dB, g0 + kStep);
        absorb_group(tA, dA, g0);
        g0 += kStep;
        if (g0 >= nvec) break;
        if (g0 + kStep < nvec) load_group(tA, dA, g0 + kStep);
        absorb_group(tB, dB, g0);
        g0 += kStep;
    }
    const Partial cT = combine_block(aT, p.k2, exps, redT);
    Partial cD{neg_inf(), 0.f, 0.f, kNoId};
    if (verified) {
        cD = combine_block(aD, p.k2, exps, redD);
        const float wd = redux_max_f32(dmax);
        if ((t & 31) == 0) sdm[t >> 5] = wd;
        __syncthreads();
        if (t == 0) {
            for (int q = 0; q < kVsWarps; ++q) rec.dmax = fmaxf(rec.dmax, sdm[q]);
        }
    }
    if (t != 0) return;
    // a position past the slice (only if every real entry of a vector is -inf and the padding
    // won the compare) names no id
    const uint32_t Vl = static_cast<uint32_t>(p.Vl);
    rec.mT = cT.m;
    rec.sT = cT.s;
    rec.argT = cT.pos < Vl ? static_cast<uint32_t>(p.v0) + cT.pos : kNoId;
    if (verified) {
        rec.mD = cD.m;
        rec.sD = cD.s;
        rec.sDd = cD.sd;
        rec.argD = cD.pos < Vl ? static_cast<uint32_t>(p.v0) + cD.pos : kNoId;
        if (cT.pos < Vl) rec.Dy = bf16_at(Drow, static_cast<int>(cT.pos));
        if (p.draft) {
            const int x = __ldg(p.draft + static_cast<size_t>(b) * p.k + i);
            if (x >= p.v0 && x < p.v0 + p.Vl) {
                rec.Dx = bf16_at(Drow, x - p.v0);
                rec.Tx = bf16_at(Trow, x - p.v0);
            }
        }
    }
    p.send1[row] = rec;
}

// ------------------------------------------------------------------------------------------
// resolve: one CTA per sequence, one warp per row whose lanes read the ranks' records; warp 0
// then takes the b_k prefix over the rows (row 32, a bonus row only, on warp 0's lane 0)
// ------------------------------------------------------------------------------------------
// (m, s, pos, aux) of another partial merged into this one: the larger maximum wins, equal
// maxima keep the lower id, sums move onto the larger maximum's reference.
__device__ __forceinline__ void merge_max(float& m, float& s, uint32_t& pos, float& aux, float m2,
                                          float s2, uint32_t pos2, float aux2, float k2) {
    const float M = fmaxf(m, m2);
    s = s * rescale(m, M, k2) + s2 * rescale(m2, M, k2);
    if (m2 > m || (m2 == m && pos2 < pos)) {
        pos = pos2;
        aux = aux2;
    }
    m = M;
}

__device__ RowState resolve_row(const VsParams& p, int b, int i, int n, bool& bad_token) {
    const int lane = threadIdx.x & 31;
    RowState s;
    s.lseD = s.lseT = s.L2D = s.L2T = quiet_nan();
    s.dl = s.rkl = s.qthr = s.Dy = 0.f;
    s.u1 = 0.f;
    s.ratio = quiet_nan();
    s.x = s.y = -1;
    s.acc = -1;
    s.flags = 0u;
    s.pad0 = s.pad1 = 0.f;
    const bool verified = i < n, bonus = i == n && n < p.kt;
    if (!verified && !bonus) return s;
    s.flags = verified ? kRowVerified : kRowBonus;
    const size_t stride = static_cast<size_t>(p.B) * p.kt;
    const size_t ri = static_cast<size_t>(b) * p.kt + i;
    const float k2 = p.k2, itau = p.itau;
    // this lane's ranks (lane, lane + 32, ...), merged in rank order
    float mD = neg_inf(), mT = neg_inf(), dmax = neg_inf();
    float sD = 0.f, sDd = 0.f, sT = 0.f, Dx = 0.f, Tx = 0.f, Dy = 0.f, nil = 0.f;
    uint32_t aD = kNoId, aT = kNoId;
    for (int r = lane; r < p.P; r += 32) {
        const Rec1 a = p.recv1[r * stride + ri];
        merge_max(mT, sT, aT, Dy, a.mT, a.sT, a.argT, a.Dy, k2);
        if (verified) {
            const float M = fmaxf(mD, a.mD);
            sDd = sDd * rescale(mD, M, k2) + a.sDd * rescale(a.mD, M, k2);
            merge_max(mD, sD, aD, nil, a.mD, a.sD, a.argD, 0.f, k2);
            dmax = fmaxf(dmax, a.dmax);
            Dx += a.Dx;
            Tx += a.Tx;
        }
    }
    // across the warp (a fixed butterfly order, the same on every rank)
    const float MT = redux_max_f32(mT);
    const uint32_t y = redux_min_u32(mT == MT ? aT : kNoId);
    const uint32_t own = __ballot_sync(0xffffffffu, aT == y && y != kNoId);
    s.Dy = __shfl_sync(0xffffffffu, Dy, own ? __ffs(own) - 1 : 0);
    s.y = y == kNoId ? -1 : static_cast<int32_t>(y);
    const float gsT = warp_sum(sT * rescale(mT, MT, k2));
    float MD = neg_inf(), gsD = 0.f, gsDd = 0.f, gdmax = neg_inf(), gDx = 0.f, gTx = 0.f;
    uint32_t xa = kNoId;
    if (verified) {
        MD = redux_max_f32(mD);
        xa = redux_min_u32(mD == MD ? aD : kNoId);
        const float f = rescale(mD, MD, k2);
        gsD = warp_sum(sD * f);
        gsDd = warp_sum(sDd * f);
        gdmax = redux_max_f32(dmax);
        gDx = warp_sum(Dx);      // one rank holds the caller's token, the others add exact zeros
        gTx = warp_sum(Tx);
    }
    const bool exps = (p.distill && verified) || p.stoch;
    float smax = 0.f;
    if (exps) {
        s.lseT = MT * itau + logf(gsT);
        s.L2T = s.lseT * kLog2e;
        if (verified) {
            s.lseD = MD * itau + logf(gsD);
            s.L2D = s.lseD * kLog2e;
            s.dl = s.lseD - s.lseT;
            s.rkl = (gsDd / gsD) * itau - s.dl;        // sum_v q_v (log q_v - log p_v)
            smax = gdmax * itau - s.dl;                // largest log q_v - log p_v
        }
    }
    if (verified) {
        uint32_t x = xa;
        if (p.draft) {
            const int xv = __ldg(p.draft + static_cast<size_t>(b) * p.k + i);
            if (xv < 0 || xv >= p.V) {
                bad_token = true;
                x = kNoId;
            } else {
                x = static_cast<uint32_t>(xv);
            }
        }
        s.x = x == kNoId ? -1 : static_cast<int32_t>(x);
        if (p.stoch) {
            const PhiloxOut ph = philox_words(p.seed, p.step, static_cast<uint32_t>(b),
                                              static_cast<uint32_t>(i));
            const float u0 = uniform24(ph.w[0]);
            s.u1 = uniform24(ph.w[1]);
            if (x != kNoId) {
                s.ratio = fast_exp2((s.dl - (gDx - gTx) * itau) * kLog2e);
                s.acc = u0 < fminf(1.f, s.ratio) ? 1 : 0;
            } else {
                s.ratio = 0.f;
                s.acc = 0;
            }
        } else {
            s.acc = (x != kNoId && x == y) ? 1 : 0;
        }
        // clipping is possible only if max_v q_v * max_v (log q_v - log p_v) reaches c
        if (p.distill && isfinite(p.cc) && smax > 0.f) {
            s.qthr = (p.cc / smax) * 0.9999f;
            const float qmax = fast_exp2(__fsub_rn(__fmul_rn(MD, k2), s.L2D));
            if (qmax * 1.001f > s.qthr) s.flags |= kRowClip;
        }
    } else if (p.stoch) {
        const PhiloxOut ph = philox_words(p.seed, p.step, static_cast<uint32_t>(b),
                                          static_cast<uint32_t>(i));
        s.u1 = uniform24(ph.w[1]);
    }
    return s;
}

__device__ __forceinline__ svd_row_info row_info_of(const VsParams& p, const RowState& s) {
    svd_row_info r;
    const bool verified = (s.flags & kRowVerified) != 0, processed = s.flags != 0u;
    r.draft_token = verified ? s.x : -1;
    r.target_argmax = processed ? s.y : -1;
    r.accepted = verified ? s.acc : -1;
    r.sample_token = (processed && !p.stoch) ? s.y : -1;
    r.ratio = (verified && p.stoch) ? s.ratio : quiet_nan();
    r.lse_draft = verified ? s.lseD : quiet_nan();
    r.lse_target = processed ? s.lseT : quiet_nan();
    r.loss = 0.f;
    return r;
}

__global__ void __launch_bounds__(1024) vs_resolve_kernel(const VsParams p) {
    __shared__ RowState srow[33];
    __shared__ int bad;
    grid_dependency_wait();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int b = blockIdx.x;
    const int k = p.k, kt = p.kt;
    const int n = vs_bk(p, b);
    if (threadIdx.x == 0) bad = 0;
    __syncthreads();
    for (int i = warp; i < kt; i += nw) {
        bool badt = false;
        const RowState s = resolve_row(p, b, i, n, badt);
        if (lane == 0) {
            srow[i] = s;
            if (badt) bad = 1;
        }
    }
    __syncthreads();
    if (warp != 0) return;
    if (lane == 0 && bad) set_device_error(&p.hdr->status, SVD_ERR_TOKEN_RANGE);
    RowState s = srow[lane < kt ? lane : 0];
    if (lane >= kt) {
        s.flags = 0u;
        s.acc = -1;
    }
    const bool has32 = kt == 33;
    RowState s32 = srow[has32 ? 32 : 0];
    // acceptance prefix: first verified row not accepted, else n
    const uint32_t accm = __ballot_sync(0xffffffffu, lane < n && s.acc == 1);
    int a = __ffs(~accm) - 1;
    if (a > n || a < 0) a = n;
    const int fix_row = a < n ? a : (n < kt ? n : -1);
    if (p.stoch) {
        if (lane == fix_row) s.flags |= kRowSample;
        if (has32 && fix_row == 32) s32.flags |= kRowSample;
    }
    int fix_tok = -1;
    if (!p.stoch && fix_row >= 0) {
        fix_tok = __shfl_sync(0xffffffffu, s.y, fix_row & 31);
        if (fix_row == 32) fix_tok = s32.y;
    }
    const size_t rbase = static_cast<size_t>(b) * kt;
    if (lane < kt) {
        p.rows[rbase + lane] = s;
        if (p.row_info) p.row_info[rbase + lane] = row_info_of(p, s);
    }
    if (has32 && lane == 0) {
        p.rows[rbase + 32] = s32;
        if (p.row_info) p.row_info[rbase + 32] = row_info_of(p, s32);
    }
    // emitted tokens: the accepted drafts, then the correction / bonus token (greedy: the
    // target argmax of that row; stochastic: written by the rank whose slice holds the draw)
    if (lane < k + 1) {
        int v = -1;
        if (lane < a) v = s.x;
        else if (lane == a && fix_row >= 0) v = fix_tok;
        p.emitted[static_cast<size_t>(b) * (k + 1) + lane] = v;
    }
    if (k == 32 && lane == 0)
        p.emitted[static_cast<size_t>(b) * (k + 1) + 32] = (a == 32 && fix_row >= 0) ? fix_tok : -1;
    if (lane == 0) {
        p.accept_len[b] = a;
        p.n_emitted[b] = a + (fix_row >= 0 ? 1 : 0);
        SeqState q;
        q.n = n;
        q.a = a;
        q.fix_row = fix_row;
        q.pad = 0;
        p.seqs[b] = q;
    }
}

// ------------------------------------------------------------------------------------------
// masses: one CTA per row that needs clip sums or sample masses (exchange 2)
// ------------------------------------------------------------------------------------------
template <bool ALIGNED>
__global__ void __launch_bounds__(kVsThreads) vs_masses_kernel(const VsParams p) {
    __shared__ float redf[kVsWarps];
    __shared__ unsigned long long redu[kVsWarps];
    grid_dependency_wait();
    const int row = gridDim.x - 1 - blockIdx.x, t = threadIdx.x;   // reverse order, as finish
    const int b = row / p.kt, i = row % p.kt;
    const RowState s = p.rows[row];
    bool clip = (s.flags & kRowClip) != 0;
    const bool samp = (s.flags & kRowSample) != 0;
    const bool verified = (s.flags & kRowVerified) != 0;
    if (clip) {
        // the vector test below, applied to this slice's maximum of D (from this rank's own
        // record): if it fails, no vector of the slice can hold a clipped entry
        const float mDown = p.recv1[static_cast<size_t>(p.rank) * p.B * p.kt + row].mD;
        clip = fast_exp2(__fsub_rn(__fmul_rn(mDown, p.k2), s.L2D)) > s.qthr;
    }
    if (!clip && !samp) {
        if (t == 0) p.send2[row] = Rec2{0.f, 0.f, 0.f, 0.f, 0ull, 0ull};
        return;
    }
    const uint16_t* Trow = p.T + (static_cast<size_t>(b) * p.kt + i) * p.Vl;
    const uint16_t* Drow = p.D + (static_cast<size_t>(b) * p.k + i) * p.Vl;
    const int nvec = (p.Vl + 7) >> 3;
    const float k2 = p.k2, itau = p.itau, cc = p.cc;
    float cd = 0.f, cq = 0.f, nc = 0.f;
    unsigned long long m = 0ull, pm = 0ull;
    for (int g0 = t; g0 < nvec; g0 += kVsThreads * kVsUnroll) {
        // a clip-only row needs T only where a vector of D passes the clip bound
        uint4 tv[kVsUnroll], dv[kVsUnroll];
#pragma unroll
        for (int u = 0; u < kVsUnroll; ++u) {
            const int g = g0 + u * kVsThreads;
            if (g < nvec) {
                if (samp) tv[u] = load_vec<ALIGNED>(Trow, g, p.Vl);
                if (verified) dv[u] = load_vec<ALIGNED>(Drow, g, p.Vl);
            }
        }
#pragma unroll
        for (int u = 0; u < kVsUnroll; ++u) {
            const int g = g0 + u * kVsThreads;
            if (g >= nvec) break;
            float xt[8], xd[8];
            if (samp) unpack8(tv[u], xt);
            if (verified) unpack8(dv[u], xd);
            if (clip) {
                // d_v = q_v s_v <= q_v s_max: only a vector whose largest q passes c / s_max
                // can hold clipped entries; those are tested exactly
                const float qv = fast_exp2(__fsub_rn(__fmul_rn(max8_bf16(dv[u]), k2), s.L2D));
                if (qv > s.qthr) {
                    if (!samp) unpack8(load_vec<ALIGNED>(Trow, g, p.Vl), xt);
#pragma unroll
                    for (int l = 0; l < 8; ++l) {
                        const float q = elem_q(xd[l], k2, s.L2D);
                        const float d = elem_d(q, elem_s(xd[l], xt[l], itau, s.dl));
                        if (d > cc) { cd += d; cq += q; nc += 1.f; }
                    }
                }
            }
            if (samp) {
#pragma unroll
                for (int l = 0; l < 8; ++l) {
                    const float pv = elem_p(xt[l], k2, s.L2T);
                    pm += to_fixed(pv);
                    if (verified) m += to_fixed(fmaxf(__fsub_rn(pv, elem_q(xd[l], k2, s.L2D)), 0.f));
                }
            }
        }
    }
    Rec2 r{0.f, 0.f, 0.f, 0.f, 0ull, 0ull};
    if (clip) {
        r.clip_d = block_sum(cd, redf);
        r.clip_q = block_sum(cq, redf);
        r.n_clip = block_sum(nc, redf);
    }
    if (samp) {
        r.pmass = block_sum_u64(pm, redu);
        r.mass = verified ? block_sum_u64(m, redu) : r.pmass;
    }
    if (t == 0) p.send2[row] = r;
}

// ------------------------------------------------------------------------------------------
// finish: one CTA per row -- gradient slice, loss row, sample search on the owning rank
// ------------------------------------------------------------------------------------------
template <bool ALIGNED, bool FP32>
__device__ __forceinline__ void store_grad(const VsParams& p, size_t drow, int g, const float (&gl)[8]) {
    if (ALIGNED) {
        if (FP32) {
            float4* o = reinterpret_cast<float4*>(static_cast<float*>(p.dlogits) + drow * p.Vl) + 2 * g;
            __stcs(o, make_float4(gl[0], gl[1], gl[2], gl[3]));
            __stcs(o + 1, make_float4(gl[4], gl[5], gl[6], gl[7]));
        } else {
            uint4 pk;
            pk.x = pack_bf16x2(gl[0], gl[1]);
            pk.y = pack_bf16x2(gl[2], gl[3]);
            pk.z = pack_bf16x2(gl[4], gl[5]);
            pk.w = pack_bf16x2(gl[6], gl[7]);
            __stcs(reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.dlogits) + drow * p.Vl) + g, pk);
        }
    } else {
#pragma unroll
        for (int l = 0; l < 8; ++l) {
            const int id = g * 8 + l;
            if (id >= p.Vl) break;
            if (FP32) static_cast<float*>(p.dlogits)[drow * p.Vl + id] = gl[l];
            else static_cast<uint16_t*>(p.dlogits)[drow * p.Vl + id] =
                static_cast<uint16_t>(pack_bf16x2(gl[l], 0.f) & 0xffffu);
        }
    }
}

// Rows run in the reverse of the stats pass's order, so the rows it read last (the ones most
// likely still in L2) are read again first.
template <bool ALIGNED, bool FP32>
__global__ void __launch_bounds__(kVsThreads, 3) vs_finish_kernel(const VsParams p) {
    __shared__ unsigned long long scan[kVsWarps];
    __shared__ float part[kVsThreads];
    grid_dependency_wait();
    __shared__ int found, last;
    const int row = gridDim.x - 1 - blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int b = row / p.kt, i = row % p.kt;
    const RowState s = p.rows[row];
    const bool verified = (s.flags & kRowVerified) != 0;
    const size_t stride = static_cast<size_t>(p.B) * p.kt;
    const uint16_t* Trow = p.T + (static_cast<size_t>(b) * p.kt + i) * p.Vl;
    const uint16_t* Drow = p.D + (static_cast<size_t>(b) * p.k + i) * p.Vl;
    const int nvec = (p.Vl + 7) >> 3;
    const float k2 = p.k2, itau = p.itau, cc = p.cc;

    if (p.distill && i < p.k) {
        const size_t drow = static_cast<size_t>(b) * p.k + i;
        if (verified) {
            float gcd = 0.f, gcq = 0.f, gnc = 0.f;
            const bool clip = (s.flags & kRowClip) != 0;
            if (clip) {
                for (int r = 0; r < p.P; ++r) {
                    const Rec2& a = p.recv2[r * stride + row];
                    gcd += a.clip_d;
                    gcq += a.clip_q;
                    gnc += a.n_clip;
                }
            }
            // S = sum over unclipped entries of q (s + 1) = (rkl - clip_d) + (1 - clip_q)
            const float S = (s.rkl - gcd) + (1.f - gcq);
            const float kc = isfinite(cc) ? (s.rkl - gcd) + cc * gnc : s.rkl;
            const float lam = p.lambda, pre = p.grad_scale * itau;
            const float P = pre * (lam + (1.f - lam) * (1.f - S - s.dl));
            const float Q = pre * (1.f - lam) * itau;
            const float Pc = pre * (lam - (1.f - lam) * S);
            const float hardc = pre * lam;
            if (t == 0) {
                const float ce = s.lseD - s.Dy * itau;   // -log q_y
                const float L = lam * ce + (1.f - lam) * kc;
                p.lrow[drow] = L;
                if (p.loss_rows) p.loss_rows[drow] = L;
                if (p.row_info) p.row_info[row].loss = L;
            }
            const int yl = s.y - p.v0;    // the target argmax, if this slice holds it
            // the thread's vectors two at a time, the next two loading while these are written
            // (register buffers A and B in turn)
            constexpr int kG = kVsUnroll / 2;
            constexpr int kStep = kVsThreads * kG;
            uint4 tA[kG], dA[kG], tB[kG], dB[kG];
            auto load_group = [&](uint4 (&tv)[kG], uint4 (&dv)[kG], int g0) {
#pragma unroll
                for (int u = 0; u < kG; ++u) {
                    const int g = g0 + u * kVsThreads;
                    if (g < nvec) {
                        tv[u] = load_vec<ALIGNED>(Trow, g, p.Vl);
                        dv[u] = load_vec<ALIGNED>(Drow, g, p.Vl);
                    }
                }
            };
            auto grad_group = [&](const uint4 (&tv)[kG], const uint4 (&dv)[kG], int g0) {
#pragma unroll
                for (int u = 0; u < kG; ++u) {
                    const int g = g0 + u * kVsThreads;
                    if (g >= nvec) break;
                    float xt[8], xd[8], gl[8];
                    unpack8(tv[u], xt);
                    unpack8(dv[u], xd);
#pragma unroll
                    for (int l = 0; l < 8; ++l) {
                        const float q = fast_exp2(__fmaf_rn(xd[l], k2, -s.L2D));
                        gl[l] = q * __fmaf_rn(Q, __fsub_rn(xd[l], xt[l]), P);
                    }
                    if (clip) {
                        const float qv = fast_exp2(__fsub_rn(__fmul_rn(max8_bf16(dv[u]), k2), s.L2D));
                        if (qv > s.qthr) {
#pragma unroll
                            for (int l = 0; l < 8; ++l) {
                                const float q = elem_q(xd[l], k2, s.L2D);
                                const float d = elem_d(q, elem_s(xd[l], xt[l], itau, s.dl));
                                if (d > cc) gl[l] = q * Pc;
                            }
                        }
                    }
                    if (yl >= g * 8 && yl < g * 8 + 8) {
#pragma unroll
                        for (int l = 0; l < 8; ++l)
                            if (g * 8 + l == yl) gl[l] -= hardc;
                    }
                    store_grad<ALIGNED, FP32>(p, drow, g, gl);
                }
            };
            int g0 = t;
            if (g0 < nvec) load_group(tA, dA, g0);
            while (g0 < nvec) {
                if (g0 + kStep < nvec) load_group(tB, dB, g0 + kStep);
                grad_group(tA, dA, g0);
                g0 += kStep;
                if (g0 >= nvec) break;
                if (g0 + kStep < nvec) load_group(tA, dA, g0 + kStep);
                grad_group(tB, dB, g0);
                g0 += kStep;
            }
        } else {
            // rows past b_k (and the bonus row's draft slot): zero gradient, zero loss
            if (t == 0) {
                p.lrow[drow] = 0.f;
                if (p.loss_rows) p.loss_rows[drow] = 0.f;
            }
            const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int g = t; g < nvec; g += kVsThreads) store_grad<ALIGNED, FP32>(p, drow, g, z);
        }
    }

    if (p.distill) {
        // the last CTA to finish adds the loss rows: per sequence in row order, sequences in a
        // fixed order (thread t takes sequences t, t + 256, ...; the threads in order)
        __syncthreads();
        if (t == 0) {
            __threadfence();
            last = atomicAdd(&p.hdr->loss_ticket, 1u) == gridDim.x - 1 ? 1 : 0;
        }
        __syncthreads();
        if (last) {
            __threadfence();
            float acc = 0.f;
            for (int bb = t; bb < p.B; bb += kVsThreads) {
                const int nb = p.seqs[bb].n;
                float ls = 0.f;
                for (int q = 0; q < nb; ++q) ls += __ldcg(p.lrow + static_cast<size_t>(bb) * p.k + q);
                acc += ls;
            }
            part[t] = acc;
            __syncthreads();
            if (t == 0) {
                float tot = 0.f;
                for (int j = 0; j < kVsThreads; ++j) tot += part[j];
                *p.loss_total = tot;
                p.hdr->loss_ticket = 0u;     // ready for the next call
            }
        }
    }

    if (!(s.flags & kRowSample)) return;
    // the correction / bonus draw: the rank whose mass interval holds the target searches
    unsigned long long R = 0ull, before = 0ull, mine = 0ull;
    for (int r = 0; r < p.P; ++r) R += p.recv2[r * stride + row].mass;
    const bool use_p = R == 0ull && verified;   // empty residual: sample from p itself
    if (use_p) R = 0ull;
    for (int r = 0; r < p.P; ++r) {
        const Rec2& a = p.recv2[r * stride + row];
        const unsigned long long mr = use_p ? a.pmass : a.mass;
        if (use_p) R += mr;
        if (r < p.rank) before += mr;
        if (r == p.rank) mine = mr;
    }
    if (R == 0ull) return;
    const unsigned long long tgt = scale_mass(R, static_cast<uint32_t>(s.u1 * 16777216.0f));
    if (mine == 0ull || tgt < before || tgt - before >= mine) return;
    const unsigned long long rel = tgt - before;
    if (t == 0) found = -1;
    unsigned long long run = 0ull;     // mass of the vectors before this round, id order
    const bool residual = verified && !use_p;
    for (int g0 = 0; g0 < nvec; g0 += kVsThreads) {
        const int g = g0 + t;
        float xt[8], xd[8];
        unsigned long long vm = 0ull;
        if (g < nvec) {
            unpack8(load_vec<ALIGNED>(Trow, g, p.Vl), xt);
            if (residual) unpack8(load_vec<ALIGNED>(Drow, g, p.Vl), xd);
#pragma unroll
            for (int l = 0; l < 8; ++l) {
                const float pv = elem_p(xt[l], k2, s.L2T);
                vm += residual ? to_fixed(fmaxf(__fsub_rn(pv, elem_q(xd[l], k2, s.L2D)), 0.f))
                               : to_fixed(pv);
            }
        }
        unsigned long long incl = vm;
        warp_inclusive_scan_u64(incl);
        __syncthreads();
        if (lane == 31) scan[warp] = incl;
        __syncthreads();
        unsigned long long wbefore = 0ull, total = 0ull;
#pragma unroll
        for (int w = 0; w < kVsWarps; ++w) {
            if (w < warp) wbefore += scan[w];
            total += scan[w];
        }
        const unsigned long long lo = run + wbefore + incl - vm;
        if (vm > 0ull && lo <= rel && rel - lo < vm) {
            // the target lies in this vector: walk its 8 masses in id order
            const unsigned long long r8 = rel - lo;
            unsigned long long cum = 0ull;
            int pick = -1;
#pragma unroll
            for (int l = 0; l < 8; ++l) {
                const float pv = elem_p(xt[l], k2, s.L2T);
                cum += residual ? to_fixed(fmaxf(__fsub_rn(pv, elem_q(xd[l], k2, s.L2D)), 0.f))
                                : to_fixed(pv);
                if (pick < 0 && cum > r8) pick = l;
            }
            if (pick < 0) pick = 7;
            found = p.v0 + g * 8 + pick;
        }
        run += total;
        if (run > rel) break;   // uniform: every thread holds the same run
    }
    __syncthreads();
    if (t == 0 && found >= 0) {
        const SeqState q = p.seqs[b];
        p.emitted[static_cast<size_t>(b) * (p.k + 1) + q.a] = found;
        if (p.row_info) p.row_info[row].sample_token = found;
    }
}

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------
bool bad_float(float v) { return std::isnan(v) || std::isinf(v); }

svd_status check_args(const svd_vs_args* a) {
    if (!a) return SVD_ERR_INVALID_ARG;
    if (a->B < 0 || a->k < 1 || a->k > 32 || (a->kt != a->k && a->kt != a->k + 1))
        return SVD_ERR_INVALID_ARG;
    if (a->V < 1 || a->Vl < 1 || a->v0 < 0 || static_cast<long long>(a->v0) + a->Vl > a->V)
        return SVD_ERR_INVALID_ARG;
    if (a->P < 1 || a->P > 64 || a->rank < 0 || a->rank >= a->P) return SVD_ERR_INVALID_ARG;
    if (a->mode != SVD_GREEDY && a->mode != SVD_STOCHASTIC) return SVD_ERR_INVALID_ARG;
    if (bad_float(a->temperature) || !(a->temperature > 0.f)) return SVD_ERR_INVALID_ARG;
    if (a->distill != 0 && a->distill != 1) return SVD_ERR_INVALID_ARG;
    if (a->distill) {
        if (bad_float(a->lambda) || a->lambda < 0.f || a->lambda > 1.f) return SVD_ERR_INVALID_ARG;
        if (std::isnan(a->clip_c) || a->clip_c < 0.f || bad_float(a->grad_scale))
            return SVD_ERR_INVALID_ARG;
        if (a->dlogits_fp32 != 0 && a->dlogits_fp32 != 1) return SVD_ERR_INVALID_ARG;
    }
    if (a->B == 0) return SVD_OK;
    if (!a->D || !a->T || !a->bk || !a->accept_len || !a->emitted || !a->n_emitted)
        return SVD_ERR_INVALID_ARG;
    if (a->mode == SVD_STOCHASTIC && !a->draft_tok) return SVD_ERR_INVALID_ARG;
    if (a->distill && (!a->dlogits || !a->loss_total)) return SVD_ERR_INVALID_ARG;
    return SVD_OK;
}

svd_status check_vs_ws(const void* ws, size_t ws_bytes, const svd_vs_args* a) {
    if (!ws) return SVD_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return SVD_ERR_ALIGNMENT;
    if (ws_bytes < vs_layout(a->B, a->k, a->kt).total) return SVD_ERR_WORKSPACE;
    return SVD_OK;
}

bool aligned16(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }

bool slice_aligned(const svd_vs_args* a, bool with_grad) {
    return a->Vl % 8 == 0 && aligned16(a->D) && aligned16(a->T) &&
           (!with_grad || aligned16(a->dlogits));
}

VsParams make_params(const svd_vs_args* a, void* ws) {
    VsParams p;
    p.D = a->D;
    p.T = a->T;
    p.draft = a->draft_tok;
    p.bk = a->bk;
    p.B = a->B;
    p.k = a->k;
    p.kt = a->kt;
    p.V = a->V;
    p.v0 = a->v0;
    p.Vl = a->Vl;
    p.P = a->P;
    p.rank = a->rank;
    p.stoch = a->mode == SVD_STOCHASTIC ? 1 : 0;
    p.distill = a->distill;
    p.dl_fp32 = a->dlogits_fp32;
    p.itau = 1.f / a->temperature;
    p.k2 = kLog2e / a->temperature;
    p.lambda = a->lambda;
    p.cc = a->clip_c;
    p.grad_scale = a->grad_scale;
    p.seed = a->seed;
    p.step = a->step;
    p.send1 = nullptr;
    p.recv1 = nullptr;
    p.send2 = nullptr;
    p.recv2 = nullptr;
    const VsLayout L = vs_layout(a->B, a->k, a->kt);
    char* base = static_cast<char*>(ws);
    p.hdr = reinterpret_cast<WsHeader*>(base);
    p.rows = reinterpret_cast<RowState*>(base + L.rows);
    p.seqs = reinterpret_cast<SeqState*>(base + L.seqs);
    p.lrow = reinterpret_cast<float*>(base + L.lrow);
    p.dlogits = a->dlogits;
    p.loss_rows = a->loss_rows;
    p.loss_total = a->loss_total;
    p.accept_len = a->accept_len;
    p.emitted = a->emitted;
    p.n_emitted = a->n_emitted;
    p.row_info = a->row_info;
    return p;
}

svd_status launched() {
    return cudaGetLastError() == cudaSuccess ? SVD_OK : SVD_ERR_CUDA;
}

}  // namespace
}  // namespace svd

using namespace svd;

extern "C" {

size_t svd_vs_exchange_bytes(int B, int kt, int which) {
    if (B < 0 || kt < 1 || kt > 33) return 0;
    const size_t rows = static_cast<size_t>(B) * kt;
    if (which == 1) return rows * sizeof(Rec1);
    if (which == 2) return rows * sizeof(Rec2);
    return 0;
}

size_t svd_vs_workspace_bytes(int B, int k, int kt) {
    if (B < 0 || k < 1 || k > 32 || (kt != k && kt != k + 1)) return 0;
    return vs_layout(B, k, kt).total;
}

svd_status svd_vs_stats(const svd_vs_args* a, void* send1, void* ws, size_t ws_bytes,
                        void* stream) {
    svd_status s = check_args(a);
    if (s != SVD_OK || a->B == 0) return s;
    if (!send1) return SVD_ERR_INVALID_ARG;
    s = check_vs_ws(ws, ws_bytes, a);
    if (s != SVD_OK) return s;
    VsParams p = make_params(a, ws);
    p.send1 = static_cast<Rec1*>(send1);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const unsigned grid = static_cast<unsigned>(a->B) * a->kt;
    const cudaError_t err = slice_aligned(a, false) ? launch_dependent(vs_stats_kernel<true>, grid, kVsThreads, st, p)
                                                    : launch_dependent(vs_stats_kernel<false>, grid, kVsThreads, st, p);
    if (err != cudaSuccess) return SVD_ERR_CUDA;
    return launched();
}

svd_status svd_vs_resolve(const svd_vs_args* a, const void* recv1, void* send2, void* ws,
                          size_t ws_bytes, void* stream) {
    svd_status s = check_args(a);
    if (s != SVD_OK || a->B == 0) return s;
    if (!recv1 || !send2) return SVD_ERR_INVALID_ARG;
    s = check_vs_ws(ws, ws_bytes, a);
    if (s != SVD_OK) return s;
    VsParams p = make_params(a, ws);
    p.recv1 = static_cast<const Rec1*>(recv1);
    p.send2 = static_cast<Rec2*>(send2);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (launch_dependent(vs_resolve_kernel, static_cast<unsigned>(a->B), 32u * (a->kt < 32 ? a->kt : 32), st, p) !=
        cudaSuccess)
        return SVD_ERR_CUDA;
    s = launched();
    if (s != SVD_OK) return s;
    const unsigned grid = static_cast<unsigned>(a->B) * a->kt;
    const cudaError_t err = slice_aligned(a, false) ? launch_dependent(vs_masses_kernel<true>, grid, kVsThreads, st, p)
                                                    : launch_dependent(vs_masses_kernel<false>, grid, kVsThreads, st, p);
    if (err != cudaSuccess) return SVD_ERR_CUDA;
    return launched();
}

svd_status svd_vs_finish(const svd_vs_args* a, const void* recv2, void* ws, size_t ws_bytes,
                         void* stream) {
    svd_status s = check_args(a);
    if (s != SVD_OK || a->B == 0) return s;
    if (!recv2) return SVD_ERR_INVALID_ARG;
    s = check_vs_ws(ws, ws_bytes, a);
    if (s != SVD_OK) return s;
    VsParams p = make_params(a, ws);
    p.recv2 = static_cast<const Rec2*>(recv2);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const unsigned grid = static_cast<unsigned>(a->B) * a->kt;
    const bool al = slice_aligned(a, a->distill != 0);
    const bool f32 = a->distill && a->dlogits_fp32;
    const cudaError_t err = (al && f32) ? launch_dependent(vs_finish_kernel<true, true>, grid, kVsThreads, st, p)
                            : al        ? launch_dependent(vs_finish_kernel<true, false>, grid, kVsThreads, st, p)
                            : f32       ? launch_dependent(vs_finish_kernel<false, true>, grid, kVsThreads, st, p)
                                        : launch_dependent(vs_finish_kernel<false, false>, grid, kVsThreads, st, p);
    if (err != cudaSuccess) return SVD_ERR_CUDA;
    return launched();
}

}  // extern "C"
