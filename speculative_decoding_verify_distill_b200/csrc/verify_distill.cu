// verify_distill.cu -- the fused row pass: truncated verification (greedy / stochastic) and the
// clipped reverse-KL + CE distillation loss with its gradient, one HBM read per logit row.
//
// What it computes (AdaFlash, Pith review page "What carries the argument", Axiom & Free-
// Parameter Ledger, Referee Report major comment 2; Pith verdict record load_bearing_attack):
// for every sequence b the first b_k draft rows are verified against the target rows, the
// acceptance length a_b and the emitted tokens follow the standard speculative-decoding rule,
// and every verified row i < b_k also yields the OPD loss L_i and dL/dD_i; rows i >= b_k get a
// zero gradient row.
//
// Design (B200, sm_100a):
//   * Persistent grid of thread-block clusters; one cluster owns one logit row at a time, each
//     CTA of the cluster a contiguous slice ("chunk") of the vocabulary.  Work items are the
//     verified rows (position-major), the bonus rows, then the rows that are only zero-filled;
//     cluster c takes items c, c + #clusters, ...
//   * A slice of D and T is staged into shared memory by 1-D bulk copies (cp.async.bulk, no
//     multicast) completing on mbarriers; the next item's copies are issued as soon as the
//     current slice has been consumed, so HBM reads stream while the cluster finishes the row.
//   * Pass A (from the staging buffer): per-thread online max / sum of exp for D and T, exp
//     values e_v of D kept in registers, delta_v = D_v - T_v kept in shared memory (fp32).
//     Cluster reduction #1 over distributed shared memory gives lse(D/tau), lse(T/tau).
//   * Pass B (registers + shared memory): sum of d_v = q_v s_v, the rare clipped entries, and in
//     stochastic mode the residual masses as 2^-48 fixed-point integers (exact, order-free
//     prefix sums).  Argmax (lowest id) is resolved lazily by the threads that hold the row max.
//     Cluster reduction #2.
//   * Pass C: dL/dD = q (P + Q delta) (+ clipped and hard-label corrections), 16-byte stores.
//   * The CTA that completes the last row of a sequence (atomic ticket; nothing ever waits on
//     another CTA) runs the warp-ballot acceptance scan and writes the sequence's outputs.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>

#include "svd_device.cuh"

namespace svd {

namespace {

constexpr uint32_t kNone = 0xffffffffu;
#define kNegInf (-__int_as_float(0x7f800000))  // -inf

enum ItemKind : int { kItemNone = 0, kItemRow = 1, kItemBonus = 2, kItemZero = 3 };

// Per-CTA exchange slot, read and written across the cluster through DSMEM.
struct alignas(16) Slot {
    float mD, sD, mT, sT;                   // reduction #1: max / sum-exp (relative to max)
    float sum_d, clip_d, clip_q, n_clip;    // reduction #2: reverse-KL partials
    unsigned long long mass;                // reduction #2: this CTA's sample mass (2^-48 units)
    unsigned long long mass2;               // fallback reduction: mass of p (2^-48 units)
    uint32_t argD, argT;                    // rank 0: lowest index holding the row max
    uint32_t tok;                           // rank 0: sampled token
    float ce;                               // rank 0: -log q_y from the owner of y
};

// Values every thread of the CTA needs for the current row.
struct RowG {
    float MD, MT;        // row maxima of D and T (bf16 values)
    float lseD, lseT;    // log sum exp(x / tau)
    float L2D, L2T;      // lse * log2(e)
    float dl;            // lseD - lseT
    float P, Q, Pc, hardc;  // gradient coefficients
    float ratio, u0, u1;
    int acc;             // stochastic decision (or greedy decision once known)
    int do_sample;       // stochastic: this row draws a token
    int attempt_p;       // residual mass was zero: sample from p instead
    uint32_t x, y;
    float Dx, Tx;
    unsigned long long R, off;  // total mass of the row, mass before this CTA's slice
    unsigned long long tgt;     // sample point in [0, R)
    float sum_d, clip_d, n_clip;
};

template <int NW>
struct Ctl {
    Slot slot;
    RowG g;
    float wred[NW][4];
    unsigned long long wmass[NW];
    int hist[34];
    int cumV[34], cumZ[34];
    int totV, totB, totZ;
    int kind, b, i;          // current item
    int nkind, nb, ni;       // next item
    int fin;                 // this CTA completed a sequence
};

__device__ __forceinline__ int get_bk(const RowParams& p, int b) {
    int n = __ldg(p.bk + b);
    if (n < 1 || n > p.k) {
        set_device_error(&p.hdr->status, SVD_ERR_INVALID_ARG);
        n = n < 1 ? 1 : p.k;
    }
    return n;
}

__device__ __forceinline__ bool zero_row_pred(const RowParams& p, int n, int i, bool verify) {
    // dlogits rows that only need zeros: i >= b_k, except the bonus row b_k (zeroed by its item)
    return i < p.k && (verify ? (n < i) : (n <= i));
}

// Lane that holds the r-th (0-based) sequence satisfying pred, found by warp ballots.
template <typename Pred>
__device__ int warp_select_rth(int B, int r, Pred pred) {
    const int lane = threadIdx.x & 31;
    for (int c = 0; c < B; c += 32) {
        const int b = c + lane;
        const bool q = b < B && pred(b);
        const uint32_t m = __ballot_sync(0xffffffffu, q);
        const int cnt = __popc(m);
        if (r < cnt) {
            const bool mine = q && __popc(m & ((1u << lane) - 1u)) == r;
            const uint32_t who = __ballot_sync(0xffffffffu, mine);
            return c + __ffs(who) - 1;
        }
        r -= cnt;
    }
    return -1;
}

// Decodes work item w into (kind, b, i); executed by a full warp.
template <int NW>
__device__ void decode_item(const RowParams& p, Ctl<NW>& c, int w, bool verify, int* kind, int* b,
                            int* i) {
    *kind = kItemNone; *b = -1; *i = -1;
    if (w < c.totV) {
        int pos = 0;
        while (c.cumV[pos + 1] <= w) ++pos;
        const int r = w - c.cumV[pos];
        *b = warp_select_rth(p.B, r, [&](int s) { return get_bk(p, s) > pos; });
        *i = pos;
        *kind = kItemRow;
    } else if (w < c.totV + c.totB) {
        const int r = w - c.totV;
        *b = warp_select_rth(p.B, r, [&](int s) { return get_bk(p, s) < p.kt; });
        *i = get_bk(p, *b);
        *kind = kItemBonus;
    } else if (w < c.totV + c.totB + c.totZ) {
        const int wz = w - c.totV - c.totB;
        int pos = 0;
        while (c.cumZ[pos + 1] <= wz) ++pos;
        const int r = wz - c.cumZ[pos];
        *b = warp_select_rth(p.B, r,
                             [&](int s) { return zero_row_pred(p, get_bk(p, s), pos, verify); });
        *i = pos;
        *kind = kItemZero;
    }
}

// (max, sum) pairs of exp sums relative to their max, merged in the log2-scaled domain.
__device__ __forceinline__ void lse_merge(float& m, float& s, float m2, float s2, float k2) {
    if (m2 > m) {
        s = s * fast_exp2((m - m2) * k2) + s2;
        m = m2;
    } else if (m2 != kNegInf) {
        s += s2 * fast_exp2((m2 - m) * k2);
    }
}

// Per-element quantities with explicit rounding (no contraction), so that the values summed in
// pass B and the values recomputed later (clip decisions, sample search) are bit-identical.
__device__ __forceinline__ float elem_q(float e, float f) { return __fmul_rn(e, f); }
__device__ __forceinline__ float elem_s(float dd, float itau, float dl) { return __fmaf_rn(dd, itau, -dl); }
__device__ __forceinline__ float elem_d(float q, float s) { return __fmul_rn(q, s); }
__device__ __forceinline__ float elem_p(float q, float s) {
    return __fmul_rn(q, fast_exp2(__fmul_rn(-s, kLog2e)));
}
// Sample masses as 2^-48 fixed-point integers: exact, associative prefix sums.
__device__ __forceinline__ unsigned long long to_fixed(float r) {
    return __float2ull_rz(r * 281474976710656.0f);
}

// floor(R * u24 / 2^24) exactly, for u24 < 2^24 and R < 2^63.
__device__ __forceinline__ unsigned long long scale_mass(unsigned long long R, uint32_t u24) {
    const unsigned long long lo = R * static_cast<unsigned long long>(u24);
    const unsigned long long hi = __umul64hi(R, static_cast<unsigned long long>(u24));
    return (lo >> 24) | (hi << 40);
}

}  // namespace

template <int NT, int NV>
__host__ __device__ constexpr size_t ctl_offset() {
    return (static_cast<size_t>(NV) * NT * 16 * 2 + static_cast<size_t>(NV) * NT * 32 +
            static_cast<size_t>(NV) * 8 + 127) & ~static_cast<size_t>(127);
}

template <int NT, int NV, bool DISTILL, bool STOCH>
__global__ void __launch_bounds__(NT, 1) row_pass_kernel(const RowParams p) {
    constexpr int NW = NT / 32;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    uint4* stageD = reinterpret_cast<uint4*>(smem_raw);
    uint4* stageT = stageD + NV * NT;
    float4* dplane = reinterpret_cast<float4*>(stageT + NV * NT);
    uint64_t* full = reinterpret_cast<uint64_t*>(dplane + 2 * NV * NT);
    Ctl<NW>& c = *reinterpret_cast<Ctl<NW>*>(smem_raw + ctl_offset<NT, NV>());

    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const uint32_t rank = cluster_rank();
    const uint32_t CL = cluster_size();
    const int cid = static_cast<int>(cluster_id_x());
    const int ncl = static_cast<int>(num_clusters_x());
    const bool verify = (p.flags & kFlagVerify) != 0;
    const bool need_lse = DISTILL || STOCH;
    const int V = p.V;
    const int v0 = static_cast<int>(rank) * p.chunk;
    const int len = max(0, min(p.chunk, V - v0));
    const int nvec = (len + 7) >> 3;
    const float k2 = p.k2, itau = p.inv_tau;

    // ---------------------------------------------------------------- prologue
    if (t == 0) {
        for (int j = 0; j < NV; ++j) mbar_init(&full[j], 1);
        fence_mbar_init();
        c.slot.argD = kNone;
        c.slot.argT = kNone;
        c.slot.tok = kNone;
        c.slot.ce = 0.f;
    }
    if (t < 34) c.hist[t] = 0;
    __syncthreads();
    // histogram of b_k -> item counts
    for (int b = t; b < p.B; b += NT) atomicAdd(&c.hist[get_bk(p, b)], 1);
    __syncthreads();
    if (t == 0) {
        const int k = p.k;
        c.cumV[0] = 0;
        c.cumZ[0] = 0;
        for (int i = 0; i < k; ++i) {
            int cv = 0, cz = 0;
            for (int n = 1; n <= k; ++n) {
                if (n > i) cv += c.hist[n];
                if (DISTILL && zero_row_pred(p, n, i, verify)) cz += c.hist[n];
            }
            c.cumV[i + 1] = c.cumV[i] + cv;
            c.cumZ[i + 1] = c.cumZ[i] + cz;
        }
        for (int i = k; i < 33; ++i) {
            c.cumV[i + 1] = c.cumV[i] + 0x3fffffff;  // sentinel: never reached by a valid w
            c.cumZ[i + 1] = c.cumZ[i] + 0x3fffffff;
        }
        c.totV = c.cumV[k];
        c.totZ = c.cumZ[k];
        c.totB = verify ? (p.B - (p.kt == k ? c.hist[k] : 0)) : 0;
    }
    __syncthreads();

    uint32_t phase = 0;   // parity of the staging barriers for the next loaded item
    bool wait_dead = false;  // a bounded wait ran out: skip later waits so the kernel finishes

    auto issue_loads = [&](int kind, int b, int i) {
        // thread 0 only; one phase of every staging barrier per loaded item
        const uint16_t* Drow = p.D + (static_cast<size_t>(b) * p.k + i) * V + v0;
        const uint16_t* Trow = p.T + (static_cast<size_t>(b) * p.kt + i) * V + v0;
        for (int j = 0; j < NV; ++j) {
            const int e0 = j * NT * 8;
            const int n = max(0, min(len - e0, NT * 8));
            const uint32_t bT = static_cast<uint32_t>(n) * 2u;         // target row: always
            const uint32_t bD = (kind == kItemRow) ? bT : 0u;           // draft row: verified rows
            mbar_arrive_expect_tx(&full[j], bD + bT);
            if (bD) bulk_load(stageD + j * NT, Drow + e0, bD, &full[j]);
            if (bT) bulk_load(stageT + j * NT, Trow + e0, bT, &full[j]);
        }
    };

    int w = cid;
    if (warp == 0) {
        int kind, b, i;
        decode_item(p, c, w, verify, &kind, &b, &i);
        if (lane == 0) { c.kind = kind; c.b = b; c.i = i; }
    }
    __syncthreads();
    cluster_sync();  // barriers and slots initialised everywhere before any remote access
    if (t == 0 && p.aligned && (c.kind == kItemRow || c.kind == kItemBonus))
        issue_loads(c.kind, c.b, c.i);

    // ---------------------------------------------------------------- item loop
    while (true) {
        const int kind = c.kind, b = c.b, i = c.i;
        if (kind == kItemNone) break;
        const int wn = w + ncl;
        if (warp == 0) {
            int nk, nb, ni;
            decode_item(p, c, wn, verify, &nk, &nb, &ni);
            if (lane == 0) { c.nkind = nk; c.nb = nb; c.ni = ni; }
        }
        const size_t drow = static_cast<size_t>(b) * p.k + i;      // draft / gradient row
        const size_t trow = static_cast<size_t>(b) * p.kt + i;     // target row

        if (kind == kItemZero) {
            // ---------------------------------------------------- zero-only gradient row
            if (p.aligned) {
                const uint4 z = make_uint4(0, 0, 0, 0);
                if (p.dl_fp32) {
                    float* g = static_cast<float*>(p.dlogits) + drow * V + v0;
                    for (int e = t * 4; e < len; e += NT * 4) __stcs(reinterpret_cast<uint4*>(g + e), z);
                } else {
                    uint16_t* g = static_cast<uint16_t*>(p.dlogits) + drow * V + v0;
                    for (int e = t * 8; e < len; e += NT * 8) __stcs(reinterpret_cast<uint4*>(g + e), z);
                }
            } else {
                for (int e = t; e < len; e += NT) {
                    if (p.dl_fp32) static_cast<float*>(p.dlogits)[drow * V + v0 + e] = 0.f;
                    else static_cast<uint16_t*>(p.dlogits)[drow * V + v0 + e] = 0;
                }
            }
            __syncthreads();
            if (t == 0) { c.kind = c.nkind; c.b = c.nb; c.i = c.ni; }
            __syncthreads();
            w = wn;
            continue;
        }

        const bool isRow = (kind == kItemRow);
        const bool rowVerify = isRow && verify;
        // draft token given by the caller: fetch D_x, T_x for the acceptance ratio
        if (t == 0) {
            uint32_t x = kNone;
            float Dx = 0.f, Tx = 0.f;
            if (rowVerify && p.draft != nullptr) {
                const int xv = __ldg(p.draft + drow);
                if (xv < 0 || xv >= V) {
                    set_device_error(&p.hdr->status, SVD_ERR_TOKEN_RANGE);
                } else {
                    x = static_cast<uint32_t>(xv);
                    if (STOCH) {
                        Dx = __uint_as_float(static_cast<uint32_t>(__ldg(p.D + drow * V + x)) << 16);
                        Tx = __uint_as_float(static_cast<uint32_t>(__ldg(p.T + trow * V + x)) << 16);
                    }
                }
            }
            c.g.x = x;
            c.g.Dx = Dx;
            c.g.Tx = Tx;
        }

        // -------------------------------------------------------- pass A: stream the slice
        float e[NV][8];
        float ref[NV];
        float RD = kNegInf, sD = 0.f, RT = kNegInf, sT = 0.f;
        uint4 bestDraw = make_uint4(0, 0, 0, 0), bestTraw = make_uint4(0, 0, 0, 0);
        int bestDj = -1, bestTj = -1;
        bool timed_out = false;
#pragma unroll
        for (int j = 0; j < NV; ++j) {
            if (p.aligned && !wait_dead) {
                if (!mbar_wait_bounded(&full[j], phase, p.wait_limit_ns)) {
                    timed_out = true;
                    wait_dead = true;
                }
            }
            const int vi = j * NT + t;
            const bool valid = vi < nvec;
#pragma unroll
            for (int l = 0; l < 8; ++l) e[j][l] = 0.f;
            ref[j] = 0.f;
            if (valid) {
                uint4 rd = make_uint4(0, 0, 0, 0), rt;
                uint32_t validmask = 0xffu;
                if (p.aligned) {
                    if (isRow) rd = stageD[j * NT + t];
                    rt = stageT[j * NT + t];
                } else {
                    // plain loads; elements past the row end read as -inf
                    uint16_t dv[8], tv[8];
                    const int base = v0 + vi * 8;
#pragma unroll
                    for (int l = 0; l < 8; ++l) {
                        const bool ok = base + l < V && vi * 8 + l < len;
                        if (!ok) validmask &= ~(1u << l);
                        dv[l] = ok && isRow ? __ldg(p.D + drow * V + base + l) : (uint16_t)0xFF80u;
                        tv[l] = ok ? __ldg(p.T + trow * V + base + l) : (uint16_t)0xFF80u;
                    }
                    rd = make_uint4(dv[0] | (uint32_t(dv[1]) << 16), dv[2] | (uint32_t(dv[3]) << 16),
                                    dv[4] | (uint32_t(dv[5]) << 16), dv[6] | (uint32_t(dv[7]) << 16));
                    rt = make_uint4(tv[0] | (uint32_t(tv[1]) << 16), tv[2] | (uint32_t(tv[3]) << 16),
                                    tv[4] | (uint32_t(tv[5]) << 16), tv[6] | (uint32_t(tv[7]) << 16));
                }
                float xt[8];
                unpack8(rt, xt);
                const float mT = max8_bf16(rt);
                if (mT > RT) {
                    if (need_lse) sT *= fast_exp2((RT - mT) * k2);
                    RT = mT;
                    bestTraw = rt;
                    bestTj = j;
                }
                if (isRow) {
                    float xd[8];
                    unpack8(rd, xd);
                    const float mD = max8_bf16(rd);
                    if (mD > RD) {
                        if (need_lse) sD *= fast_exp2((RD - mD) * k2);
                        RD = mD;
                        bestDraw = rd;
                        bestDj = j;
                    }
                    if (need_lse) {
                        const float AD = RD * k2, AT = RT * k2;
                        ref[j] = RD;
#pragma unroll
                        for (int l = 0; l < 8; ++l) {
                            const float ed = fast_exp2(fmaf(xd[l], k2, -AD));
                            e[j][l] = ed;
                            sD += ed;
                            sT += fast_exp2(fmaf(xt[l], k2, -AT));
                        }
                        float dd[8];
#pragma unroll
                        for (int l = 0; l < 8; ++l)
                            dd[l] = ((validmask >> l) & 1u) ? xd[l] - xt[l] : 0.f;
                        dplane[(2 * j) * NT + t] = make_float4(dd[0], dd[1], dd[2], dd[3]);
                        dplane[(2 * j + 1) * NT + t] = make_float4(dd[4], dd[5], dd[6], dd[7]);
                    }
                } else if (need_lse) {
                    const float AT = RT * k2;
                    ref[j] = RT;
#pragma unroll
                    for (int l = 0; l < 8; ++l) {
                        const float et = fast_exp2(fmaf(xt[l], k2, -AT));
                        e[j][l] = et;
                        sT += et;
                    }
                }
            }
        }
        phase ^= 1u;
        if (timed_out) set_device_error(&p.hdr->status, SVD_ERR_TIMEOUT);

        // per-thread partials -> warp (own maxima stay per-thread for the lazy argmax)
        float wmD = RD, wsD = sD, wmT = RT, wsT = sT;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, wmD, o);
            const float s2 = __shfl_xor_sync(0xffffffffu, wsD, o);
            const float m3 = __shfl_xor_sync(0xffffffffu, wmT, o);
            const float s3 = __shfl_xor_sync(0xffffffffu, wsT, o);
            lse_merge(wmD, wsD, m2, s2, k2);
            lse_merge(wmT, wsT, m3, s3, k2);
        }
        if (lane == 0) {
            c.wred[warp][0] = wmD;
            c.wred[warp][1] = wsD;
            c.wred[warp][2] = wmT;
            c.wred[warp][3] = wsT;
        }
        __syncthreads();  // staging fully consumed; warp partials visible
        {
            const int nk = c.nkind;
            if (t == 0 && p.aligned && (nk == kItemRow || nk == kItemBonus))
                issue_loads(nk, c.nb, c.ni);
        }
        if (warp == 0) {
            float m0 = kNegInf, s0 = 0.f, m1 = kNegInf, s1 = 0.f;
            if (lane < NW) { m0 = c.wred[lane][0]; s0 = c.wred[lane][1]; m1 = c.wred[lane][2]; s1 = c.wred[lane][3]; }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float a = __shfl_xor_sync(0xffffffffu, m0, o);
                const float bb = __shfl_xor_sync(0xffffffffu, s0, o);
                const float cc = __shfl_xor_sync(0xffffffffu, m1, o);
                const float d = __shfl_xor_sync(0xffffffffu, s1, o);
                lse_merge(m0, s0, a, bb, k2);
                lse_merge(m1, s1, cc, d, k2);
            }
            if (lane == 0) { c.slot.mD = m0; c.slot.sD = s0; c.slot.mT = m1; c.slot.sT = s1; }
        }
        cluster_sync();  // #1

        // ---------------------------------------------------- row statistics (every rank)
        if (warp == 0) {
            float m0 = kNegInf, s0 = 0.f, m1 = kNegInf, s1 = 0.f;
            if (lane < static_cast<int>(CL)) {
                const uint32_t a = dsmem_map(&c.slot, lane);
                m0 = dsmem_ld_f32(a + offsetof(Slot, mD));
                s0 = dsmem_ld_f32(a + offsetof(Slot, sD));
                m1 = dsmem_ld_f32(a + offsetof(Slot, mT));
                s1 = dsmem_ld_f32(a + offsetof(Slot, sT));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float a = __shfl_xor_sync(0xffffffffu, m0, o);
                const float bb = __shfl_xor_sync(0xffffffffu, s0, o);
                const float cc = __shfl_xor_sync(0xffffffffu, m1, o);
                const float d = __shfl_xor_sync(0xffffffffu, s1, o);
                lse_merge(m0, s0, a, bb, k2);
                lse_merge(m1, s1, cc, d, k2);
            }
            if (lane == 0) {
                RowG& g = c.g;
                g.MD = m0;
                g.MT = m1;
                if (need_lse) {
                    g.lseD = isRow ? m0 * itau + logf(s0) : __int_as_float(0x7fc00000);
                    g.lseT = m1 * itau + logf(s1);
                    g.L2D = g.lseD * kLog2e;
                    g.L2T = g.lseT * kLog2e;
                    g.dl = g.lseD - g.lseT;
                } else {
                    g.lseD = g.lseT = __int_as_float(0x7fc00000);
                    g.L2D = g.L2T = g.dl = 0.f;
                }
                g.ratio = __int_as_float(0x7fc00000);
                g.acc = 0;
                g.do_sample = 0;
                g.attempt_p = 0;
                g.u0 = g.u1 = 0.f;
                if (STOCH) {
                    const PhiloxOut ph = philox_words(p.seed, p.step, static_cast<uint32_t>(b),
                                                      static_cast<uint32_t>(i));
                    g.u0 = uniform24(ph.w[0]);
                    g.u1 = uniform24(ph.w[1]);
                    if (rowVerify) {
                        if (g.x != kNone) {
                            g.ratio = fast_exp2((g.dl - (g.Dx - g.Tx) * itau) * kLog2e);
                            g.acc = g.u0 < fminf(1.f, g.ratio) ? 1 : 0;
                        } else {
                            g.ratio = 0.f;
                            g.acc = 0;
                        }
                        g.do_sample = g.acc ? 0 : 1;
                    } else if (!isRow) {
                        g.do_sample = 1;  // bonus row: sample from p
                    }
                }
            }
        }
        __syncthreads();

        // lazy argmax: only the threads that hold the row maximum inspect their best vector
        {
            const RowG& g = c.g;
            const uint32_t rank0 = 0;
            if (rowVerify && p.draft == nullptr && bestDj >= 0 && RD == g.MD) {
                float xd[8];
                unpack8(bestDraw, xd);
                int l = 0;
                while (l < 7 && xd[l] != g.MD) ++l;
                dsmem_min_u32(dsmem_map(&c.slot.argD, rank0),
                              static_cast<uint32_t>(v0 + (bestDj * NT + t) * 8 + l));
            }
            if (bestTj >= 0 && RT == g.MT) {
                float xt[8];
                unpack8(bestTraw, xt);
                int l = 0;
                while (l < 7 && xt[l] != g.MT) ++l;
                dsmem_min_u32(dsmem_map(&c.slot.argT, rank0),
                              static_cast<uint32_t>(v0 + (bestTj * NT + t) * 8 + l));
            }
        }

        // -------------------------------------------------------- pass B
        float sum_d = 0.f, clip_d = 0.f, clip_q = 0.f, n_clip = 0.f;
        uint32_t clipmask = 0;
        unsigned long long vmass[NV];
#pragma unroll
        for (int j = 0; j < NV; ++j) vmass[j] = 0ull;
        const bool has_clip = DISTILL && isRow && isfinite(p.clip_c);
        const bool do_sample = STOCH && c.g.do_sample;
        if ((DISTILL && isRow) || do_sample) {
            const RowG& g = c.g;
            const float dl = g.dl, cc = p.clip_c;
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                const int vi = j * NT + t;
                if (vi < nvec) {
                    if (isRow) {
                        const float f = fast_exp2(ref[j] * k2 - g.L2D);
                        const float4 lo = dplane[(2 * j) * NT + t];
                        const float4 hi = dplane[(2 * j + 1) * NT + t];
                        const float dd[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
                        float vmax = kNegInf;
                        unsigned long long ms = 0ull;
#pragma unroll
                        for (int l = 0; l < 8; ++l) {
                            const float q = elem_q(e[j][l], f);
                            const float s = elem_s(dd[l], itau, dl);
                            if (DISTILL) {
                                const float d = elem_d(q, s);
                                sum_d += d;
                                vmax = fmaxf(vmax, d);
                            }
                            if (STOCH && do_sample)
                                ms += to_fixed(fmaxf(__fsub_rn(elem_p(q, s), q), 0.f));
                        }
                        if (STOCH) vmass[j] = ms;
                        if (has_clip && vmax > cc) {
                            clipmask |= 1u << j;
#pragma unroll
                            for (int l = 0; l < 8; ++l) {
                                const float q = elem_q(e[j][l], f);
                                const float d = elem_d(q, elem_s(dd[l], itau, dl));
                                if (d > cc) { clip_d += d; clip_q += q; n_clip += 1.f; }
                            }
                        }
                    } else if (STOCH) {
                        // bonus row: masses of p itself
                        const float f = fast_exp2(ref[j] * k2 - g.L2T);
                        unsigned long long ms = 0ull;
#pragma unroll
                        for (int l = 0; l < 8; ++l) ms += to_fixed(elem_q(e[j][l], f));
                        vmass[j] = ms;
                    }
                }
            }
        }

        // exclusive prefix of the sample masses in (round, thread) order; CTA total
        unsigned long long vpre[NV];
#pragma unroll
        for (int j = 0; j < NV; ++j) vpre[j] = 0ull;
        unsigned long long cta_mass = 0ull;
        if (STOCH && do_sample) {
            unsigned long long carry = 0ull;
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                unsigned long long incl = vmass[j];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                if (lane == 31) c.wmass[warp] = incl;
                __syncthreads();
                unsigned long long woff = 0ull, tot = 0ull;
                for (int q = 0; q < NW; ++q) {
                    const unsigned long long v = c.wmass[q];
                    if (q < warp) woff += v;
                    tot += v;
                }
                vpre[j] = carry + woff + incl - vmass[j];
                carry += tot;
                __syncthreads();
            }
            cta_mass = carry;
        }

        // CTA partials of pass B -> slot
        if (DISTILL && isRow) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                sum_d += __shfl_xor_sync(0xffffffffu, sum_d, o);
                clip_d += __shfl_xor_sync(0xffffffffu, clip_d, o);
                clip_q += __shfl_xor_sync(0xffffffffu, clip_q, o);
                n_clip += __shfl_xor_sync(0xffffffffu, n_clip, o);
            }
            if (lane == 0) {
                c.wred[warp][0] = sum_d;
                c.wred[warp][1] = clip_d;
                c.wred[warp][2] = clip_q;
                c.wred[warp][3] = n_clip;
            }
        }
        __syncthreads();
        if (t == 0) {
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
            if (DISTILL && isRow) {
                for (int q = 0; q < NW; ++q) {
                    a0 += c.wred[q][0];
                    a1 += c.wred[q][1];
                    a2 += c.wred[q][2];
                    a3 += c.wred[q][3];
                }
            }
            c.slot.sum_d = a0;
            c.slot.clip_d = a1;
            c.slot.clip_q = a2;
            c.slot.n_clip = a3;
            c.slot.mass = cta_mass;
        }
        cluster_sync();  // #2

        // ---------------------------------------------------- row results (every rank)
        if (warp == 0) {
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
            unsigned long long mass = 0ull, before = 0ull;
            if (lane < static_cast<int>(CL)) {
                const uint32_t a = dsmem_map(&c.slot, lane);
                a0 = dsmem_ld_f32(a + offsetof(Slot, sum_d));
                a1 = dsmem_ld_f32(a + offsetof(Slot, clip_d));
                a2 = dsmem_ld_f32(a + offsetof(Slot, clip_q));
                a3 = dsmem_ld_f32(a + offsetof(Slot, n_clip));
                const uint32_t lo = dsmem_ld_u32(a + offsetof(Slot, mass));
                const uint32_t hi = dsmem_ld_u32(a + offsetof(Slot, mass) + 4);
                mass = (static_cast<unsigned long long>(hi) << 32) | lo;
            }
            // fixed-order sums over ranks (lane order), identical on every rank
            float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
            unsigned long long R = 0ull;
            for (int r = 0; r < static_cast<int>(CL); ++r) {
                s0 += __shfl_sync(0xffffffffu, a0, r);
                s1 += __shfl_sync(0xffffffffu, a1, r);
                s2 += __shfl_sync(0xffffffffu, a2, r);
                s3 += __shfl_sync(0xffffffffu, a3, r);
                const unsigned long long mr = __shfl_sync(0xffffffffu, mass, r);
                if (r < static_cast<int>(rank)) before += mr;
                R += mr;
            }
            if (lane == 0) {
                RowG& g = c.g;
                const uint32_t a = dsmem_map(&c.slot, 0);
                const uint32_t argD = dsmem_ld_u32(a + offsetof(Slot, argD));
                const uint32_t argT = dsmem_ld_u32(a + offsetof(Slot, argT));
                g.y = argT;
                if (isRow && p.draft == nullptr) g.x = argD;
                if (rowVerify && !STOCH) g.acc = (g.x == g.y) ? 1 : 0;
                g.R = R;
                g.off = before;
                g.tgt = scale_mass(R, static_cast<uint32_t>(g.u1 * 16777216.0f));
                g.sum_d = s0;
                g.clip_d = s1;
                g.n_clip = s3;
                if (DISTILL && isRow) {
                    // S = sum over unclipped entries of q (s + 1) = (sum_d - clip_d) + (1 - clip_q)
                    const float S = (s0 - s1) + (1.f - s2);
                    const float lam = p.lambda, pre = p.grad_scale * itau;
                    g.P = pre * (lam + (1.f - lam) * (1.f - S - g.dl));
                    g.Q = pre * (1.f - lam) * itau;
                    g.Pc = pre * (lam - (1.f - lam) * S);
                    g.hardc = pre * lam;
                }
                if (STOCH && g.do_sample && R == 0ull) g.attempt_p = 1;
            }
        }
        __syncthreads();

        // stochastic fallback: residual mass zero -> sample from p (rare; extra reduction)
        if (STOCH && do_sample && c.g.attempt_p) {
            const RowG& g = c.g;
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                vmass[j] = 0ull;
                const int vi = j * NT + t;
                if (vi < nvec) {
                    const float f = fast_exp2(ref[j] * k2 - g.L2D);
                    const float4 lo = dplane[(2 * j) * NT + t];
                    const float4 hi = dplane[(2 * j + 1) * NT + t];
                    const float dd[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
                    unsigned long long ms = 0ull;
#pragma unroll
                    for (int l = 0; l < 8; ++l) {
                        const float q = elem_q(e[j][l], f);
                        ms += to_fixed(elem_p(q, elem_s(dd[l], itau, g.dl)));
                    }
                    vmass[j] = ms;
                }
            }
            unsigned long long carry = 0ull;
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                unsigned long long incl = vmass[j];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                if (lane == 31) c.wmass[warp] = incl;
                __syncthreads();
                unsigned long long woff = 0ull, tot = 0ull;
                for (int q = 0; q < NW; ++q) {
                    const unsigned long long v = c.wmass[q];
                    if (q < warp) woff += v;
                    tot += v;
                }
                vpre[j] = carry + woff + incl - vmass[j];
                carry += tot;
                __syncthreads();
            }
            if (t == 0) c.slot.mass2 = carry;
            cluster_sync();
            if (t == 0) {
                unsigned long long R = 0ull, before = 0ull;
                for (int r = 0; r < static_cast<int>(CL); ++r) {
                    const uint32_t a = dsmem_map(&c.slot, r);
                    const uint32_t lo = dsmem_ld_u32(a + offsetof(Slot, mass2));
                    const uint32_t hi = dsmem_ld_u32(a + offsetof(Slot, mass2) + 4);
                    const unsigned long long mr = (static_cast<unsigned long long>(hi) << 32) | lo;
                    if (r < static_cast<int>(rank)) before += mr;
                    R += mr;
                }
                c.g.R = R;
                c.g.off = before;
                c.g.tgt = scale_mass(R, static_cast<uint32_t>(c.g.u1 * 16777216.0f));
            }
            __syncthreads();
        }

        // -------------------------------------------------------- sample search
        if (STOCH && do_sample && c.g.R > 0ull) {
            const RowG& g = c.g;
            const bool use_p = g.attempt_p != 0;
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                const int vi = j * NT + t;
                const unsigned long long lo = g.off + vpre[j];
                if (vi < nvec && vmass[j] > 0ull && lo <= g.tgt && g.tgt - lo < vmass[j]) {
                    // the sample point lies in this vector: walk its 8 masses in id order
                    const unsigned long long rel = g.tgt - lo;
                    unsigned long long cum = 0ull;
                    int pick = -1;
                    if (isRow) {
                        const float f = fast_exp2(ref[j] * k2 - g.L2D);
                        const float4 a = dplane[(2 * j) * NT + t];
                        const float4 bq = dplane[(2 * j + 1) * NT + t];
                        const float dd[8] = {a.x, a.y, a.z, a.w, bq.x, bq.y, bq.z, bq.w};
#pragma unroll
                        for (int l = 0; l < 8; ++l) {
                            const float q = elem_q(e[j][l], f);
                            const float pv = elem_p(q, elem_s(dd[l], itau, g.dl));
                            cum += use_p ? to_fixed(pv) : to_fixed(fmaxf(__fsub_rn(pv, q), 0.f));
                            if (pick < 0 && cum > rel) pick = l;
                        }
                    } else {
                        const float f = fast_exp2(ref[j] * k2 - g.L2T);
#pragma unroll
                        for (int l = 0; l < 8; ++l) {
                            cum += to_fixed(elem_q(e[j][l], f));
                            if (pick < 0 && cum > rel) pick = l;
                        }
                    }
                    if (pick < 0) pick = 7;
                    dsmem_min_u32(dsmem_map(&c.slot.tok, 0), static_cast<uint32_t>(v0 + vi * 8 + pick));
                }
            }
        }

        // -------------------------------------------------------- pass C: gradient row
        if (DISTILL && isRow) {
            const RowG& g = c.g;
            const float dl = g.dl, cc = p.clip_c;
            const uint32_t y = g.y;
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                const int vi = j * NT + t;
                if (vi < nvec) {
                    const float f = fast_exp2(ref[j] * k2 - g.L2D);
                    const float Pj = f * g.P, Qj = f * g.Q;
                    const float4 lo = dplane[(2 * j) * NT + t];
                    const float4 hi = dplane[(2 * j + 1) * NT + t];
                    const float dd[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
                    float gv[8];
#pragma unroll
                    for (int l = 0; l < 8; ++l) gv[l] = e[j][l] * fmaf(Qj, dd[l], Pj);
                    if (clipmask & (1u << j)) {
#pragma unroll
                        for (int l = 0; l < 8; ++l) {
                            const float q = elem_q(e[j][l], f);
                            const float d = elem_d(q, elem_s(dd[l], itau, dl));
                            if (d > cc) gv[l] = q * g.Pc;
                        }
                    }
                    const int base = v0 + vi * 8;
                    if (y >= static_cast<uint32_t>(base) && y < static_cast<uint32_t>(base + 8)) {
                        const int l = static_cast<int>(y) - base;
                        float dy = dd[0];
#pragma unroll
                        for (int q = 1; q < 8; ++q) if (q == l) dy = dd[q];
#pragma unroll
                        for (int q = 0; q < 8; ++q) if (q == l) gv[q] -= g.hardc;
                        // -log q_y = lseD - D_y / tau, with D_y = delta_y + T_y and T_y = max T
                        dsmem_st_f32(dsmem_map(&c.slot.ce, 0), g.lseD - (dy + g.MT) * itau);
                    }
                    if (p.aligned) {
                        if (p.dl_fp32) {
                            float4* o = reinterpret_cast<float4*>(static_cast<float*>(p.dlogits) + drow * V + base);
                            __stcs(o, make_float4(gv[0], gv[1], gv[2], gv[3]));
                            __stcs(o + 1, make_float4(gv[4], gv[5], gv[6], gv[7]));
                        } else {
                            uint4 pk;
                            pk.x = pack_bf16x2(gv[0], gv[1]);
                            pk.y = pack_bf16x2(gv[2], gv[3]);
                            pk.z = pack_bf16x2(gv[4], gv[5]);
                            pk.w = pack_bf16x2(gv[6], gv[7]);
                            __stcs(reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.dlogits) + drow * V + base), pk);
                        }
                    } else {
#pragma unroll
                        for (int l = 0; l < 8; ++l) {
                            if (base + l < V && vi * 8 + l < len) {
                                if (p.dl_fp32) static_cast<float*>(p.dlogits)[drow * V + base + l] = gv[l];
                                else static_cast<uint16_t*>(p.dlogits)[drow * V + base + l] =
                                    static_cast<uint16_t>(pack_bf16x2(gv[l], 0.f) & 0xffffu);
                            }
                        }
                    }
                }
            }
        } else if (DISTILL && !isRow && i < p.k) {
            // bonus row: its gradient row is zero
            if (p.aligned) {
                const uint4 z = make_uint4(0, 0, 0, 0);
                if (p.dl_fp32) {
                    float* gp = static_cast<float*>(p.dlogits) + drow * V + v0;
                    for (int e2 = t * 4; e2 < len; e2 += NT * 4) __stcs(reinterpret_cast<uint4*>(gp + e2), z);
                } else {
                    uint16_t* gp = static_cast<uint16_t*>(p.dlogits) + drow * V + v0;
                    for (int e2 = t * 8; e2 < len; e2 += NT * 8) __stcs(reinterpret_cast<uint4*>(gp + e2), z);
                }
            } else {
                for (int e2 = t; e2 < len; e2 += NT) {
                    if (p.dl_fp32) static_cast<float*>(p.dlogits)[drow * V + v0 + e2] = 0.f;
                    else static_cast<uint16_t*>(p.dlogits)[drow * V + v0 + e2] = 0;
                }
            }
        }
        cluster_sync();  // #3: deposits (token, CE) visible in rank 0

        // -------------------------------------------------------- row record, ticket, scan
        if (rank == 0 && warp == 0) {
            int fin = 0;
            if (lane == 0) {
                const RowG& g = c.g;
                svd_row_info r;
                r.draft_token = rowVerify ? static_cast<int32_t>(g.x == kNone ? -1 : static_cast<int>(g.x)) : -1;
                r.target_argmax = static_cast<int32_t>(g.y);
                r.accepted = rowVerify ? g.acc : -1;
                if (!verify) r.sample_token = -1;
                else if (!STOCH) r.sample_token = static_cast<int32_t>(g.y);
                else r.sample_token = (g.do_sample && c.slot.tok != kNone) ? static_cast<int32_t>(c.slot.tok) : -1;
                r.ratio = g.ratio;
                r.lse_draft = isRow ? g.lseD : __int_as_float(0x7fc00000);
                r.lse_target = g.lseT;
                float L = 0.f;
                if (DISTILL && isRow) {
                    const float Kc = isfinite(p.clip_c) ? (g.sum_d - g.clip_d) + p.clip_c * g.n_clip : g.sum_d;
                    L = p.lambda * c.slot.ce + (1.f - p.lambda) * Kc;
                    if (p.loss_rows) p.loss_rows[drow] = L;
                }
                r.loss = L;
                p.rec[trow] = r;
                if (p.row_info) p.row_info[trow] = r;
                // reset the rank-0 deposit targets for the next row
                c.slot.argD = kNone;
                c.slot.argT = kNone;
                c.slot.tok = kNone;
                c.slot.ce = 0.f;
                __threadfence();
                const int n = get_bk(p, b);
                const uint32_t expected = static_cast<uint32_t>(n + ((verify && n < p.kt) ? 1 : 0));
                const uint32_t old = atomicAdd(&p.seq_ticket[b], 1u);
                fin = (old + 1u == expected) ? 1 : 0;
            }
            fin = __shfl_sync(0xffffffffu, fin, 0);
            if (fin) {
                // ---------------- sequence b complete: acceptance scan (one lane per position)
                __threadfence();
                const int n = get_bk(p, b);
                const int kt = p.kt, k = p.k;
                svd_row_info r;
                r.draft_token = -1; r.target_argmax = -1; r.accepted = -1; r.sample_token = -1;
                r.ratio = r.lse_draft = r.lse_target = __int_as_float(0x7fc00000);
                r.loss = 0.f;
                auto is_processed = [&](int row) { return row < n || (verify && row == n && n < kt); };
                if (lane < kt && is_processed(lane)) {
                    const svd_row_info* src = p.rec + static_cast<size_t>(b) * kt + lane;
                    r.draft_token = __ldcg(&src->draft_token);
                    r.target_argmax = __ldcg(&src->target_argmax);
                    r.accepted = __ldcg(&src->accepted);
                    r.sample_token = __ldcg(&src->sample_token);
                    r.loss = __ldcg(&src->loss);
                } else if (lane < kt && p.row_info) {
                    p.row_info[static_cast<size_t>(b) * kt + lane] = r;  // unprocessed row
                }
                if (kt == 33 && lane == 0 && !is_processed(32) && p.row_info) {
                    svd_row_info u = r;
                    u.draft_token = u.target_argmax = u.accepted = u.sample_token = -1;
                    u.ratio = u.lse_draft = u.lse_target = __int_as_float(0x7fc00000);
                    u.loss = 0.f;
                    p.row_info[static_cast<size_t>(b) * kt + 32] = u;
                }
                if (verify) {
                    const uint32_t accm = __ballot_sync(0xffffffffu, lane < n && r.accepted == 1);
                    const uint32_t notacc = ~accm;
                    int a = __ffs(notacc) - 1;
                    if (a > n || a < 0) a = n;
                    const int fix_row = a < n ? a : ((n < kt) ? n : -1);
                    int fix_tok = __shfl_sync(0xffffffffu, r.sample_token, fix_row < 0 ? 0 : (fix_row & 31));
                    if (fix_row >= 32)  // bonus row 32 (k = 32, kt = 33) has no lane of its own
                        fix_tok = __ldcg(&p.rec[static_cast<size_t>(b) * kt + 32].sample_token);
                    // lane q holds row q's record; slot k (= 32 at most) has no row of its own and
                    // can only hold the correction / bonus token
                    if (lane < k + 1) {
                        int v = -1;
                        if (lane < a) v = r.draft_token;
                        else if (lane == a && fix_row >= 0) v = fix_tok;
                        p.emitted[static_cast<size_t>(b) * (k + 1) + lane] = v;
                    }
                    if (k == 32 && lane == 0)
                        p.emitted[static_cast<size_t>(b) * (k + 1) + 32] = (a == 32 && fix_row >= 0) ? fix_tok : -1;
                    if (lane == 0) {
                        p.accept_len[b] = a;
                        p.n_emitted[b] = a + (fix_row >= 0 ? 1 : 0);
                    }
                }
                if (DISTILL) {
                    // rows past b_k have no loss: their entries of loss_rows are zero
                    if (p.loss_rows && lane >= n && lane < k)
                        p.loss_rows[static_cast<size_t>(b) * k + lane] = 0.f;
                    float ls = 0.f;
                    for (int q = 0; q < n; ++q) ls += __shfl_sync(0xffffffffu, r.loss, q);
                    if (lane == 0) {
                        p.seq_loss[b] = ls;
                        p.seq_ticket[b] = 0u;
                        __threadfence();
                        const uint32_t old = atomicAdd(&p.hdr->loss_ticket, 1u);
                        if (old + 1u == static_cast<uint32_t>(p.B)) {
                            __threadfence();
                            float tot = 0.f;
                            for (int s = 0; s < p.B; ++s) tot += __ldcg(p.seq_loss + s);
                            *p.loss_total = tot;
                            p.hdr->loss_ticket = 0u;
                        }
                    }
                } else if (lane == 0) {
                    p.seq_ticket[b] = 0u;
                }
            }
        }
        __syncthreads();
        if (t == 0) { c.kind = c.nkind; c.b = c.nb; c.i = c.ni; }
        __syncthreads();
        w = wn;
    }
}

// ------------------------------------------------------------------------------------------
// host side: geometry, occupancy, launch
// ------------------------------------------------------------------------------------------
namespace {

template <int NT, int NV>
constexpr size_t smem_bytes() {
    // staging D, T | delta planes | barriers | control block
    return ctl_offset<NT, NV>() + sizeof(Ctl<NT / 32>);
}

using KernelFn = void (*)(RowParams);

template <int NT, int NV>
KernelFn pick_kernel(int flags) {
    const bool dist = (flags & kFlagDistill) != 0, sto = (flags & kFlagStochastic) != 0;
    if (dist && sto) return row_pass_kernel<NT, NV, true, true>;
    if (dist) return row_pass_kernel<NT, NV, true, false>;
    if (sto) return row_pass_kernel<NT, NV, false, true>;
    return row_pass_kernel<NT, NV, false, false>;
}

constexpr int kSmallNT = 128, kSmallNV = 2;
constexpr int kLargeNT = 512, kLargeNV = 5;

int next_pow2(int x) {
    int r = 1;
    while (r < x) r <<= 1;
    return r;
}

}  // namespace

bool row_geometry(int V, RowGeometry* g) {
    if (V < 1) return false;
    const int small_cap = kSmallNT * kSmallNV * 8;   // 2048
    const int large_cap = kLargeNT * kLargeNV * 8;   // 20480
    if (V <= 8 * small_cap) {
        g->variant = 0;
        g->threads = kSmallNT;
        g->cluster = next_pow2((V + small_cap - 1) / small_cap);
        g->smem = smem_bytes<kSmallNT, kSmallNV>();
    } else {
        g->variant = 1;
        g->threads = kLargeNT;
        g->cluster = next_pow2((V + large_cap - 1) / large_cap);
        g->smem = smem_bytes<kLargeNT, kLargeNV>();
    }
    if (g->cluster > 16) return false;
    const int per = (V + g->cluster - 1) / g->cluster;
    g->chunk = (per + 7) & ~7;
    return true;
}

int launch_row_pass(const RowParams& p, void* stream) {
    RowGeometry geo;
    if (!row_geometry(p.V, &geo)) return static_cast<int>(cudaErrorInvalidValue);
    KernelFn fn = geo.variant == 0 ? pick_kernel<kSmallNT, kSmallNV>(p.flags)
                                   : pick_kernel<kLargeNT, kLargeNV>(p.flags);
    cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(geo.smem));
    if (err != cudaSuccess) return static_cast<int>(err);
    if (geo.cluster > 8) {
        err = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (err != cudaSuccess) return static_cast<int>(err);
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = geo.cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.blockDim = dim3(geo.threads, 1, 1);
    cfg.dynamicSmemBytes = geo.smem;
    cfg.stream = static_cast<cudaStream_t>(stream);
    // persistent grid: as many clusters as can be resident at once
    static int cached_clusters[2][17][8] = {};
    const int fidx = p.flags & 7;
    int& cache = cached_clusters[geo.variant][geo.cluster][fidx];
    if (cache == 0) {
        int dev = 0, sms = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cfg.gridDim = dim3(geo.cluster * sms, 1, 1);
        int n = 0;
        err = cudaOccupancyMaxActiveClusters(&n, fn, &cfg);
        if (err != cudaSuccess || n < 1) n = sms / geo.cluster > 0 ? sms / geo.cluster : 1;
        cache = n;
    }
    const long long max_items = static_cast<long long>(p.B) * (p.kt + p.k);
    int nclusters = cache;
    if (max_items < nclusters) nclusters = static_cast<int>(max_items > 0 ? max_items : 1);
    cfg.gridDim = dim3(geo.cluster * nclusters, 1, 1);
    RowParams q = p;
    q.chunk = geo.chunk;
    err = cudaLaunchKernelEx(&cfg, fn, q);
    return static_cast<int>(err);
}

}  // namespace svd
