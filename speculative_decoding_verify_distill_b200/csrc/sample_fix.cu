// sample_fix.cu -- stochastic verification's drawn token, one per sequence: from the residual
// max(0, p - q) of the first rejected row, or from p of the bonus row when every verified draft
// was accepted and a bonus row exists (speculative sampling, the acceptance rule of the Pith
// review page's Axiom & Free-Parameter Ledger after Leviathan et al. 2023), by inverse CDF over
// ascending ids with the Philox word that row owns (word 1 of (seed, step, sequence, row)).
//
// Runs after the finalize pass, which fixed the accepted length a_b and so the one row per
// sequence whose draw is emitted; the row pass draws nothing.  One cluster of C CTAs per
// sequence (C = ceil(V / 16384), at most 8), each CTA a contiguous slice of ids:
//   1. the slice's masses, as 2^-48 fixed-point integers, of the residual and of p (so an empty
//      residual falls back to p without a second pass), sent to every CTA of the cluster over
//      distributed shared memory;
//   2. every CTA forms the same totals and the same prefix in rank order; the CTA whose
//      interval holds the target floor(R * u / 2^24) finds the round of 256 vectors that holds
//      it from the per-round masses it kept in shared memory in step 1, the vector by a block
//      scan over that round, and the token by re-reading that one vector.  (Slices of more
//      than 16 rounds, and an empty residual that falls back to p, search by re-reading the
//      slice round by round instead.)
// Integer masses make the prefix sums exact and associative, so the split over CTAs cannot
// change the draw.  Element arithmetic is the row pass's (svd_device.cuh) with lse(D/tau) and
// lse(T/tau) read back from the row record.
#include <cuda_runtime.h>

#include "svd_device.cuh"

namespace svd {
namespace {

constexpr int kFixThreads = 256;
constexpr int kFixWarps = kFixThreads / 32;
constexpr int kFixMaxCluster = 8;
constexpr int kFixSlice = 16384;              // ids per CTA before the cluster grows
constexpr int kFixMaxRounds = 16;             // rounds of 256 vectors whose masses are kept
constexpr int kFixUnroll = 2;                 // vectors in flight per thread in step 1

// Vector g (ids 8g .. 8g+7) of a row of V ids; ids past V read as the lowest finite bf16,
// whose probability is 0.
template <bool ALIGNED>
__device__ __forceinline__ uint4 row_vec(const uint16_t* row, int g, int V) {
    if constexpr (ALIGNED) {
        return __ldg(reinterpret_cast<const uint4*>(row) + g);
    } else {
        uint32_t w[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const int id = g * 8 + 2 * h;
            const uint32_t lo = id < V ? __ldg(row + id) : 0xFF7Fu;
            const uint32_t hi = id + 1 < V ? __ldg(row + id + 1) : 0xFF7Fu;
            w[h] = lo | (hi << 16);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// The sample weights of a vector's 8 elements in 2^-48 units: wp = p, and with `residual`
// also wr = max(0, p - q).
__device__ __forceinline__ void vec_masses(const uint4& tv, const uint4& dv, bool residual,
                                           float k2, float L2T, float L2D,
                                           unsigned long long (&wp)[8],
                                           unsigned long long (&wr)[8]) {
    float xt[8], xd[8];
    unpack8(tv, xt);
    if (residual) unpack8(dv, xd);
#pragma unroll
    for (int l = 0; l < 8; ++l) {
        const float pv = elem_p(xt[l], k2, L2T);
        wp[l] = to_fixed(pv);
        wr[l] = residual ? to_fixed(fmaxf(__fsub_rn(pv, elem_q(xd[l], k2, L2D)), 0.f)) : 0ull;
    }
}

template <bool ALIGNED>
__global__ void __launch_bounds__(kFixThreads, 4) sample_fix_kernel(const RowParams p, int slice) {
    __shared__ unsigned long long red[2][kFixWarps];
    __shared__ unsigned long long cm[kFixMaxCluster][2];   // [rank][residual, p] masses
    __shared__ unsigned long long scan[kFixWarps];
    __shared__ unsigned long long vmr[kFixMaxRounds][kFixThreads];   // [round][thread] masses
    __shared__ unsigned long long rtot[kFixMaxRounds][kFixWarps];    // [round][warp] sums
    __shared__ int found, sround;
    __shared__ unsigned long long srel;
    // launched as a programmatic dependent of the finalize pass: wait for its accepted lengths
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const uint32_t rank = cluster_rank(), CL = cluster_size();
    const int b = static_cast<int>(cluster_id_x());
    const int k = p.k, kt = p.kt, V = p.V;
    int n = p.bk_const > 0 ? p.bk_const : __ldg(p.bk + b);
    n = n < 1 ? 1 : (n > k ? k : n);
    const int a = p.accept_len[b];
    const int fix = a < n ? a : (n < kt ? n : -1);
    if (fix < 0) return;                       // the same for every CTA of the cluster
    const bool residual = a < n;               // a rejected row; else the bonus row
    const svd_row_info& rr = p.rec[static_cast<size_t>(b) * kt + fix];
    const float k2 = p.k2;
    const float L2T = rr.lse_target * kLog2e;  // as the row pass formed them
    const float L2D = residual ? rr.lse_draft * kLog2e : 0.f;
    const uint16_t* Trow = p.T + (static_cast<size_t>(b) * kt + fix) * V;
    const uint16_t* Drow = p.D + (static_cast<size_t>(b) * k + fix) * V;
    const int v0 = static_cast<int>(rank) * slice;          // slice: a multiple of 8 ids
    const int v1 = min(V, v0 + slice);
    const int gbeg = v0 / 8, gend = v1 > v0 ? (v1 + 7) / 8 : gbeg;

    // 1. this slice's masses, to every CTA of the cluster; per round of 256 vectors each thread
    //    also keeps its vector's mass of the column a search would use (residual, or p)
    const int rounds = (gend - gbeg + kFixThreads - 1) / kFixThreads;
    const bool keep = rounds <= kFixMaxRounds;
    unsigned long long m = 0ull, pm = 0ull;
    for (int i0 = 0; i0 < rounds; i0 += kFixUnroll) {
        uint4 tv[kFixUnroll], dv[kFixUnroll];
#pragma unroll
        for (int u = 0; u < kFixUnroll; ++u) {
            const int g = gbeg + t + (i0 + u) * kFixThreads;
            if (g < gend) {
                tv[u] = row_vec<ALIGNED>(Trow, g, V);
                dv[u] = residual ? row_vec<ALIGNED>(Drow, g, V) : tv[u];
            }
        }
#pragma unroll
        for (int u = 0; u < kFixUnroll; ++u) {
            const int i = i0 + u;
            if (i >= rounds) break;
            const int g = gbeg + t + i * kFixThreads;
            unsigned long long vr = 0ull, vp = 0ull;
            if (g < gend) {
                unsigned long long wp[8], wr[8];
                vec_masses(tv[u], dv[u], residual, k2, L2T, L2D, wp, wr);
#pragma unroll
                for (int l = 0; l < 8; ++l) { vr += wr[l]; vp += wp[l]; }
            }
            m += vr;
            pm += vp;
            if (keep) vmr[i][t] = residual ? vr : vp;
        }
    }
    m = warp_sum_u64(m);
    pm = warp_sum_u64(pm);
    if (lane == 0) { red[0][warp] = m; red[1][warp] = pm; }
    __syncthreads();
    if (t < static_cast<int>(CL)) {
        unsigned long long sm = 0ull, sp = 0ull;
        for (int q = 0; q < kFixWarps; ++q) { sm += red[0][q]; sp += red[1][q]; }
        if (!residual) sm = sp;
        const uint32_t dst = dsmem_map(&cm[rank][0], static_cast<uint32_t>(t));
        dsmem_st_u32(dst, static_cast<uint32_t>(sm));
        dsmem_st_u32(dst + 4, static_cast<uint32_t>(sm >> 32));
        dsmem_st_u32(dst + 8, static_cast<uint32_t>(sp));
        dsmem_st_u32(dst + 12, static_cast<uint32_t>(sp >> 32));
    }
    cluster_sync();   // every CTA holds every slice's masses; no remote access after this

    // 2. totals, the target and the owning slice (the same arithmetic in every CTA)
    unsigned long long R = 0ull;
    for (uint32_t r = 0; r < CL; ++r) R += cm[r][0];
    const int col = (residual && R == 0ull) ? 1 : 0;   // empty residual: sample from p
    if (col == 1)
        for (uint32_t r = 0; r < CL; ++r) R += cm[r][1];
    if (R == 0ull) return;
    const PhiloxOut ph = philox_words(p.seed, p.step, static_cast<uint32_t>(b), static_cast<uint32_t>(fix));
    const unsigned long long tgt = scale_mass(R, static_cast<uint32_t>(uniform24(ph.w[1]) * 16777216.0f));
    unsigned long long before = 0ull;
    for (uint32_t r = 0; r < rank; ++r) before += cm[r][col];
    const unsigned long long mine = cm[rank][col];
    if (mine == 0ull || tgt < before || tgt - before >= mine) return;
    const unsigned long long rel = tgt - before;
    const bool res = residual && col == 0;
    if (t == 0) found = -1;
    if (keep && col == 0) {
        // the round holding the target, from the kept masses (every thread of a round holds the
        // vector gbeg + t + i * 256, so thread order is id order within a round)
        for (int i = 0; i < rounds; ++i) {
            const unsigned long long ws = warp_sum_u64(vmr[i][t]);
            if (lane == 0) rtot[i][warp] = ws;
        }
        __syncthreads();
        if (t == 0) {
            unsigned long long run = 0ull;
            sround = rounds - 1;
            srel = 0ull;
            for (int i = 0; i < rounds; ++i) {
                unsigned long long tot = 0ull;
                for (int q = 0; q < kFixWarps; ++q) tot += rtot[i][q];
                if (rel - run < tot) {   // run <= rel throughout: the first round passing rel
                    sround = i;
                    srel = rel - run;
                    break;
                }
                run += tot;
            }
        }
        __syncthreads();
        const int i = sround;
        const unsigned long long rr = srel;
        const unsigned long long vm = vmr[i][t];
        unsigned long long incl = vm;
        warp_inclusive_scan_u64(incl);
        if (lane == 31) scan[warp] = incl;
        __syncthreads();
        unsigned long long wbefore = 0ull;
#pragma unroll
        for (int q = 0; q < kFixWarps; ++q)
            if (q < warp) wbefore += scan[q];
        const unsigned long long lo = wbefore + incl - vm;
        if (vm > 0ull && lo <= rr && rr - lo < vm) {
            // the target lies in this vector: its 8 masses again, walked in id order
            const int g = gbeg + t + i * kFixThreads;
            const uint4 tv = row_vec<ALIGNED>(Trow, g, V);
            const uint4 dv = res ? row_vec<ALIGNED>(Drow, g, V) : tv;
            unsigned long long w[8], wr[8];
            vec_masses(tv, dv, res, k2, L2T, L2D, w, wr);
            const unsigned long long r8 = rr - lo;
            unsigned long long cum = 0ull;
            int pick = -1;
#pragma unroll
            for (int l = 0; l < 8; ++l) {
                cum += res ? wr[l] : w[l];
                if (pick < 0 && cum > r8) pick = l;
            }
            found = g * 8 + (pick < 0 ? 7 : pick);
        }
        __syncthreads();
        if (t == 0 && found >= 0) {
            p.emitted[static_cast<size_t>(b) * (k + 1) + a] = found;
            p.rec[static_cast<size_t>(b) * kt + fix].sample_token = found;
            if (p.row_info) p.row_info[static_cast<size_t>(b) * kt + fix].sample_token = found;
        }
        return;
    }
    unsigned long long run = 0ull;    // mass of this slice's vectors before the round, id order
    for (int r0 = gbeg; r0 < gend; r0 += kFixThreads) {
        const int g = r0 + t;
        unsigned long long w[8], wr[8];
        unsigned long long vm = 0ull;
        if (g < gend) {
            const uint4 tv = row_vec<ALIGNED>(Trow, g, V);
            const uint4 dv = res ? row_vec<ALIGNED>(Drow, g, V) : tv;
            vec_masses(tv, dv, res, k2, L2T, L2D, w, wr);
#pragma unroll
            for (int l = 0; l < 8; ++l) {
                if (res) w[l] = wr[l];
                vm += w[l];
            }
        }
        unsigned long long incl = vm;
        warp_inclusive_scan_u64(incl);
        __syncthreads();
        if (lane == 31) scan[warp] = incl;
        __syncthreads();
        unsigned long long wbefore = 0ull, total = 0ull;
#pragma unroll
        for (int q = 0; q < kFixWarps; ++q) {
            if (q < warp) wbefore += scan[q];
            total += scan[q];
        }
        const unsigned long long lo = run + wbefore + incl - vm;
        if (vm > 0ull && lo <= rel && rel - lo < vm) {
            // the target lies in this vector: walk its 8 masses in id order
            const unsigned long long r8 = rel - lo;
            unsigned long long cum = 0ull;
            int pick = -1;
#pragma unroll
            for (int l = 0; l < 8; ++l) {
                cum += w[l];
                if (pick < 0 && cum > r8) pick = l;
            }
            found = g * 8 + (pick < 0 ? 7 : pick);
        }
        run += total;
        if (run > rel) break;   // uniform: every thread holds the same run
    }
    __syncthreads();
    if (t == 0 && found >= 0) {
        p.emitted[static_cast<size_t>(b) * (k + 1) + a] = found;
        p.rec[static_cast<size_t>(b) * kt + fix].sample_token = found;
        if (p.row_info) p.row_info[static_cast<size_t>(b) * kt + fix].sample_token = found;
    }
}

}  // namespace

int launch_sample_fix(const RowParams& p, void* stream) {
    if (p.B < 1) return 0;
    int cl = (p.V + kFixSlice - 1) / kFixSlice;
    cl = cl < 1 ? 1 : (cl > kFixMaxCluster ? kFixMaxCluster : cl);
    const int per = (p.V + cl - 1) / cl;
    const int slice = (per + 7) & ~7;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(cl);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // a programmatic dependent of the finalize pass (its CTAs start while finalize runs and
    // wait in griddepcontrol.wait): the launch latency overlaps the finalize pass
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cfg.gridDim = dim3(static_cast<unsigned>(p.B) * cl, 1, 1);
    cfg.blockDim = dim3(kFixThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaError_t err = p.aligned ? cudaLaunchKernelEx(&cfg, sample_fix_kernel<true>, p, slice)
                                : cudaLaunchKernelEx(&cfg, sample_fix_kernel<false>, p, slice);
    return static_cast<int>(err);
}

}  // namespace svd
