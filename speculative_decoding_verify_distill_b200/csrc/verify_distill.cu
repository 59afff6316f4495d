// verify_distill.cu -- the fused row pass: truncated verification (greedy / stochastic) and the
// clipped reverse-KL + CE distillation loss with its gradient, one HBM read per logit row; and the
// small finalize pass that turns per-row records into accepted lengths, emitted tokens and loss
// sums.
//
// What it computes (AdaFlash; Pith review page "What carries the argument", Axiom & Free-
// Parameter Ledger, Referee Report major comment 2; Pith verdict record load_bearing_attack):
// for every sequence b the first b_k draft rows are verified against the target rows, the
// acceptance length a_b and the emitted tokens follow the standard speculative-decoding rule,
// and every verified row i < b_k also yields the OPD loss L_i and dL/dD_i; rows i >= b_k get a
// zero gradient row.
//
// Design (B200, sm_100a):
//   * A persistent grid of thread-block clusters (16 CTAs of 256 threads for a 151936-id
//     vocabulary, several CTAs per SM).  A cluster owns one logit row at a time; each CTA a
//     contiguous slice of the vocabulary; each warp a contiguous run of 16-byte vectors of the
//     slice.  Loaded work items (verified rows and bonus rows) form a compact list (prefix sums
//     of loaded rows per sequence) handed out one row at a time from a workspace ticket, so a
//     cluster that starts late (behind the length head, or beside other work) simply takes fewer
//     rows.  Zero-only gradient rows follow, in quarter-row units handed out to single CTAs,
//     without cluster barriers.
//   * Each warp stages its run of D and T in shared memory with its own 1-D bulk copies
//     (cp.async.bulk, no multicast) on its own mbarrier.  The staged bf16 slice is the only copy:
//     every pass re-reads it, so a CTA holds no per-element state in registers and several CTAs
//     fit on one SM, each hiding the others' barrier and reduction latency.
//   * Pass A: a max pre-pass fixes each thread's exp reference, then exp of D and T, the tree
//     sums, the reverse-KL moment sum e(D - T) and max(D - T).  Reduction #1 (warp -> CTA ->
//     cluster over DSMEM) gives lse(D/tau), lse(T/tau) and the unclipped reverse-KL.
//   * Pass B: only entries with q > c / max(log q - log p) can be clipped; those vectors alone
//     are re-read and tested.  Stochastic rows take their sample masses here as 2^-48 fixed-point
//     integers (exact, associative prefix sums).  Argmax (lowest id) is resolved lazily by the
//     threads holding the row maximum.  Reduction #2.
//   * Pass C: dL/dD = q (P + Q (D - T)) with the clipped and hard-label corrections, q
//     recomputed from the staged logits, 16-byte streaming stores.
//   * Rank 0 writes the row record after the next cluster barrier; the finalize kernel runs the
//     warp-ballot acceptance scan per sequence and the fixed-order loss sums.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>

#include "svd_device.cuh"

namespace svd {

namespace {

constexpr uint32_t kNone = 0xffffffffu;
#define kNegInf (-__int_as_float(0x7f800000))
#define kQNaN (__int_as_float(0x7fc00000))

enum ItemKind : int { kItemNone = 0, kItemRow = 1, kItemBonus = 2 };

// Per-warp / per-CTA partials of the two cluster reductions.  Sums are relative to the maxima
// they travel with (exp(x - m) in the log2-scaled domain).
struct alignas(16) Part1 {
    float mD, sD, sDd, dmax;   // max D, sum exp, sum exp * (D - T), max (D - T)
    float mT, sT, pad0, pad1;  // max T, sum exp
};
struct alignas(16) Part2 {
    float clip_d, clip_q, n_clip, pad0;    // clipped reverse-KL entries
    unsigned long long mass;               // sample mass (2^-48 units)
    unsigned long long pad1;
};
// Deposit targets in rank 0, double-buffered by row parity (read one row later).
struct alignas(16) Deposit {
    uint32_t argD, argT;       // lowest index holding the row max (red.min)
    uint32_t tok;              // sampled token (red.min)
    float ce;                  // -log q_y, from the owner of y
};
// Row values rank 0 keeps until the record is written.
struct Pending {
    int b, i, kind;
    int x, y, acc, do_sample;
    float ratio, lseD, lseT, kc;
};

template <int NW>
struct Ctl {
    Part1 p1[NW];              // per-warp partials (local)
    Part2 p2[NW];
    Part1 cta1;                // CTA partials, read by every warp of the cluster over DSMEM
    Part2 cta2;
    Part2 cta3;                // fallback reduction (residual mass zero: sample from p)
    unsigned long long wpre[NW];  // exclusive prefix of the warps' sample masses in this CTA
    Deposit dep[2];
    Pending pend;
    int wscan[NW];             // prologue scan of the loaded-row counts
    int wscanz[NW];            // ... and of the zero-gradient row counts
    int next_w[2];             // rank 0: the next loaded item, by row parity (read over DSMEM)
    int zs;                    // zero phase: the CTA's next unit
};

// Batches up to this size keep b_k and the prefixes of loaded and zero-gradient rows per sequence
// in shared memory (compact lists, handed out dynamically); larger batches walk the uncompacted
// (sequence, row) slots in a fixed order.
constexpr int kCompactMaxB = 4096;
// Zero-gradient rows are handed out in quarters (about 75 KB of stores each at V = 151936).
constexpr int kZeroSplit = 4;

struct Item {
    int kind, b, i;
};

__device__ __forceinline__ int clamp_bk(const RowParams& p, int n) {
    if (n < 1 || n > p.k) {
        set_device_error(&p.hdr->status, SVD_ERR_INVALID_ARG);
        n = n < 1 ? 1 : p.k;
    }
    return n;
}

// Loaded rows of a sequence: its verified rows, plus the bonus row when b_k < kt.
__device__ __forceinline__ int loaded_rows(int n, int kt, bool verify) {
    return n + ((verify && n < kt) ? 1 : 0);
}

// Gradient rows that only need zeros: i >= b_k, except the bonus row b_k (zeroed by its item).
__device__ __forceinline__ bool zero_row_pred(int k, int n, int i, bool verify) {
    return i < k && (verify ? (n < i) : (n <= i));
}
// How many there are in a sequence, and the first of them.
__device__ __forceinline__ int zero_rows(int k, int n, bool verify) {
    return verify ? max(0, k - n - 1) : k - n;
}
__device__ __forceinline__ int first_zero_row(int n, bool verify) { return verify ? n + 1 : n; }

// b_k of sequence b: from shared memory (compact mode) or global memory (clamped).
struct BkView {
    const int* s;       // shared copy, or nullptr
    const int32_t* g;   // global
    __device__ __forceinline__ int operator()(const RowParams& p, int b) const {
        return s ? s[b] : clamp_bk(p, __ldg(g + b));
    }
};

// Loaded item w of the whole batch.  Compact mode: w indexes the list of loaded rows ordered by
// sequence (prefix sums in shared memory, binary search).  Otherwise w is a (sequence, row) slot
// and holes decode to kItemNone.
__device__ __forceinline__ Item decode_loaded(const RowParams& p, const int* spre, const BkView& bkv,
                                              int w, bool verify) {
    Item it{kItemNone, -1, -1};
    if (spre) {
        if (w >= spre[p.B]) return it;
        int lo = 0, hi = p.B;  // largest b with spre[b] <= w
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (spre[mid] <= w) lo = mid; else hi = mid;
        }
        const int i = w - spre[lo];
        const int n = bkv(p, lo);
        it = Item{i < n ? kItemRow : kItemBonus, lo, i};
    } else {
        if (w >= p.B * p.kt) return it;
        const int b = w / p.kt, i = w % p.kt;
        const int n = bkv(p, b);
        if (i < n) it = Item{kItemRow, b, i};
        else if (verify && i == n) it = Item{kItemBonus, b, i};
    }
    return it;
}

// Number of loaded-item slots to walk (compact: exact count; otherwise all slots).
__device__ __forceinline__ int loaded_slots(const RowParams& p, const int* spre) {
    return spre ? spre[p.B] : p.B * p.kt;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
// Scale factor that moves a sum relative to max m onto the common max M (0 for empty sums).
__device__ __forceinline__ float rescale(float m, float M, float k2) {
    return m == kNegInf ? 0.f : fast_exp2((m - M) * k2);
}
// Reduces per-lane Part1 values over the warp: maxima first, then one rescale per lane, then
// plain sums; every lane ends with the result.
__device__ __forceinline__ Part1 warp_reduce_part1(const Part1& a, float k2) {
    Part1 r;
    r.mD = warp_max(a.mD);
    r.mT = warp_max(a.mT);
    r.dmax = warp_max(a.dmax);
    const float cD = rescale(a.mD, r.mD, k2), cT = rescale(a.mT, r.mT, k2);
    r.sD = warp_sum(a.sD * cD);
    r.sDd = warp_sum(a.sDd * cD);
    r.sT = warp_sum(a.sT * cT);
    r.pad0 = r.pad1 = 0.f;
    return r;
}
__device__ __forceinline__ Part1 empty_part1() {
    Part1 r;
    r.mD = r.mT = r.dmax = kNegInf;
    r.sD = r.sDd = r.sT = 0.f;
    r.pad0 = r.pad1 = 0.f;
    return r;
}
__device__ __forceinline__ float sum8(const float (&v)[8]) {
    return ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
}
__device__ __forceinline__ float max8f(const float (&v)[8]) {
    return fmaxf(fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3])), fmaxf(fmaxf(v[4], v[5]), fmaxf(v[6], v[7])));
}

// Per-element quantities with explicit rounding (no contraction), so that the values summed in
// pass B and the values recomputed later (clip decisions, sample search) are bit-identical.
// q_v = exp(D_v / tau - lseD) and p_v = exp(T_v / tau - lseT) from the staged bf16 logits.
__device__ __forceinline__ float elem_q(float xd, float k2, float L2D) {
    return fast_exp2(__fmaf_rn(xd, k2, -L2D));
}
__device__ __forceinline__ float elem_p(float xt, float k2, float L2T) {
    return fast_exp2(__fmaf_rn(xt, k2, -L2T));
}
__device__ __forceinline__ float elem_s(float xd, float xt, float itau, float dl) {
    return __fmaf_rn(__fsub_rn(xd, xt), itau, -dl);
}
__device__ __forceinline__ float elem_d(float q, float s) { return __fmul_rn(q, s); }
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

__device__ __forceinline__ void dsmem_ld4(uint32_t a, float (&v)[4]) {
    asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3])
                 : "r"(a)
                 : "memory");
}
__device__ __forceinline__ unsigned long long dsmem_ld_u64(uint32_t a) {
    unsigned long long v;
    asm volatile("ld.shared::cluster.u64 %0, [%1];" : "=l"(v) : "r"(a) : "memory");
    return v;
}

__device__ __forceinline__ void warp_inclusive_scan_u64(unsigned long long& x) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
}

}  // namespace

template <int NT, int NV>
__host__ __device__ constexpr size_t ctl_offset() {
    // staging D, T: NV*NT uint4 each | one barrier per warp
    return (static_cast<size_t>(NV) * NT * 16 * 2 + static_cast<size_t>(NT / 32) * 8 + 127) &
           ~static_cast<size_t>(127);
}

template <int NT, int NV, int MINB, bool DISTILL, bool STOCH, bool ALIGNED>
__global__ void __launch_bounds__(NT, MINB) row_pass_kernel(const RowParams p) {
    constexpr int NW = NT / 32;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    uint4* stageD = reinterpret_cast<uint4*>(smem_raw);
    uint4* stageT = stageD + NV * NT;
    uint64_t* full = reinterpret_cast<uint64_t*>(stageT + NV * NT);
    Ctl<NW>& c = *reinterpret_cast<Ctl<NW>*>(smem_raw + ctl_offset<NT, NV>());
    // compact mode: b_k [B] and the prefixes of loaded and zero rows [B + 1] each follow the
    // control block
    int* sbk = reinterpret_cast<int*>(smem_raw + ctl_offset<NT, NV>() + ((sizeof(Ctl<NW>) + 15) & ~size_t(15)));
    int* spre = sbk + p.B;
    int* zpre = spre + p.B + 1;

    // the finalize pass may be scheduled as soon as SM resources allow; it waits for this grid
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const uint32_t rank = cluster_rank();
    const int CL = static_cast<int>(cluster_size());
    const int cid = static_cast<int>(cluster_id_x());
    const int ncl = static_cast<int>(num_clusters_x());
    const bool verify = (p.flags & kFlagVerify) != 0;
    const int V = p.V, k = p.k, kt = p.kt;
    const int v0 = static_cast<int>(rank) * p.chunk;
    const int len = max(0, min(p.chunk, V - v0));
    const int nvec = (len + 7) >> 3;
    // this warp's contiguous run of vectors: [wv0, wv0 + wcnt), at most 32 * NV
    const int vpw = (nvec + NW - 1) / NW;
    const int wv0 = min(nvec, warp * vpw);
    const int wcnt = max(0, min(nvec, wv0 + vpw) - wv0);
    const float k2 = p.k2, itau = p.inv_tau;
    uint4* myD = stageD + warp * NV * 32;
    uint4* myT = stageT + warp * NV * 32;

    // ---------------------------------------------------------------- prologue
    if (t == 0) {
        for (int q = 0; q < NW; ++q) mbar_init(&full[q], 1);
        fence_mbar_init();
        for (int q = 0; q < 2; ++q) {
            c.dep[q].argD = kNone;
            c.dep[q].argT = kNone;
            c.dep[q].tok = kNone;
            c.dep[q].ce = 0.f;
        }
    }
    // Vectors past the end of a warp's run hold a finite sentinel (the most negative bf16) in
    // both D and T: its exp is 0 and D - T is 0, so the passes run straight-line code over all
    // NV rounds with no per-vector branches.  The bulk copies never touch this tail.
    {
        const uint4 sent = make_uint4(0xFF7FFF7Fu, 0xFF7FFF7Fu, 0xFF7FFF7Fu, 0xFF7FFF7Fu);
        for (int lv = wcnt + lane; lv < NV * 32; lv += 32) {
            myD[lv] = sent;
            myT[lv] = sent;
        }
    }
    __syncthreads();
    // behind the length head (programmatic dependent launch) the prologue above overlapped its
    // tail; b_k is read only after the head's writes are visible
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const bool compact = p.B <= kCompactMaxB;
    if (compact) {
        // b_k and the exclusive prefix of loaded rows per sequence, in shared memory
        int carry = 0, carryz = 0;
        for (int c0 = 0; c0 < p.B; c0 += NT) {
            const int b = c0 + t;
            int n = 0, L = 0, Z = 0;
            if (b < p.B) {
                n = clamp_bk(p, __ldg(p.bk + b));
                L = loaded_rows(n, kt, verify);
                Z = DISTILL ? zero_rows(k, n, verify) : 0;
                sbk[b] = n;
            }
            int incl = L, inclz = Z;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                const int yz = __shfl_up_sync(0xffffffffu, inclz, o);
                if (lane >= o) { incl += y; inclz += yz; }
            }
            if (lane == 31) { c.wscan[warp] = incl; c.wscanz[warp] = inclz; }
            __syncthreads();
            int before = 0, tot = 0, beforez = 0, totz = 0;
            for (int q = 0; q < NW; ++q) {
                const int v = c.wscan[q], vz = c.wscanz[q];
                if (q < warp) { before += v; beforez += vz; }
                tot += v;
                totz += vz;
            }
            if (b < p.B) {
                spre[b] = carry + before + incl - L;
                zpre[b] = carryz + beforez + inclz - Z;
            }
            carry += tot;
            carryz += totz;
            __syncthreads();
        }
        if (t == 0) {
            spre[p.B] = carry;
            zpre[p.B] = carryz;
            // the cluster's first loaded item
            if (rank == 0) c.next_w[0] = static_cast<int>(atomicAdd(&p.hdr->item_ticket, 1u));
        }
    }
    __syncthreads();
    cluster_sync();  // barriers, deposit slots and the item list ready everywhere

    const BkView bkv{compact ? sbk : nullptr, p.bk};
    const int* list = compact ? spre : nullptr;
    const int nslots = loaded_slots(p, list);
    // Compact mode: rank 0 takes the cluster's loaded items one at a time from the workspace
    // ticket, one row ahead, and every warp reads the index from rank 0 over DSMEM (slot by row
    // parity: written before barrier #1 of one row, read after it, rewritten two rows later).
    // Otherwise the cluster's items are slots cid, cid + ncl, ...; holes are skipped.
    auto shared_item = [&](int slot) -> int {
        int wv = 0;
        if (lane == 0) wv = static_cast<int>(dsmem_ld_u32(dsmem_map(&c.next_w[slot], 0)));
        return __shfl_sync(0xffffffffu, wv, 0);
    };
    auto next_loaded = [&](int& w) -> Item {
        while (w < nslots) {
            const Item it = decode_loaded(p, list, bkv, w, verify);
            if (it.kind != kItemNone) return it;
            w += ncl;
        }
        return Item{kItemNone, -1, -1};
    };

    // one warp's bulk copies of item `it` into its staging run (lane 0 only)
    auto issue_loads = [&](const Item& it) {
        const uint32_t bT = static_cast<uint32_t>(wcnt) * 16u;
        const uint32_t bD = (it.kind == kItemRow) ? bT : 0u;
        mbar_arrive_expect_tx(&full[warp], bD + bT);
        if (bT) {
            const size_t e0 = static_cast<size_t>(v0) + static_cast<size_t>(wv0) * 8;
            if (bD) bulk_load(myD, p.D + (static_cast<size_t>(it.b) * k + it.i) * V + e0, bD, &full[warp]);
            bulk_load(myT, p.T + (static_cast<size_t>(it.b) * kt + it.i) * V + e0, bT, &full[warp]);
        }
    };

    int w = compact ? shared_item(0) : cid;
    Item cur = compact ? decode_loaded(p, list, bkv, w, verify) : next_loaded(w);
    if (ALIGNED && lane == 0 && cur.kind != kItemNone) issue_loads(cur);
    int iter = 0;                // loaded rows done by this cluster (parity of next_w)
    uint32_t phase = 0;          // parity of this warp's staging barrier
    bool wait_dead = false;      // a bounded wait ran out: skip later waits so the kernel ends
    int par = 0;                 // parity of the loaded rows (deposit double buffer)
    bool pending = false;        // rank 0 owes the record of the previous loaded row

    // rank 0, warp NW-1: write the record of the previous loaded row (its deposits are visible)
    auto write_record = [&]() {
        if (lane != 0) return;
        const Pending& pd = c.pend;
        Deposit& dp = c.dep[par ^ 1];
        const bool isRow = pd.kind == kItemRow;
        svd_row_info r;
        r.draft_token = pd.x;
        r.target_argmax = pd.y;
        r.accepted = pd.acc;
        if (!verify) r.sample_token = -1;
        else if (!STOCH) r.sample_token = pd.y;
        else r.sample_token = (pd.do_sample && dp.tok != kNone) ? static_cast<int32_t>(dp.tok) : -1;
        r.ratio = pd.ratio;
        r.lse_draft = pd.lseD;
        r.lse_target = pd.lseT;
        float L = 0.f;
        if (DISTILL && isRow) {
            L = p.lambda * dp.ce + (1.f - p.lambda) * pd.kc;
            if (p.loss_rows) p.loss_rows[static_cast<size_t>(pd.b) * k + pd.i] = L;
        }
        r.loss = L;
        const size_t trow = static_cast<size_t>(pd.b) * kt + pd.i;
        p.rec[trow] = r;
        if (p.row_info) p.row_info[trow] = r;
        dp.argD = kNone;
        dp.argT = kNone;
        dp.tok = kNone;
        dp.ce = 0.f;
    };

    // ---------------------------------------------------------------- loaded rows
    while (cur.kind != kItemNone) {
        int wn = w + ncl;
        Item nxt{kItemNone, -1, -1};
        if (!compact) nxt = next_loaded(wn);
        // rank 0 asks for the next item now; the answer is stored before barrier #1
        int fetched = 0;
        if (compact && rank == 0 && t == 0) fetched = static_cast<int>(atomicAdd(&p.hdr->item_ticket, 1u));
        const int b = cur.b, i = cur.i;
        const size_t drow = static_cast<size_t>(b) * k + i;      // draft / gradient row
        const size_t trow = static_cast<size_t>(b) * kt + i;     // target row
        const bool isRow = (cur.kind == kItemRow);
        const bool rowVerify = isRow && verify;
        // exps are needed for distillation rows and for stochastic sampling
        const bool need_lse = (DISTILL && isRow) || STOCH;

        // caller's draft token and, in stochastic mode, D_x and T_x for the acceptance ratio
        uint32_t x = kNone;
        float Dx = 0.f, Tx = 0.f;
        if (rowVerify && p.draft != nullptr) {
            int xv = 0;
            if (lane == 0) {
                xv = __ldg(p.draft + drow);
                if (xv < 0 || xv >= V) {
                    if (warp == 0) set_device_error(&p.hdr->status, SVD_ERR_TOKEN_RANGE);
                    xv = -1;
                } else if (STOCH) {
                    Dx = __uint_as_float(static_cast<uint32_t>(__ldg(p.D + drow * V + xv)) << 16);
                    Tx = __uint_as_float(static_cast<uint32_t>(__ldg(p.T + trow * V + xv)) << 16);
                }
            }
            xv = __shfl_sync(0xffffffffu, xv, 0);
            Dx = __shfl_sync(0xffffffffu, Dx, 0);
            Tx = __shfl_sync(0xffffffffu, Tx, 0);
            x = xv < 0 ? kNone : static_cast<uint32_t>(xv);
        }

        // -------------------------------------------------------- staging
        if (ALIGNED) {
            if (!wait_dead && !mbar_wait_bounded(&full[warp], phase, p.wait_limit_ns)) {
                wait_dead = true;
                set_device_error(&p.hdr->status, SVD_ERR_TIMEOUT);
            }
            phase ^= 1u;
        } else {
            // plain loads; elements past the row end read as the sentinel
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                const int lv = j * 32 + lane;
                if (lv < wcnt) {
                    uint16_t dv[8], tv[8];
                    const int base = v0 + (wv0 + lv) * 8;
#pragma unroll
                    for (int l = 0; l < 8; ++l) {
                        const bool ok = base + l < V && (wv0 + lv) * 8 + l < len;
                        dv[l] = ok && isRow ? __ldg(p.D + drow * V + base + l) : (uint16_t)0xFF7Fu;
                        tv[l] = ok ? __ldg(p.T + trow * V + base + l) : (uint16_t)0xFF7Fu;
                    }
                    myD[lv] = make_uint4(dv[0] | (uint32_t(dv[1]) << 16), dv[2] | (uint32_t(dv[3]) << 16),
                                         dv[4] | (uint32_t(dv[5]) << 16), dv[6] | (uint32_t(dv[7]) << 16));
                    myT[lv] = make_uint4(tv[0] | (uint32_t(tv[1]) << 16), tv[2] | (uint32_t(tv[3]) << 16),
                                         tv[4] | (uint32_t(tv[5]) << 16), tv[6] | (uint32_t(tv[7]) << 16));
                }
            }
            __syncwarp();
        }

        // -------------------------------------------------------- pass A
        // pre-pass: this thread's maxima (exact bf16 compares) and the first vector holding each
        float RD = kNegInf, RT = kNegInf;
        int bjD = 0, bjT = 0;
#pragma unroll
        for (int j = 0; j < NV; ++j) {
            const float mT = max8_bf16(myT[j * 32 + lane]);
            const bool upT = mT > RT;
            RT = upT ? mT : RT;
            bjT = upT ? j : bjT;
            if (isRow) {
                const float mD = max8_bf16(myD[j * 32 + lane]);
                const bool upD = mD > RD;
                RD = upD ? mD : RD;
                bjD = upD ? j : bjD;
            }
        }
        // argmax candidates: the first element equal to the thread maximum in that vector
        uint32_t candD = kNone, candT = kNone;
        {
            float xv[8];
            unpack8(myT[bjT * 32 + lane], xv);
            int l = 0;
            while (l < 7 && xv[l] != RT) ++l;
            candT = static_cast<uint32_t>(v0 + (wv0 + bjT * 32 + lane) * 8 + l);
        }
        if (rowVerify && p.draft == nullptr) {
            float xv[8];
            unpack8(myD[bjD * 32 + lane], xv);
            int l = 0;
            while (l < 7 && xv[l] != RD) ++l;
            candD = static_cast<uint32_t>(v0 + (wv0 + bjD * 32 + lane) * 8 + l);
        }
        // main pass: exp relative to the thread maxima (no rescaling) and the reverse-KL moment;
        // straight-line over all rounds (sentinel vectors contribute exact zeros).  A thread
        // holding sentinels only keeps a zero reference.
        float emax[NV];
        float sD = 0.f, sDd = 0.f, sT = 0.f, dmax = kNegInf;
        const float AD = RD > -1e38f ? RD * k2 : 0.f, AT = RT > -1e38f ? RT * k2 : 0.f;
#pragma unroll
        for (int j = 0; j < NV; ++j) {
            emax[j] = 0.f;
            if (!need_lse) continue;
            const int lv = j * 32 + lane;
            float xt[8], et[8];
            unpack8(myT[lv], xt);
#pragma unroll
            for (int l = 0; l < 8; ++l) et[l] = fast_exp2(fmaf(xt[l], k2, -AT));
            sT += sum8(et);
            if (isRow) {
                float xd[8], ed[8], dd[8];
                unpack8(myD[lv], xd);
#pragma unroll
                for (int l = 0; l < 8; ++l) {
                    ed[l] = fast_exp2(fmaf(xd[l], k2, -AD));
                    dd[l] = xd[l] - xt[l];
                }
                sD += sum8(ed);
                float a0 = ed[0] * dd[0], a1 = ed[1] * dd[1];
                a0 = fmaf(ed[2], dd[2], a0); a1 = fmaf(ed[3], dd[3], a1);
                a0 = fmaf(ed[4], dd[4], a0); a1 = fmaf(ed[5], dd[5], a1);
                a0 = fmaf(ed[6], dd[6], a0); a1 = fmaf(ed[7], dd[7], a1);
                sDd += a0 + a1;
                if (DISTILL) {
                    dmax = fmaxf(dmax, max8f(dd));
                    emax[j] = max8f(ed);
                }
            }
        }

        // reduction #1: warp -> CTA (local shared memory) -> cluster (one DSMEM load per rank)
        {
            Part1 a;
            a.mD = RD; a.sD = sD; a.sDd = sDd; a.dmax = dmax; a.mT = RT; a.sT = sT;
            a.pad0 = a.pad1 = 0.f;
            const Part1 r = warp_reduce_part1(a, k2);
            if (lane == 0) c.p1[warp] = r;
        }
        __syncthreads();
        if (warp == 0) {
            const Part1 a = lane < NW ? c.p1[lane] : empty_part1();
            const Part1 r = warp_reduce_part1(a, k2);
            if (lane == 0) c.cta1 = r;
        }
        if (compact && rank == 0 && t == 0) c.next_w[(iter + 1) & 1] = fetched;
        cluster_sync();  // #1
        if (compact) {
            wn = shared_item((iter + 1) & 1);
            nxt = decode_loaded(p, list, bkv, wn, verify);
        }

        // ------------------------------------------------ row statistics (every warp)
        float MD, MT, lseD = kQNaN, lseT = kQNaN, L2D = 0.f, L2T = 0.f, dl = 0.f, rkl = 0.f, smax = 0.f;
        {
            Part1 a = empty_part1();
            if (lane < CL) {
                const uint32_t ad = dsmem_map(&c.cta1, lane);
                float v[4], u[4];
                dsmem_ld4(ad, v);
                dsmem_ld4(ad + 16, u);
                a.mD = v[0]; a.sD = v[1]; a.sDd = v[2]; a.dmax = v[3]; a.mT = u[0]; a.sT = u[1];
            }
            const Part1 r = warp_reduce_part1(a, k2);   // identical in every lane, warp and rank
            MD = r.mD;
            MT = r.mT;
            if (need_lse) {
                if (isRow) lseD = r.mD * itau + logf(r.sD);
                lseT = r.mT * itau + logf(r.sT);
                L2D = lseD * kLog2e;
                L2T = lseT * kLog2e;
                dl = lseD - lseT;
                if (isRow) {
                    rkl = (r.sDd / r.sD) * itau - dl;   // sum_v q_v (log q_v - log p_v)
                    smax = r.dmax * itau - dl;          // largest log q_v - log p_v
                }
            }
        }
        // rank 0 writes the previous row's record while the rest of the cluster works
        if (pending && rank == 0 && warp == NW - 1) write_record();
        pending = false;

        // stochastic decision (every warp computes the same value)
        float ratio = kQNaN, u1 = 0.f;
        int acc = 0, do_sample = 0;
        if (STOCH) {
            const PhiloxOut ph = philox_words(p.seed, p.step, static_cast<uint32_t>(b),
                                              static_cast<uint32_t>(i));
            const float u0 = uniform24(ph.w[0]);
            u1 = uniform24(ph.w[1]);
            if (rowVerify) {
                if (x != kNone) {
                    ratio = fast_exp2((dl - (Dx - Tx) * itau) * kLog2e);
                    acc = u0 < fminf(1.f, ratio) ? 1 : 0;
                } else {
                    ratio = 0.f;
                    acc = 0;
                }
                do_sample = acc ? 0 : 1;
            } else if (!isRow) {
                do_sample = 1;  // bonus row: sample from p
            }
        }

        // lazy argmax: only the threads holding the row maximum offer their candidate
        Deposit* dep0 = &c.dep[par];
        if (candD != kNone && RD == MD) dsmem_min_u32(dsmem_map(&dep0->argD, 0), candD);
        if (RT == MT) dsmem_min_u32(dsmem_map(&dep0->argT, 0), candT);

        // -------------------------------------------------------- pass B
        // d_v = q_v s_v <= q_v s_max, so only entries with q_v > c / s_max can be clipped; those
        // vectors alone are re-read and tested exactly
        float clip_d = 0.f, clip_q = 0.f, n_clip = 0.f;
        uint32_t clipmask = 0;
        const float cc = p.clip_c;
        if (DISTILL && isRow && isfinite(cc) && smax > 0.f) {
            const float fD = fast_exp2(AD - L2D);          // q = e * fD for this thread's exps
            const float qthr = (cc / smax) * 0.9999f;
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                if (emax[j] * fD > qthr) {
                    clipmask |= 1u << j;
                    float xd[8], xt[8];
                    unpack8(myD[j * 32 + lane], xd);
                    unpack8(myT[j * 32 + lane], xt);
#pragma unroll
                    for (int l = 0; l < 8; ++l) {
                        const float q = elem_q(xd[l], k2, L2D);
                        const float d = elem_d(q, elem_s(xd[l], xt[l], itau, dl));
                        if (d > cc) { clip_d += d; clip_q += q; n_clip += 1.f; }
                    }
                }
            }
        }
        // stochastic rows: sample masses (residual max(0, p - q) of a rejected row, p of a bonus row)
        unsigned long long vmass[NV];
#pragma unroll
        for (int j = 0; j < NV; ++j) vmass[j] = 0ull;
        unsigned long long wmass = 0ull;
        if (STOCH && do_sample) {
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                float xt[8];
                unpack8(myT[j * 32 + lane], xt);
                unsigned long long ms = 0ull;
                if (isRow) {
                    float xd[8];
                    unpack8(myD[j * 32 + lane], xd);
#pragma unroll
                    for (int l = 0; l < 8; ++l)
                        ms += to_fixed(fmaxf(__fsub_rn(elem_p(xt[l], k2, L2T), elem_q(xd[l], k2, L2D)), 0.f));
                } else {
#pragma unroll
                    for (int l = 0; l < 8; ++l) ms += to_fixed(elem_p(xt[l], k2, L2T));
                }
                vmass[j] = ms;
                wmass += ms;
            }
            wmass = warp_sum_u64(wmass);
        }
        // reduction #2: warp -> CTA (fixed order) -> cluster
        if (DISTILL && isRow) {
            clip_d = warp_sum(clip_d);
            clip_q = warp_sum(clip_q);
            n_clip = warp_sum(n_clip);
        }
        if (lane == 0) {
            Part2 q2;
            q2.clip_d = clip_d; q2.clip_q = clip_q; q2.n_clip = n_clip; q2.pad0 = 0.f;
            q2.mass = wmass;
            q2.pad1 = 0ull;
            c.p2[warp] = q2;
        }
        __syncthreads();
        if (warp == 0) {
            float a0 = 0.f, a1 = 0.f, a2 = 0.f;
            unsigned long long m = 0ull;
            if (lane < NW) {
                const Part2 q = c.p2[lane];
                a0 = q.clip_d; a1 = q.clip_q; a2 = q.n_clip; m = q.mass;
            }
            unsigned long long incl = m;
            warp_inclusive_scan_u64(incl);
            if (lane < NW) c.wpre[lane] = incl - m;
            a0 = warp_sum(a0);
            a1 = warp_sum(a1);
            a2 = warp_sum(a2);
            const unsigned long long tot = __shfl_sync(0xffffffffu, incl, 31);
            if (lane == 0) {
                Part2 q2;
                q2.clip_d = a0; q2.clip_q = a1; q2.n_clip = a2; q2.pad0 = 0.f;
                q2.mass = tot;
                q2.pad1 = 0ull;
                c.cta2 = q2;
            }
        }
        cluster_sync();  // #2

        // ------------------------------------------------ row results (every warp)
        float kc = 0.f, P = 0.f, Q = 0.f, Pc = 0.f, hardc = 0.f;
        unsigned long long R = 0ull, before = 0ull;
        {
            float a0 = 0.f, a1 = 0.f, a2 = 0.f;
            unsigned long long m = 0ull;
            if (lane < CL) {
                const uint32_t a = dsmem_map(&c.cta2, lane);
                float v[4];
                dsmem_ld4(a, v);
                a0 = v[0]; a1 = v[1]; a2 = v[2];
                m = dsmem_ld_u64(a + offsetof(Part2, mass));
            }
            R = warp_sum_u64(m);
            before = warp_sum_u64(lane < static_cast<int>(rank) ? m : 0ull) + c.wpre[warp];
            if (DISTILL && isRow) {
                a0 = warp_sum(a0);
                a1 = warp_sum(a1);
                a2 = warp_sum(a2);
                // S = sum over unclipped entries of q (s + 1) = (rkl - clip_d) + (1 - clip_q)
                const float S = (rkl - a0) + (1.f - a1);
                kc = isfinite(cc) ? (rkl - a0) + cc * a2 : rkl;
                const float lam = p.lambda, pre = p.grad_scale * itau;
                P = pre * (lam + (1.f - lam) * (1.f - S - dl));
                Q = pre * (1.f - lam) * itau;
                Pc = pre * (lam - (1.f - lam) * S);
                hardc = pre * lam;
            }
        }
        uint32_t y = kNone;
        {
            const uint32_t a = dsmem_map(dep0, 0);
            uint32_t yv = 0, xv = 0;
            if (lane == 0) {
                yv = dsmem_ld_u32(a + offsetof(Deposit, argT));
                if (rowVerify && p.draft == nullptr) xv = dsmem_ld_u32(a + offsetof(Deposit, argD));
            }
            y = __shfl_sync(0xffffffffu, yv, 0);
            if (rowVerify && p.draft == nullptr) x = __shfl_sync(0xffffffffu, xv, 0);
        }
        if (rowVerify && !STOCH) acc = (x == y) ? 1 : 0;

        // stochastic fallback: residual mass zero -> sample from p (rare; one more reduction)
        bool use_p = false;
        if (STOCH && do_sample && R == 0ull && isRow) {
            use_p = true;
            wmass = 0ull;
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                float xt[8];
                unpack8(myT[j * 32 + lane], xt);
                unsigned long long ms = 0ull;
#pragma unroll
                for (int l = 0; l < 8; ++l) ms += to_fixed(elem_p(xt[l], k2, L2T));
                vmass[j] = ms;
                wmass += ms;
            }
            wmass = warp_sum_u64(wmass);
            if (lane == 0) c.p2[warp].mass = wmass;
            __syncthreads();
            if (warp == 0) {
                const unsigned long long m = lane < NW ? c.p2[lane].mass : 0ull;
                unsigned long long incl = m;
                warp_inclusive_scan_u64(incl);
                if (lane < NW) c.wpre[lane] = incl - m;
                const unsigned long long tot = __shfl_sync(0xffffffffu, incl, 31);
                if (lane == 0) c.cta3.mass = tot;
            }
            cluster_sync();
            const unsigned long long m =
                lane < CL ? dsmem_ld_u64(dsmem_map(&c.cta3, lane) + offsetof(Part2, mass)) : 0ull;
            R = warp_sum_u64(m);
            before = warp_sum_u64(lane < static_cast<int>(rank) ? m : 0ull) + c.wpre[warp];
        }

        // -------------------------------------------------------- sample search
        if (STOCH && do_sample && R > 0ull) {
            const unsigned long long tgt = scale_mass(R, static_cast<uint32_t>(u1 * 16777216.0f));
            unsigned long long run = before;   // mass before this lane's vector, id order
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                unsigned long long incl = vmass[j];
                warp_inclusive_scan_u64(incl);
                const unsigned long long lo = run + incl - vmass[j];
                run += __shfl_sync(0xffffffffu, incl, 31);
                if (j * 32 + lane < wcnt && vmass[j] > 0ull && lo <= tgt && tgt - lo < vmass[j]) {
                    // the sample point lies in this vector: walk its 8 masses in id order
                    const unsigned long long rel = tgt - lo;
                    unsigned long long cum = 0ull;
                    int pick = -1;
                    float xt[8];
                    unpack8(myT[j * 32 + lane], xt);
                    if (isRow) {
                        float xd[8];
                        unpack8(myD[j * 32 + lane], xd);
#pragma unroll
                        for (int l = 0; l < 8; ++l) {
                            const float pv = elem_p(xt[l], k2, L2T);
                            cum += use_p ? to_fixed(pv) : to_fixed(fmaxf(__fsub_rn(pv, elem_q(xd[l], k2, L2D)), 0.f));
                            if (pick < 0 && cum > rel) pick = l;
                        }
                    } else {
#pragma unroll
                        for (int l = 0; l < 8; ++l) {
                            cum += to_fixed(elem_p(xt[l], k2, L2T));
                            if (pick < 0 && cum > rel) pick = l;
                        }
                    }
                    if (pick < 0) pick = 7;
                    dsmem_min_u32(dsmem_map(&dep0->tok, 0),
                                  static_cast<uint32_t>(v0 + (wv0 + j * 32 + lane) * 8 + pick));
                }
            }
        }

        // -------------------------------------------------------- pass C: gradient row
        if (DISTILL && isRow) {
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                const int lv = j * 32 + lane;
                float xd[8], xt[8], gv[8];
                unpack8(myD[lv], xd);
                unpack8(myT[lv], xt);
#pragma unroll
                for (int l = 0; l < 8; ++l) {
                    const float q = fast_exp2(fmaf(xd[l], k2, -L2D));
                    gv[l] = q * fmaf(Q, xd[l] - xt[l], P);
                }
                if (clipmask & (1u << j)) {
#pragma unroll
                    for (int l = 0; l < 8; ++l) {
                        const float q = elem_q(xd[l], k2, L2D);
                        const float d = elem_d(q, elem_s(xd[l], xt[l], itau, dl));
                        if (d > cc) gv[l] = q * Pc;
                    }
                }
                if (lv < wcnt) {
                    const int base = v0 + (wv0 + lv) * 8;
                    if (y >= static_cast<uint32_t>(base) && y < static_cast<uint32_t>(base + 8)) {
                        const int ly = static_cast<int>(y) - base;
                        float dy = xd[0];
#pragma unroll
                        for (int q = 1; q < 8; ++q) if (q == ly) dy = xd[q];
#pragma unroll
                        for (int q = 0; q < 8; ++q) if (q == ly) gv[q] -= hardc;
                        // -log q_y = lseD - D_y / tau
                        dsmem_st_f32(dsmem_map(&dep0->ce, 0), lseD - dy * itau);
                    }
                    if (ALIGNED) {
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
                            if (base + l < V && (wv0 + lv) * 8 + l < len) {
                                if (p.dl_fp32) static_cast<float*>(p.dlogits)[drow * V + base + l] = gv[l];
                                else static_cast<uint16_t*>(p.dlogits)[drow * V + base + l] =
                                    static_cast<uint16_t>(pack_bf16x2(gv[l], 0.f) & 0xffffu);
                            }
                        }
                    }
                }
            }
        } else if (DISTILL && !isRow && i < k) {
            // bonus row: its gradient row is zero
            if (ALIGNED) {
                const uint4 z = make_uint4(0, 0, 0, 0);
                if (p.dl_fp32) {
                    float* g = static_cast<float*>(p.dlogits) + drow * V + v0 + wv0 * 8;
                    for (int e2 = lane; e2 < wcnt * 2; e2 += 32) __stcs(reinterpret_cast<uint4*>(g) + e2, z);
                } else {
                    uint16_t* g = static_cast<uint16_t*>(p.dlogits) + drow * V + v0 + wv0 * 8;
                    for (int e2 = lane; e2 < wcnt; e2 += 32) __stcs(reinterpret_cast<uint4*>(g) + e2, z);
                }
            } else {
                const int e_end = min(len, (wv0 + wcnt) * 8);
                for (int e2 = wv0 * 8 + lane; e2 < e_end; e2 += 32) {
                    if (p.dl_fp32) static_cast<float*>(p.dlogits)[drow * V + v0 + e2] = 0.f;
                    else static_cast<uint16_t*>(p.dlogits)[drow * V + v0 + e2] = 0;
                }
            }
        }

        // this warp is done with its staging: start the next item's copies
        __syncwarp();
        if (ALIGNED && lane == 0 && nxt.kind != kItemNone) issue_loads(nxt);

        // rank 0 keeps this row's values; the record is written after the next cluster barrier
        if (rank == 0 && warp == NW - 1 && lane == 0) {
            Pending& pd = c.pend;
            pd.b = b; pd.i = i; pd.kind = cur.kind;
            pd.x = rowVerify ? (x == kNone ? -1 : static_cast<int>(x)) : -1;
            pd.y = static_cast<int>(y);
            pd.acc = rowVerify ? acc : -1;
            pd.do_sample = do_sample;
            pd.ratio = ratio;
            pd.lseD = isRow ? lseD : kQNaN;
            pd.lseT = lseT;
            pd.kc = kc;
        }
        pending = true;
        par ^= 1;
        cur = nxt;
        w = wn;
        ++iter;
    }
    if (pending) {  // uniform: every rank walked the same items
        cluster_sync();
        if (rank == 0 && warp == NW - 1) write_record();
    }

    // ---------------------------------------------------------------- zero-only gradient rows
    if (DISTILL && compact) {
        // quarters of the zero rows in the compact list, handed to CTAs one at a time (the next
        // unit is requested while the current one is written)
        const int units = zpre[p.B] * kZeroSplit;
        if (t == 0) c.zs = static_cast<int>(atomicAdd(&p.hdr->zero_ticket, 1u));
        __syncthreads();
        int u = c.zs;
        __syncthreads();
        while (u < units) {
            int nextu = 0;
            if (t == 0) nextu = static_cast<int>(atomicAdd(&p.hdr->zero_ticket, 1u));
            const int j = u / kZeroSplit, qq = u % kZeroSplit;
            int lo = 0, hi = p.B;  // largest b with zpre[b] <= j
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (zpre[mid] <= j) lo = mid; else hi = mid;
            }
            const int i = first_zero_row(sbk[lo], verify) + (j - zpre[lo]);
            const size_t drow = static_cast<size_t>(lo) * k + i;
            if (ALIGNED) {
                const uint4 zz = make_uint4(0, 0, 0, 0);
                const int per_elem = p.dl_fp32 ? 2 : 1;       // 16-byte stores per 8 ids
                const int nv = (V / 8) * per_elem;
                const int a0 = static_cast<int>(static_cast<long long>(nv) * qq / kZeroSplit);
                const int a1 = static_cast<int>(static_cast<long long>(nv) * (qq + 1) / kZeroSplit);
                uint4* g = p.dl_fp32 ? reinterpret_cast<uint4*>(static_cast<float*>(p.dlogits) + drow * V)
                                     : reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.dlogits) + drow * V);
                for (int e = a0 + t; e < a1; e += NT) __stcs(g + e, zz);
            } else {
                const int a0 = static_cast<int>(static_cast<long long>(V) * qq / kZeroSplit);
                const int a1 = static_cast<int>(static_cast<long long>(V) * (qq + 1) / kZeroSplit);
                for (int e = a0 + t; e < a1; e += NT) {
                    if (p.dl_fp32) static_cast<float*>(p.dlogits)[drow * V + e] = 0.f;
                    else static_cast<uint16_t*>(p.dlogits)[drow * V + e] = 0;
                }
            }
            if (t == 0) c.zs = nextu;
            __syncthreads();
            u = c.zs;
            __syncthreads();
        }
    } else if (DISTILL) {
        for (int z = cid; z < p.B * k; z += ncl) {
            const int b = z / k, i = z % k;
            if (!zero_row_pred(k, bkv(p, b), i, verify)) continue;
            const size_t drow = static_cast<size_t>(b) * k + i;
            if (ALIGNED) {
                const uint4 zz = make_uint4(0, 0, 0, 0);
                if (p.dl_fp32) {
                    float* g = static_cast<float*>(p.dlogits) + drow * V + v0 + wv0 * 8;
                    for (int e = lane; e < wcnt * 2; e += 32) __stcs(reinterpret_cast<uint4*>(g) + e, zz);
                } else {
                    uint16_t* g = static_cast<uint16_t*>(p.dlogits) + drow * V + v0 + wv0 * 8;
                    for (int e = lane; e < wcnt; e += 32) __stcs(reinterpret_cast<uint4*>(g) + e, zz);
                }
            } else {
                const int e_end = min(len, (wv0 + wcnt) * 8);
                for (int e = wv0 * 8 + lane; e < e_end; e += 32) {
                    if (p.dl_fp32) static_cast<float*>(p.dlogits)[drow * V + v0 + e] = 0.f;
                    else static_cast<uint16_t*>(p.dlogits)[drow * V + v0 + e] = 0;
                }
            }
        }
    }
    // no CTA leaves while another may still read its shared memory
    cluster_sync();
}

// ------------------------------------------------------------------------------------------
// finalize: per sequence, the acceptance scan over its row records (one lane per position),
// the emitted tokens, the loss rows past b_k and the sequence loss; the last CTA adds the
// sequence losses in sequence order.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) finalize_kernel(const RowParams p) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __shared__ int last;
    // the row pass has finished: its work tickets go back to zero for the next call
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        p.hdr->item_ticket = 0u;
        p.hdr->zero_ticket = 0u;
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const bool verify = (p.flags & kFlagVerify) != 0;
    const bool distill = (p.flags & kFlagDistill) != 0;
    const int k = p.k, kt = p.kt;
    const int b = blockIdx.x * 8 + warp;
    if (b < p.B) {
        int n = __ldg(p.bk + b);
        n = n < 1 ? 1 : (n > k ? k : n);   // the row pass already flagged out-of-range values
        svd_row_info r;
        r.draft_token = -1; r.target_argmax = -1; r.accepted = -1; r.sample_token = -1;
        r.ratio = r.lse_draft = r.lse_target = kQNaN;
        r.loss = 0.f;
        auto is_processed = [&](int row) { return row < n || (verify && row == n && n < kt); };
        if (lane < kt && is_processed(lane)) {
            const svd_row_info* src = p.rec + static_cast<size_t>(b) * kt + lane;
            r.draft_token = src->draft_token;
            r.target_argmax = src->target_argmax;
            r.accepted = src->accepted;
            r.sample_token = src->sample_token;
            r.loss = src->loss;
        } else if (lane < kt && p.row_info) {
            p.row_info[static_cast<size_t>(b) * kt + lane] = r;  // unprocessed row
        }
        if (kt == 33 && lane == 0 && !is_processed(32) && p.row_info) {
            svd_row_info u;
            u.draft_token = u.target_argmax = u.accepted = u.sample_token = -1;
            u.ratio = u.lse_draft = u.lse_target = kQNaN;
            u.loss = 0.f;
            p.row_info[static_cast<size_t>(b) * kt + 32] = u;
        }
        if (verify) {
            const uint32_t accm = __ballot_sync(0xffffffffu, lane < n && r.accepted == 1);
            int a = __ffs(~accm) - 1;
            if (a > n || a < 0) a = n;
            const int fix_row = a < n ? a : ((n < kt) ? n : -1);
            int fix_tok = __shfl_sync(0xffffffffu, r.sample_token, fix_row < 0 ? 0 : (fix_row & 31));
            if (fix_row >= 32)  // bonus row 32 (k = 32, kt = 33) has no lane of its own
                fix_tok = p.rec[static_cast<size_t>(b) * kt + 32].sample_token;
            // lane q holds row q's record; slot k (= 32 at most) can only hold the fix token
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
        if (distill) {
            if (p.loss_rows && lane >= n && lane < k) p.loss_rows[static_cast<size_t>(b) * k + lane] = 0.f;
            float ls = 0.f;
            for (int q = 0; q < n; ++q) ls += __shfl_sync(0xffffffffu, r.loss, q);
            if (lane == 0) p.seq_loss[b] = ls;
        }
    }
    if (!distill) return;
    // the last CTA adds the sequence losses in sequence order
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t old = atomicAdd(&p.hdr->loss_ticket, 1u);
        last = (old + 1u == gridDim.x) ? 1 : 0;
    }
    __syncthreads();
    if (!last || threadIdx.x != 0) return;
    __threadfence();
    float tot = 0.f;
    for (int s = 0; s < p.B; ++s) tot += __ldcg(p.seq_loss + s);
    *p.loss_total = tot;
    p.hdr->loss_ticket = 0u;
}

// ------------------------------------------------------------------------------------------
// host side: geometry, occupancy, launch
// ------------------------------------------------------------------------------------------
namespace {

template <int NT, int NV>
constexpr size_t smem_fixed() {
    return ctl_offset<NT, NV>() + ((sizeof(Ctl<NT / 32>) + 15) & ~size_t(15));
}

using KernelFn = void (*)(RowParams);

template <int NT, int NV, int MINB, bool AL>
KernelFn pick_kernel3(int flags) {
    const bool dist = (flags & kFlagDistill) != 0, sto = (flags & kFlagStochastic) != 0;
    if (dist && sto) return row_pass_kernel<NT, NV, MINB, true, true, AL>;
    if (dist) return row_pass_kernel<NT, NV, MINB, true, false, AL>;
    if (sto) return row_pass_kernel<NT, NV, MINB, false, true, AL>;
    return row_pass_kernel<NT, NV, MINB, false, false, AL>;
}

template <int NT, int NV, int MINB>
KernelFn pick_kernel(int flags, bool aligned) {
    return aligned ? pick_kernel3<NT, NV, MINB, true>(flags) : pick_kernel3<NT, NV, MINB, false>(flags);
}

// Variants: (threads, vectors per lane, min CTAs per SM) -> ids per CTA = 8 * NT * NV.
constexpr int kSNT = 128, kSNV = 2, kSMB = 8;     //  2048 ids per CTA
constexpr int kMNT = 256, kMNV = 5, kMMB = 4;     // 10240 ids per CTA
constexpr int kLNT = 256, kLNV = 10, kLMB = 2;    // 20480 ids per CTA

int next_pow2(int x) {
    int r = 1;
    while (r < x) r <<= 1;
    return r;
}

}  // namespace

bool row_geometry(int V, RowGeometry* g) {
    if (V < 1) return false;
    const int capS = kSNT * kSNV * 8, capM = kMNT * kMNV * 8, capL = kLNT * kLNV * 8;
    if (V <= 8 * capS) {
        g->variant = 0; g->threads = kSNT;
        g->cluster = next_pow2((V + capS - 1) / capS);
        g->smem = smem_fixed<kSNT, kSNV>();
    } else if (V <= 16 * capM) {
        g->variant = 1; g->threads = kMNT;
        g->cluster = next_pow2((V + capM - 1) / capM);
        g->smem = smem_fixed<kMNT, kMNV>();
    } else {
        g->variant = 2; g->threads = kLNT;
        g->cluster = next_pow2((V + capL - 1) / capL);
        g->smem = smem_fixed<kLNT, kLNV>();
    }
    if (g->cluster > 16) return false;
    const int per = (V + g->cluster - 1) / g->cluster;
    g->chunk = (per + 7) & ~7;
    return true;
}

size_t row_smem_bytes(const RowGeometry& g, int B) {
    // compact mode: b_k [B], loaded-row prefix [B + 1], zero-row prefix [B + 1]
    const size_t list = B <= kCompactMaxB ? (static_cast<size_t>(3 * B + 2) * 4 + 15) & ~size_t(15) : 0;
    return g.smem + list;
}

int launch_row_pass(const RowParams& p, void* stream) {
    RowGeometry geo;
    if (!row_geometry(p.V, &geo)) return static_cast<int>(cudaErrorInvalidValue);
    const bool aligned = p.aligned != 0;
    KernelFn fn = geo.variant == 0 ? pick_kernel<kSNT, kSNV, kSMB>(p.flags, aligned)
                : geo.variant == 1 ? pick_kernel<kMNT, kMNV, kMMB>(p.flags, aligned)
                                   : pick_kernel<kLNT, kLNV, kLMB>(p.flags, aligned);
    const size_t smem = row_smem_bytes(geo, p.B);
    cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return static_cast<int>(err);
    if (geo.cluster > 8) {
        err = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (err != cudaSuccess) return static_cast<int>(err);
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = geo.cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (p.pdl) {
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.numAttrs = 2;
    }
    cfg.blockDim = dim3(geo.threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = static_cast<cudaStream_t>(stream);
    // persistent grid: as many clusters as can be resident at once (cached per configuration)
    static int cached_clusters[3][17][8][2] = {};
    static size_t cached_smem[3][17][8][2] = {};
    int& cache = cached_clusters[geo.variant][geo.cluster][p.flags & 7][aligned ? 1 : 0];
    size_t& csm = cached_smem[geo.variant][geo.cluster][p.flags & 7][aligned ? 1 : 0];
    if (cache == 0 || csm != smem) {
        int dev = 0, sms = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cfg.gridDim = dim3(geo.cluster * sms, 1, 1);
        int n = 0;
        err = cudaOccupancyMaxActiveClusters(&n, fn, &cfg);
        if (err != cudaSuccess || n < 1) {
            cudaGetLastError();
            n = sms / geo.cluster > 0 ? sms / geo.cluster : 1;
        }
        cache = n;
        csm = smem;
    }
    const long long max_items = static_cast<long long>(p.B) * (p.kt + p.k);
    int nclusters = cache;
    if (max_items < nclusters) nclusters = static_cast<int>(max_items > 0 ? max_items : 1);
    cfg.gridDim = dim3(geo.cluster * nclusters, 1, 1);
    RowParams q = p;
    q.chunk = geo.chunk;
    err = cudaLaunchKernelEx(&cfg, fn, q);
    if (err != cudaSuccess) return static_cast<int>(err);

    // finalize pass: one warp per sequence, launched as a programmatic dependent
    cudaLaunchConfig_t fc = {};
    cudaLaunchAttribute fattr[1];
    fattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    fattr[0].val.programmaticStreamSerializationAllowed = 1;
    fc.attrs = fattr;
    fc.numAttrs = 1;
    fc.blockDim = dim3(256, 1, 1);
    fc.gridDim = dim3((p.B + 7) / 8, 1, 1);
    fc.dynamicSmemBytes = 0;
    fc.stream = static_cast<cudaStream_t>(stream);
    err = cudaLaunchKernelEx(&fc, finalize_kernel, q);
    return static_cast<int>(err);
}

}  // namespace svd
