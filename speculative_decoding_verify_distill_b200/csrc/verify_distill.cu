// verify_distill.cu -- the fused row pass: truncated verification (greedy / stochastic) and the
// clipped reverse-KL + CE distillation loss with its gradient, one HBM read per logit row; the
// small finalize pass that turns per-row records into accepted lengths, emitted tokens and loss
// sums; and, in stochastic mode, the draw of each sequence's correction or bonus token.
//
// What it computes (AdaFlash; Pith review page "What carries the argument", Axiom & Free-
// Parameter Ledger, Referee Report major comment 2; Pith verdict record load_bearing_attack):
// for every sequence b the first b_k draft rows are verified against the target rows, the
// acceptance length a_b and the emitted tokens follow the standard speculative-decoding rule,
// and every verified row i < b_k also yields the OPD loss L_i and dL/dD_i; rows i >= b_k get a
// zero gradient row.
//
// Design (B200, sm_100a):
//   * A persistent grid of thread-block clusters (10 CTAs of 256 threads for a 151936-id
//     vocabulary, three CTAs per SM).  A cluster owns one logit row at a time; each CTA a
//     contiguous slice of the vocabulary; each warp a contiguous run of 16-byte vectors of the
//     slice.  Loaded work items (verified rows and bonus rows) form a compact list (prefix sums
//     of loaded rows per sequence) handed out one row at a time from a workspace ticket, so a
//     cluster that starts late (behind the length head, or beside other work) simply takes fewer
//     rows.  Zero-only gradient rows are handed to single CTAs in sixteenth-row units: one per
//     CTA while each row's exchange is in flight, the rest after the loaded rows.
//   * Each warp stages its run of D and T in shared memory with its own 1-D bulk copies
//     (cp.async.bulk, no multicast) on its own mbarrier.  The staged bf16 slice is the only copy:
//     every pass re-reads it, so a CTA holds no per-element state in registers and several CTAs
//     fit on one SM, each hiding the others' barrier and reduction latency.
//   * Pass A: a max pre-pass fixes each thread's exp reference, then exp of D and T, the tree
//     sums, the reverse-KL moment sum e(D - T) and max(D - T).  Reduction #1 (warp -> CTA ->
//     cluster over DSMEM) gives lse(D/tau), lse(T/tau) and the unclipped reverse-KL.
//   * Pass B: only entries with q > c / max(log q - log p) can be clipped; those vectors alone
//     are re-read and tested.  Argmax (lowest id) is resolved lazily by the threads holding the
//     row maximum.  Reduction #2 (only when some entry can be clipped).
//   * Pass C: dL/dD = q (P + Q (D - T)) with the clipped and hard-label corrections, q
//     recomputed from the staged logits, 16-byte streaming stores.
//   * Rank 0 writes the row record after the next cluster barrier; the finalize kernel runs the
//     warp-ballot acceptance scan per sequence and the fixed-order loss sums.
//   * Stochastic mode: a sequence emits one drawn token, from its first rejected row (residual
//     max(0, p - q)) or else its bonus row (p).  The row pass draws nothing; once the finalize
//     pass knows the emitted row, one cluster per sequence takes that row's sample masses as
//     2^-48 fixed-point integers (exact, associative prefix sums, so the split over CTAs does not
//     change the draw) and the CTA holding the Philox target searches its slice in id order.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <mutex>
#include <utility>
#include <vector>

#include "svd_device.cuh"
#include "svd_head_unit.cuh"

namespace svd {

namespace {

constexpr uint32_t kNone = 0xffffffffu;
#define kNegInf (-__int_as_float(0x7f800000))
#define kQNaN (__int_as_float(0x7fc00000))

enum ItemKind : int { kItemNone = 0, kItemRow = 1, kItemBonus = 2 };

// Messages of the per-row exchanges.  Every CTA of a cluster sends its message to every CTA
// (itself included) with st.async into the receiver's shared memory; the bytes complete the
// receiver's exchange barrier, so a CTA waits only for the data it needs and no cluster-wide
// barrier (with its release fence over the CTA's outstanding gradient stores) is taken per row.
// Sums travel relative to the maxima they come with (2^((x - m) k2), k2 = log2(e) / tau).
struct alignas(16) Msg1 {          // after pass A
    float mD, sD, sDd, dmax;        // max D, sum 2^((D - mD) k2), sum of those times (D - T), max (D - T)
    float mT, sT;                   // max T, sum 2^((T - mT) k2)
    uint32_t argT, argD;            // lowest id holding mT / mD in the sender's slice
    float prev_ce;                  // -log q_y of the previous row from the owner of y, else 0
    uint32_t next_item;             // rank 0: the cluster's next loaded item (packed)
    float Dx, Tx;                   // stochastic: D and T at the draft token from its owner, else 0
};
struct alignas(16) Msg2 {          // after pass B: clipped reverse-KL entries
    float clip_d, clip_q, n_clip, pad0;
};
static_assert(sizeof(Msg1) == 48 && sizeof(Msg2) == 16, "message sizes are multiples of 16 bytes");
// Row values rank 0 keeps until the record is written.
struct Pending {
    int b, i, kind;
    int x, y, acc;
    float ratio, lseD, lseT, kc;
};

template <int NW>
struct Ctl {
    Msg1 w1[NW];                    // per-warp partials (local)
    Msg2 w2[NW];
    Msg1 in1[2][16];                // exchange #1 by row parity and sender rank
    Msg2 in2[16];                   // exchange #2 by sender rank
    uint64_t x1[2], x2;             // exchange barriers
    uint64_t hbar;                  // length head inside the pass: its staging barrier
    float my_ce[2];                 // -log q_y computed in this CTA, by row parity
    Pending pend;
    int wscan[NW];                  // prologue scan of the loaded-row counts
    int wscanz[NW];                 // ... and of the zero-gradient row counts
    uint32_t first_raw[2];          // rank 0: the cluster's first loaded-item ticket (and a spare)
    int hunit, hflag;               // length head inside the pass: current unit, its ticket flag
    int list_flag;                  // the head has finished: build the compact lists
    int zs;                         // zero phase: the CTA's next unit
    int zu[2];                      // zero unit written while exchange #1 of a row is in flight
};

// Batches up to this size keep b_k and the prefixes of loaded and zero-gradient rows per sequence
// in shared memory (compact lists, handed out dynamically); larger batches walk the uncompacted
// (sequence, row) slots in a fixed order.
constexpr int kCompactMaxB = kRowCompactMaxB;

// Zero-gradient rows are handed out in sixteenths (about 19 KB of bf16 stores at V = 151936):
// one unit per CTA fills the wait for each row's exchange, the rest follow the loaded rows.
constexpr int kZeroSplit = 16;

struct Item {
    int kind, b, i;
};
// Items travel between CTAs as one word: (b << 8) | (i << 2) | kind; 0 means none.
__device__ __forceinline__ uint32_t pack_item(const Item& it) {
    return it.kind == kItemNone ? 0u
                                : (static_cast<uint32_t>(it.b) << 8) | (static_cast<uint32_t>(it.i) << 2) |
                                      static_cast<uint32_t>(it.kind);
}
__device__ __forceinline__ Item unpack_item(uint32_t v) {
    if ((v & 3u) == 0u) return Item{kItemNone, -1, -1};
    return Item{static_cast<int>(v & 3u), static_cast<int>(v >> 8), static_cast<int>((v >> 2) & 63u)};
}
__device__ __forceinline__ Msg1 empty_msg1() {
    Msg1 m;
    m.mD = m.mT = m.dmax = kNegInf;
    m.sD = m.sDd = m.sT = 0.f;
    m.argT = m.argD = kNone;
    m.prev_ce = 0.f;
    m.next_item = 0u;
    m.Dx = m.Tx = 0.f;
    return m;
}

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

// Rows sequence b verifies: all k in full-k mode, else its b_k (clamped).
__device__ __forceinline__ int load_bk(const RowParams& p, int b) {
    if (p.bk_const > 0) return p.bk_const;
    // b_k written by this grid's own head units is read through L2, not the read-only path
    return clamp_bk(p, p.head_fused ? __ldcg(p.bk + b) : __ldg(p.bk + b));
}
// b_k of sequence b: from shared memory (compact mode) or global memory.
struct BkView {
    const int* s;       // shared copy, or nullptr
    __device__ __forceinline__ int operator()(const RowParams& p, int b) const {
        return s ? s[b] : load_bk(p, b);
    }
};

// Loaded item w of the whole batch.  Compact mode: items 0 .. B-1 are row 0 of sequences
// 0 .. B-1, which every sequence verifies whatever its b_k (b_k >= 1), so they need no b_k;
// items from B on are the remaining loaded rows of each sequence in order (rows 1 .. b_k - 1 and
// the bonus row), from the prefix sums spre of (loaded rows - 1) per sequence (binary search).
// Otherwise w is a (sequence, row) slot and holes decode to kItemNone.
__device__ __forceinline__ Item decode_loaded(const RowParams& p, bool compact, const int* spre,
                                              const BkView& bkv, int w, bool verify) {
    Item it{kItemNone, -1, -1};
    if (compact) {
        if (w < p.B) return Item{kItemRow, w, 0};
        const int r = w - p.B;
        if (r >= spre[p.B]) return it;
        int lo = 0, hi = p.B;  // largest b with spre[b] <= r
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (spre[mid] <= r) lo = mid; else hi = mid;
        }
        const int i = 1 + (r - spre[lo]);
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

    // launched as a programmatic dependent of whatever kernel precedes it on the stream: its
    // CTAs may be resident early, but read nothing before that grid has finished (the previous
    // step's finalize pass resets this workspace's tickets)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // the finalize pass may be scheduled as soon as SM resources allow; it waits for this grid
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const uint32_t rank = cluster_rank();
    const int CL = static_cast<int>(cluster_size());
    const int cid = static_cast<int>(cluster_id_x());
    const int ncl = static_cast<int>(num_clusters_x());
    const bool verify = (p.flags & kFlagVerify) != 0;
    const bool greedy_x = verify && p.draft == nullptr;   // draft token = argmax of the draft row
    const int V = p.V, k = p.k, kt = p.kt;
    const int v0 = static_cast<int>(rank) * p.chunk;
    const int len = max(0, min(p.chunk, V - v0));
    const int nvec = (len + 7) >> 3;
    // this warp's contiguous run of vectors: [wv0, wv0 + wcnt), at most 32 * NV
    const int vpw = (nvec + NW - 1) / NW;
    const int wv0 = min(nvec, warp * vpw);
    const int wcnt = max(0, min(nvec, wv0 + vpw) - wv0);
    const float k2 = p.k2, itau = p.inv_tau, cc = p.clip_c;
    uint4* myD = stageD + warp * NV * 32;
    uint4* myT = stageT + warp * NV * 32;

    // ---------------------------------------------------------------- prologue
    if (t == 0) {
        for (int q = 0; q < NW; ++q) mbar_init(&full[q], 1);
        mbar_init(&c.x1[0], 1);
        mbar_init(&c.x1[1], 1);
        mbar_init(&c.x2, 1);
        mbar_init(&c.hbar, 1);
        fence_mbar_init();
        c.my_ce[0] = c.my_ce[1] = 0.f;
        c.first_raw[0] = c.first_raw[1] = 0u;
    }
    // Vectors past the end of a warp's run hold a finite sentinel (the most negative bf16) in
    // both D and T: its exp is 0 and D - T is 0, so the passes run straight-line code over all
    // NV rounds with no per-vector branches.  The bulk copies never touch this tail.  (With the
    // length head inside the pass, the staging area serves the head first; the tail is written
    // after it.)
    auto fill_sentinel = [&]() {
        const uint4 sent = make_uint4(0xFF7FFF7Fu, 0xFF7FFF7Fu, 0xFF7FFF7Fu, 0xFF7FFF7Fu);
        for (int lv = wcnt + lane; lv < NV * 32; lv += 32) {
            myD[lv] = sent;
            myT[lv] = sent;
        }
    };
    if (!p.head_fused) fill_sentinel();
    __syncthreads();
    const bool compact = p.B <= kCompactMaxB;
    // b_k and the exclusive prefixes of loaded rows past row 0 and of zero-gradient rows per
    // sequence, in shared memory (the whole CTA takes part).
    auto build_list = [&]() {
        int carry = 0, carryz = 0;
        for (int c0 = 0; c0 < p.B; c0 += NT) {
            const int b = c0 + t;
            int n = 0, L = 0, Z = 0;
            if (b < p.B) {
                n = load_bk(p, b);
                L = loaded_rows(n, kt, verify) - 1;
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
        }
        __syncthreads();
    };
    // With the length head inside this pass, the lists wait for its b_k (full-k mode verifies
    // every row and needs none).  Rows 0 need no list.
    const bool head_first = p.head_fused && p.bk_const == 0;
    bool list_ready = false;
    if (compact && !head_first) {
        build_list();
        list_ready = true;
    }
    // rank 0 takes the cluster's first loaded-item ticket
    if (compact && rank == 0 && t == 0) c.first_raw[0] = atomicAdd(&p.hdr->item_ticket, 1u);
    __syncthreads();
    cluster_sync();  // barriers, lists and the first ticket ready everywhere

    const BkView bkv{compact ? sbk : nullptr};
    const int nslots = p.B * p.kt;   // (sequence, row) slots of the uncompacted walk
    // Compact mode: rank 0 takes loaded items one at a time from the workspace ticket, one row
    // ahead, and passes each in its exchange message.  Otherwise the cluster's items are slots
    // cid, cid + ncl, ...; holes are skipped.
    auto next_loaded = [&](int& w) -> Item {
        while (w < nslots) {
            const Item it = decode_loaded(p, false, nullptr, bkv, w, verify);
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

    // gradient stores of one 8-id vector (lv: index in this warp's run) of row drow
    auto store_vec = [&](size_t drow, int lv, const float2 (&g)[4]) {
        const int base = v0 + (wv0 + lv) * 8;
        if (ALIGNED) {
            if (p.dl_fp32) {
                float4* o = reinterpret_cast<float4*>(static_cast<float*>(p.dlogits) + drow * V + base);
                __stcs(o, make_float4(g[0].x, g[0].y, g[1].x, g[1].y));
                __stcs(o + 1, make_float4(g[2].x, g[2].y, g[3].x, g[3].y));
            } else {
                uint4 pk;
                pk.x = pack_bf16x2(g[0].x, g[0].y);
                pk.y = pack_bf16x2(g[1].x, g[1].y);
                pk.z = pack_bf16x2(g[2].x, g[2].y);
                pk.w = pack_bf16x2(g[3].x, g[3].y);
                __stcs(reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.dlogits) + drow * V + base), pk);
            }
        } else {
            const float gl[8] = {g[0].x, g[0].y, g[1].x, g[1].y, g[2].x, g[2].y, g[3].x, g[3].y};
#pragma unroll
            for (int l = 0; l < 8; ++l) {
                if (base + l < V && (wv0 + lv) * 8 + l < len) {
                    if (p.dl_fp32) static_cast<float*>(p.dlogits)[drow * V + base + l] = gl[l];
                    else static_cast<uint16_t*>(p.dlogits)[drow * V + base + l] =
                        static_cast<uint16_t>(pack_bf16x2(gl[l], 0.f) & 0xffffu);
                }
            }
        }
    };
    auto store_elem = [&](size_t drow, int id, float g) {
        if (p.dl_fp32) static_cast<float*>(p.dlogits)[drow * V + id] = g;
        else static_cast<uint16_t*>(p.dlogits)[drow * V + id] = static_cast<uint16_t>(pack_bf16x2(g, 0.f) & 0xffffu);
    };

    // unit u of the compact zero-row list: a sixteenth of gradient row (b, i), i past b_k
    int zunits = (DISTILL && compact && list_ready) ? zpre[p.B] * kZeroSplit : 0;
    auto write_zero_unit = [&](int u) {
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
    };

    // Thread 0: whether the length head has written every b_k; with `block`, waits for it at most
    // the wait limit.  A wait that runs out records a timeout, and the lists are then built from
    // b_k as they stand (every value is clamped to [1, k], so no access leaves its row).
    auto head_finished = [&](bool block) -> bool {
        const uint32_t need = static_cast<uint32_t>(head_seq_tiles(p.head));
        if (ld_acquire_gpu(&p.hdr->head_done) >= need) return true;
        if (!block) return false;
        const uint64_t t0 = global_timer_ns();
        while (ld_acquire_gpu(&p.hdr->head_done) < need) {
            if (global_timer_ns() - t0 > p.wait_limit_ns) {
                set_device_error(&p.hdr->status, SVD_ERR_TIMEOUT);
                return true;
            }
            __nanosleep(256);
        }
        return true;
    };
    // The whole CTA: build the lists if the head has finished (with `block` from thread 0: once
    // it has).
    auto try_list = [&](bool block) {
        if (t == 0) c.list_flag = head_finished(block) ? 1 : 0;
        __syncthreads();
        if (c.list_flag) {
            build_list();
            list_ready = true;
            zunits = DISTILL ? zpre[p.B] * kZeroSplit : 0;
        }
    };

    bool wait_dead = false;      // a bounded wait ran out: skip later waits so the kernel ends
    // The length head's work units, taken from a ticket by whichever CTAs are running (no unit
    // waits for another, so the head finishes even if only part of the grid is resident), staged
    // through this CTA's (still idle) staging area before its first row uses it.
    if (p.head_fused) {
        const int U = head_units(p.head);
        uint32_t hphase = 0;
        while (true) {
            if (t == 0) c.hunit = static_cast<int>(atomicAdd(&p.hdr->head_unit, 1u));
            __syncthreads();
            const int u = c.hunit;
            __syncthreads();
            if (u >= U) break;
            if (!head_unit<NW>(p.head, u, &c.hflag, false, reinterpret_cast<uint16_t*>(stageD),
                               static_cast<size_t>(NV) * NT * 32, &c.hbar, hphase, p.wait_limit_ns))
                wait_dead = true;
        }
        fill_sentinel();
        __syncthreads();
    }

    Item cur{kItemNone, -1, -1};
    int w = cid;
    if (compact) {
        uint32_t v = 0;
        if (lane == 0) v = dsmem_ld_u32(dsmem_map(&c.first_raw[0], 0));
        const int raw0 = static_cast<int>(__shfl_sync(0xffffffffu, v, 0));
        // a row-0 item needs no list; a later one waits for the head's b_k
        if (raw0 >= p.B && !list_ready) try_list(true);
        cur = decode_loaded(p, true, spre, bkv, raw0, verify);
    } else {
        cur = next_loaded(w);
    }
    if (ALIGNED && lane == 0 && cur.kind != kItemNone) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // after the head's reads
        issue_loads(cur);
    }
    uint32_t phase = 0;          // parity of this warp's staging barrier
    int it = 0;                  // loaded rows done (row parity selects the exchange #1 buffers)
    uint32_t n2 = 0;             // completed phases of exchange barrier #2
    bool pending = false;        // rank 0 owes the record of the previous loaded row

    auto wait_x = [&](uint64_t* bar, uint32_t parity) {
        if (!wait_dead && !mbar_wait_cluster_bounded(bar, parity, p.wait_limit_ns)) {
            wait_dead = true;
            set_device_error(&p.hdr->status, SVD_ERR_TIMEOUT);
        }
    };
    // warp 0: message #1 (48 bytes) to every rank of the cluster, lane r -> rank r
    auto send1 = [&](const uint4& q0, const uint4& q1, const uint4& q2, int par) {
        if (lane < CL) {
            const uint32_t dst = dsmem_map(&c.in1[par][rank], static_cast<uint32_t>(lane));
            const uint32_t bar = dsmem_map(&c.x1[par], static_cast<uint32_t>(lane));
            st_async_v4(dst, q0, bar);
            st_async_v4(dst + 16, q1, bar);
            st_async_v4(dst + 32, q2, bar);
        }
    };
    // rank 0, one lane: the record of the previous loaded row
    // (stochastic rows: the one draw a sequence emits is made after the finalize pass)
    auto write_record = [&](float ce) {
        const Pending& pd = c.pend;
        svd_row_info r;
        r.draft_token = pd.x;
        r.target_argmax = pd.y;
        r.accepted = pd.acc;
        r.sample_token = (verify && !STOCH) ? pd.y : -1;
        r.ratio = pd.ratio;
        r.lse_draft = pd.lseD;
        r.lse_target = pd.lseT;
        float L = 0.f;
        if (DISTILL && pd.kind == kItemRow) {
            L = p.lambda * ce + (1.f - p.lambda) * pd.kc;
            if (p.loss_rows) p.loss_rows[static_cast<size_t>(pd.b) * k + pd.i] = L;
        }
        r.loss = L;
        const size_t trow = static_cast<size_t>(pd.b) * kt + pd.i;
        p.rec[trow] = r;
        if (p.row_info) p.row_info[trow] = r;
    };

    // ---------------------------------------------------------------- loaded rows
    while (cur.kind != kItemNone) {
        const int par = it & 1;
        int wn = w + ncl;
        Item nxt{kItemNone, -1, -1};
        if (!compact) nxt = next_loaded(wn);
        // rank 0 asks for the next item now; it travels in this row's message #1
        uint32_t fetched = 0;
        if (compact && rank == 0 && t == 0) fetched = atomicAdd(&p.hdr->item_ticket, 1u);
        // until the head has finished: build the lists as soon as it has, and before rank 0
        // decodes a ticket past the row-0 items
        if (compact && !list_ready) try_list(rank == 0 && fetched >= static_cast<uint32_t>(p.B));
        // and every CTA asks for one zero-row unit to write while this row's exchange is in flight
        int zfetch = 0;
        if (zunits > 0 && t == 0) zfetch = static_cast<int>(atomicAdd(&p.hdr->zero_ticket, 1u));
        if (t == 0) mbar_arrive_expect_tx(&c.x1[par], static_cast<uint32_t>(CL * sizeof(Msg1)));
        const int b = cur.b, i = cur.i;
        const size_t drow = static_cast<size_t>(b) * k + i;      // draft / gradient row
        const size_t trow = static_cast<size_t>(b) * kt + i;     // target row
        const bool isRow = (cur.kind == kItemRow);
        const bool rowVerify = isRow && verify;
        // exps are needed for distillation rows and for the stochastic ratio and sampler (lse)
        const bool need_lse = (DISTILL && isRow) || STOCH;

        // The caller's draft token: loaded now, first used after pass A (its latency hides behind
        // the staging wait and pass A).  In stochastic mode D_x and T_x come from the staged
        // slice of the CTA that holds x, through the exchange: no dependent global loads.
        uint32_t x = kNone;
        float Dx = 0.f, Tx = 0.f;
        int xraw = -1;
        if (rowVerify && p.draft != nullptr && lane == 0) xraw = __ldg(p.draft + drow);

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
        // argmax candidates: the first id equal to the thread maximum
        uint32_t candT = kNone, candD = kNone;
        {
            const int lvT = bjT * 32 + lane;
            if (lvT < wcnt) candT = static_cast<uint32_t>(v0 + (wv0 + lvT) * 8 + first_pos(myT[lvT], RT));
            if (greedy_x && isRow) {
                const int lvD = bjD * 32 + lane;
                if (lvD < wcnt) candD = static_cast<uint32_t>(v0 + (wv0 + lvD) * 8 + first_pos(myD[lvD], RD));
            }
        }
        // main pass: exp relative to the thread maxima (no rescaling) and the reverse-KL moment;
        // straight-line over all rounds (sentinel vectors contribute exact zeros).  A thread
        // holding sentinels only keeps a zero reference.
        float2 aD = make_float2(0.f, 0.f), aDd = make_float2(0.f, 0.f), aT = make_float2(0.f, 0.f);
        float dmax = kNegInf;
        const float AD = RD > -1e38f ? __fmul_rn(RD, k2) : 0.f, AT = RT > -1e38f ? __fmul_rn(RT, k2) : 0.f;
        const float2 K2 = make_float2(k2, k2);
#pragma unroll
        for (int j = 0; j < NV; ++j) {
            if (!need_lse) continue;
            const int lv = j * 32 + lane;
            float2 xt[4], et[4];
            unpack8x2(myT[lv], xt);
            const float2 nAT = make_float2(-AT, -AT);
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float2 a = fma2(xt[h], K2, nAT);
                et[h] = make_float2(fast_exp2(a.x), fast_exp2(a.y));
            }
            aT = add2(aT, add2(add2(et[0], et[1]), add2(et[2], et[3])));
            if (isRow) {
                float2 xd[4], ed[4];
                unpack8x2(myD[lv], xd);
                const float2 nAD = make_float2(-AD, -AD);
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float2 a = fma2(xd[h], K2, nAD);
                    ed[h] = make_float2(fast_exp2(a.x), fast_exp2(a.y));
                }
                aD = add2(aD, add2(add2(ed[0], ed[1]), add2(ed[2], ed[3])));
                float2 dd[4];
#pragma unroll
                for (int h = 0; h < 4; ++h) dd[h] = sub2(xd[h], xt[h]);
                aDd = fma2(ed[0], dd[0], aDd);
                aDd = fma2(ed[1], dd[1], aDd);
                aDd = fma2(ed[2], dd[2], aDd);
                aDd = fma2(ed[3], dd[3], aDd);
                if (DISTILL) {
                    dmax = fmax3(fmax3(dd[0].x, dd[0].y, dd[1].x), fmax3(dd[1].y, dd[2].x, dd[2].y),
                                 fmax3(dd[3].x, dd[3].y, dmax));
                }
            }
        }

        // the caller's token, range-checked; the lane whose staged vector holds it reads D_x, T_x
        float wDx = 0.f, wTx = 0.f;
        if (rowVerify && p.draft != nullptr) {
            int xv = __shfl_sync(0xffffffffu, xraw, 0);
            if (xv < 0 || xv >= V) {
                if (warp == 0 && lane == 0) set_device_error(&p.hdr->status, SVD_ERR_TOKEN_RANGE);
                xv = -1;
            }
            x = xv < 0 ? kNone : static_cast<uint32_t>(xv);
            if (STOCH && xv >= 0) {
                const int xl = xv - v0;
                float dv = 0.f, tv = 0.f;
                if (xl >= 0 && xl < len) {
                    const int vi = xl >> 3;
                    if (vi / vpw == warp && ((vi - wv0) & 31) == lane) {
                        const int lvx = vi - wv0;
                        dv = __uint_as_float(static_cast<uint32_t>(
                            reinterpret_cast<const uint16_t*>(myD + lvx)[xl & 7]) << 16);
                        tv = __uint_as_float(static_cast<uint32_t>(
                            reinterpret_cast<const uint16_t*>(myT + lvx)[xl & 7]) << 16);
                    }
                }
                wDx = warp_sum(dv);    // one lane of the cluster holds them; the rest add zeros
                wTx = warp_sum(tv);
            }
        }

        // warp partials -> shared memory -> warp 0 -> message #1 to every rank
        {
            const float wmD = redux_max_f32(RD), wmT = redux_max_f32(RT);
            Msg1 m;
            m.mD = wmD;
            m.mT = wmT;
            m.argT = redux_min_u32(RT == wmT ? candT : kNone);
            m.argD = (greedy_x && isRow) ? redux_min_u32(RD == wmD ? candD : kNone) : kNone;
            m.sD = m.sDd = m.sT = 0.f;
            m.dmax = kNegInf;
            if (need_lse) {
                m.sT = warp_sum((aT.x + aT.y) * (RT > -1e38f ? fast_exp2(__fsub_rn(AT, __fmul_rn(wmT, k2))) : 0.f));
                if (isRow) {
                    const float fD = RD > -1e38f ? fast_exp2(__fsub_rn(AD, __fmul_rn(wmD, k2))) : 0.f;
                    m.sD = warp_sum((aD.x + aD.y) * fD);
                    m.sDd = warp_sum((aDd.x + aDd.y) * fD);
                    if (DISTILL) m.dmax = redux_max_f32(dmax);
                }
            }
            m.prev_ce = 0.f;
            m.next_item = 0u;
            m.Dx = wDx;
            m.Tx = wTx;
            if (lane == 0) c.w1[warp] = m;
        }
        if (zunits > 0 && t == 0) c.zu[par] = zfetch;
        __syncthreads();
        if (warp == 0) {
            const Msg1 a = lane < NW ? c.w1[lane] : empty_msg1();
            const float cmD = redux_max_f32(a.mD), cmT = redux_max_f32(a.mT);
            const uint32_t cargT = redux_min_u32(a.mT == cmT ? a.argT : kNone);
            const uint32_t cargD = redux_min_u32(a.mD == cmD ? a.argD : kNone);
            const float cdmax = redux_max_f32(a.dmax);
            const float cDx = STOCH ? warp_sum(a.Dx) : 0.f, cTx = STOCH ? warp_sum(a.Tx) : 0.f;
            float csD = 0.f, csDd = 0.f, csT = 0.f;
            if (need_lse) {
                const float fT = rescale(a.mT, cmT, k2);
                csT = warp_sum(a.sT * fT);
                if (isRow) {
                    const float fD = rescale(a.mD, cmD, k2);
                    csD = warp_sum(a.sD * fD);
                    csDd = warp_sum(a.sDd * fD);
                }
            }
            uint32_t nitem = 0u;
            if (compact && rank == 0) {
                const int fw = static_cast<int>(__shfl_sync(0xffffffffu, fetched, 0));
                nitem = pack_item(decode_loaded(p, true, spre, bkv, fw, verify));
            }
            // the previous row's -log q_y (if this CTA owns its y) goes out with this row's message
            const float pce = c.my_ce[par ^ 1];
            send1(make_uint4(__float_as_uint(cmD), __float_as_uint(csD), __float_as_uint(csDd), __float_as_uint(cdmax)),
                  make_uint4(__float_as_uint(cmT), __float_as_uint(csT), cargT, cargD),
                  make_uint4(__float_as_uint(pce), nitem, __float_as_uint(cDx), __float_as_uint(cTx)), par);
            __syncwarp();
            if (lane == 0) c.my_ce[par ^ 1] = 0.f;
        }
        if (zunits > 0) {
            const int zu = c.zu[par];
            if (zu < zunits) write_zero_unit(zu);
        }
        wait_x(&c.x1[par], static_cast<uint32_t>(it >> 1) & 1u);

        // ------------------------------------------------ row statistics (every warp)
        float MD, MT, lseD = kQNaN, lseT = kQNaN, L2D = 0.f, L2T = 0.f, dl = 0.f, rkl = 0.f, smax = 0.f;
        uint32_t y;
        {
            const Msg1 a = lane < CL ? c.in1[par][lane] : empty_msg1();
            MD = redux_max_f32(a.mD);
            MT = redux_max_f32(a.mT);
            y = redux_min_u32(a.mT == MT ? a.argT : kNone);
            if (greedy_x && isRow) x = redux_min_u32(a.mD == MD ? a.argD : kNone);
            if (STOCH && rowVerify) {
                Dx = warp_sum(a.Dx);
                Tx = warp_sum(a.Tx);
            }
            if (compact) nxt = unpack_item(__shfl_sync(0xffffffffu, a.next_item, 0));
            if (need_lse) {
                const float sT = warp_sum(a.sT * rescale(a.mT, MT, k2));
                lseT = MT * itau + logf(sT);
                L2T = lseT * kLog2e;
                if (isRow) {
                    const float fD = rescale(a.mD, MD, k2);
                    const float sD = warp_sum(a.sD * fD);
                    const float sDd = warp_sum(a.sDd * fD);
                    lseD = MD * itau + logf(sD);
                    L2D = lseD * kLog2e;
                    dl = lseD - lseT;
                    rkl = (sDd / sD) * itau - dl;   // sum_v q_v (log q_v - log p_v)
                    if (DISTILL) smax = redux_max_f32(a.dmax) * itau - dl;   // largest log q_v - log p_v
                }
            }
            // rank 0 writes the previous row's record (its -log q_y arrived just now)
            if (pending && rank == 0 && warp == NW - 1) {
                const float pce = warp_sum(a.prev_ce);   // one owner sends it, the rest send 0
                if (lane == 0) write_record(pce);
            }
        }
        pending = false;

        // stochastic decision (every warp computes the same value); the correction or bonus
        // token of a sequence is drawn after the finalize pass, from its one emitted row
        float ratio = kQNaN;
        int acc = 0;
        if (STOCH && rowVerify) {
            const PhiloxOut ph = philox_words(p.seed, p.step, static_cast<uint32_t>(b),
                                              static_cast<uint32_t>(i));
            const float u0 = uniform24(ph.w[0]);
            if (x != kNone) {
                ratio = fast_exp2((dl - (Dx - Tx) * itau) * kLog2e);
                acc = u0 < fminf(1.f, ratio) ? 1 : 0;
            } else {
                ratio = 0.f;
                acc = 0;
            }
        }
        if (rowVerify && !STOCH) acc = (x == y) ? 1 : 0;

        // Clipping is possible only if max_v q_v * max_v (log q_v - log p_v) reaches c; the
        // bound is the same in every CTA, so the second exchange is skipped uniformly.
        bool do_clip = false;
        float qthr = 0.f;
        if (DISTILL && isRow && isfinite(cc) && smax > 0.f) {
            qthr = (cc / smax) * 0.9999f;
            const float qmax = fast_exp2(__fsub_rn(__fmul_rn(MD, k2), L2D));
            do_clip = qmax * 1.001f > qthr;
        }
        const bool need_x2 = do_clip;

        // -------------------------------------------------------- pass B
        // d_v = q_v s_v <= q_v s_max, so only entries with q_v > c / s_max can be clipped; those
        // vectors alone are re-read and tested exactly
        float clip_d = 0.f, clip_q = 0.f, n_clip = 0.f;
        uint32_t clipmask = 0;
        if (do_clip) {
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                // largest q of the vector, from its largest draft logit (exact bf16 max)
                const float qv = fast_exp2(__fsub_rn(__fmul_rn(max8_bf16(myD[j * 32 + lane]), k2), L2D));
                if (qv > qthr) {
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
        // exchange #2: clip sums (skipped when no entry can be clipped)
        float g_clip_d = 0.f, g_clip_q = 0.f, g_n_clip = 0.f;
        if (need_x2) {
            if (t == 0) mbar_arrive_expect_tx(&c.x2, static_cast<uint32_t>(CL * sizeof(Msg2)));
            clip_d = warp_sum(clip_d);
            clip_q = warp_sum(clip_q);
            n_clip = warp_sum(n_clip);
            if (lane == 0) {
                Msg2 q2;
                q2.clip_d = clip_d; q2.clip_q = clip_q; q2.n_clip = n_clip; q2.pad0 = 0.f;
                c.w2[warp] = q2;
            }
            __syncthreads();
            if (warp == 0) {
                float a0 = 0.f, a1 = 0.f, a2 = 0.f;
                if (lane < NW) {
                    a0 = c.w2[lane].clip_d; a1 = c.w2[lane].clip_q; a2 = c.w2[lane].n_clip;
                }
                a0 = warp_sum(a0);
                a1 = warp_sum(a1);
                a2 = warp_sum(a2);
                if (lane < CL) {
                    const uint32_t dst = dsmem_map(&c.in2[rank], static_cast<uint32_t>(lane));
                    const uint32_t bar = dsmem_map(&c.x2, static_cast<uint32_t>(lane));
                    st_async_v4(dst, make_uint4(__float_as_uint(a0), __float_as_uint(a1), __float_as_uint(a2), 0u), bar);
                }
            }
            wait_x(&c.x2, n2 & 1u);
            ++n2;
            const Msg2 a = lane < CL ? c.in2[lane] : Msg2{0.f, 0.f, 0.f, 0.f};
            g_clip_d = warp_sum(a.clip_d);
            g_clip_q = warp_sum(a.clip_q);
            g_n_clip = warp_sum(a.n_clip);
        }

        // ------------------------------------------------ row results (every warp)
        float kc = 0.f, P = 0.f, Q = 0.f, Pc = 0.f, hardc = 0.f;
        if (DISTILL && isRow) {
            // S = sum over unclipped entries of q (s + 1) = (rkl - clip_d) + (1 - clip_q)
            const float S = (rkl - g_clip_d) + (1.f - g_clip_q);
            kc = isfinite(cc) ? (rkl - g_clip_d) + cc * g_n_clip : rkl;
            const float lam = p.lambda, pre = p.grad_scale * itau;
            P = pre * (lam + (1.f - lam) * (1.f - S - dl));
            Q = pre * (1.f - lam) * itau;
            Pc = pre * (lam - (1.f - lam) * S);
            hardc = pre * lam;
        }

        // -------------------------------------------------------- pass C: gradient row
        if (DISTILL && isRow) {
            const float2 nL2D = make_float2(-L2D, -L2D), QQ = make_float2(Q, Q), PP = make_float2(P, P);
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                const int lv = j * 32 + lane;
                float2 xd[4], xt[4], g[4];
                unpack8x2(myD[lv], xd);
                unpack8x2(myT[lv], xt);
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float2 a = fma2(xd[h], K2, nL2D);
                    const float2 q = make_float2(fast_exp2(a.x), fast_exp2(a.y));
                    g[h] = mul2(q, fma2(QQ, sub2(xd[h], xt[h]), PP));
                }
                if (lv < wcnt) store_vec(drow, lv, g);
            }
            // vectors holding clipped entries are stored again with the clipped form
            while (clipmask) {
                const int j = __ffs(clipmask) - 1;
                clipmask &= clipmask - 1u;
                const int lv = j * 32 + lane;
                float xd[8], xt[8];
                unpack8(myD[lv], xd);
                unpack8(myT[lv], xt);
                float gl[8];
#pragma unroll
                for (int l = 0; l < 8; ++l) {
                    const float q = elem_q(xd[l], k2, L2D);
                    const float d = elem_d(q, elem_s(xd[l], xt[l], itau, dl));
                    gl[l] = d > cc ? q * Pc : q * fmaf(Q, xd[l] - xt[l], P);
                }
                const float2 g[4] = {make_float2(gl[0], gl[1]), make_float2(gl[2], gl[3]),
                                     make_float2(gl[4], gl[5]), make_float2(gl[6], gl[7])};
                if (lv < wcnt) store_vec(drow, lv, g);
            }
            // the owner of y stores its entry again with the hard-label term and reports -log q_y
            const int yl = static_cast<int>(y) - v0;
            if (y != kNone && yl >= 0 && yl < len) {
                const int vi = yl >> 3;
                if (vi / vpw == warp) {
                    const int lvy = vi - wv0;
                    if ((lvy & 31) == lane) {
                        // the two bf16 values straight from the staged vectors (dynamic index
                        // into shared memory, not into a register array)
                        const float dy = __uint_as_float(static_cast<uint32_t>(
                            reinterpret_cast<const uint16_t*>(myD + lvy)[yl & 7]) << 16);
                        const float ty = __uint_as_float(static_cast<uint32_t>(
                            reinterpret_cast<const uint16_t*>(myT + lvy)[yl & 7]) << 16);
                        const float qa = fast_exp2(fmaf(dy, k2, -L2D));
                        float gy = qa * fmaf(Q, dy - ty, P);
                        if (do_clip) {
                            const float q = elem_q(dy, k2, L2D);
                            if (elem_d(q, elem_s(dy, ty, itau, dl)) > cc) gy = q * Pc;
                        }
                        store_elem(drow, static_cast<int>(y), gy - hardc);
                        c.my_ce[par] = lseD - dy * itau;   // -log q_y
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

        // rank 0 keeps this row's values; the record is written after the next exchange #1
        if (rank == 0 && warp == NW - 1 && lane == 0) {
            Pending& pd = c.pend;
            pd.b = b; pd.i = i; pd.kind = cur.kind;
            pd.x = rowVerify ? (x == kNone ? -1 : static_cast<int>(x)) : -1;
            pd.y = static_cast<int>(y);
            pd.acc = rowVerify ? acc : -1;
            pd.ratio = ratio;
            pd.lseD = isRow ? lseD : kQNaN;
            pd.lseT = lseT;
            pd.kc = kc;
        }
        pending = true;
        cur = nxt;
        w = wn;
        ++it;
    }
    if (pending) {
        // uniform: every rank walked the same items.  One more exchange #1 carries the last
        // row's -log q_y to rank 0.
        const int par = it & 1;
        if (t == 0) mbar_arrive_expect_tx(&c.x1[par], static_cast<uint32_t>(CL * sizeof(Msg1)));
        __syncthreads();
        if (warp == 0) {
            const float pce = c.my_ce[par ^ 1];
            const uint32_t ninf = __float_as_uint(kNegInf);
            send1(make_uint4(ninf, 0u, 0u, ninf), make_uint4(ninf, 0u, kNone, kNone),
                  make_uint4(__float_as_uint(pce), 0u, 0u, 0u), par);
        }
        wait_x(&c.x1[par], static_cast<uint32_t>(it >> 1) & 1u);
        if (rank == 0 && warp == NW - 1) {
            const Msg1 a = lane < CL ? c.in1[par][lane] : empty_msg1();
            const float pce = warp_sum(a.prev_ce);
            if (lane == 0) write_record(pce);
        }
    }

    // ---------------------------------------------------------------- zero-only gradient rows
    if (DISTILL && compact) {
        if (!list_ready) try_list(true);
        // the zero-row units not yet taken, handed to CTAs one at a time (the next unit is
        // requested while the current one is written)
        const int units = zunits;
        if (t == 0) c.zs = static_cast<int>(atomicAdd(&p.hdr->zero_ticket, 1u));
        __syncthreads();
        int u = c.zs;
        __syncthreads();
        while (u < units) {
            int nextu = 0;
            if (t == 0) nextu = static_cast<int>(atomicAdd(&p.hdr->zero_ticket, 1u));
            write_zero_unit(u);
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
// sequence losses in a fixed order (per lane in sequence order, then a butterfly).
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) finalize_kernel(const RowParams p) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // the stochastic draw (a programmatic dependent of this pass) may be scheduled now; it waits
    // for this grid's results
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __shared__ int last;
    // the row pass has finished: its work tickets go back to zero for the next call
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        p.hdr->item_ticket = 0u;
        p.hdr->zero_ticket = 0u;
        p.hdr->head_unit = 0u;
        p.hdr->head_done = 0u;
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const bool verify = (p.flags & kFlagVerify) != 0;
    const bool distill = (p.flags & kFlagDistill) != 0;
    const int k = p.k, kt = p.kt;
    const int b = blockIdx.x * 8 + warp;
    if (b < p.B) {
        int n = p.bk_const > 0 ? p.bk_const : __ldg(p.bk + b);
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
                // length-head labels: the observable proxy a / b_k and, verifying all k, a / k
                if (p.bk_const > 0) {
                    int nt = __ldg(p.bk_trunc + b);
                    nt = nt < 1 ? 1 : (nt > k ? k : nt);
                    if (p.label_proxy) p.label_proxy[b] = static_cast<float>(min(a, nt)) / static_cast<float>(nt);
                    if (p.label_full) p.label_full[b] = static_cast<float>(a) / static_cast<float>(k);
                } else {
                    if (p.label_proxy) p.label_proxy[b] = static_cast<float>(a) / static_cast<float>(n);
                    if (p.label_full) p.label_full[b] = kQNaN;
                }
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
    // the last CTA adds the sequence losses in a fixed order
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t old = atomicAdd(&p.hdr->loss_ticket, 1u);
        last = (old + 1u == gridDim.x) ? 1 : 0;
    }
    __syncthreads();
    if (!last || threadIdx.x >= 32) return;
    __threadfence();
    // warp 0: lane l adds sequences l, l + 32, ... in order, then a fixed butterfly
    float tot = 0.f;
#pragma unroll 4
    for (int s = lane; s < p.B; s += 32) tot += __ldcg(p.seq_loss + s);
    tot = warp_sum(tot);
    if (lane == 0) {
        *p.loss_total = tot;
        p.hdr->loss_ticket = 0u;
    }
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
// Large vocabularies: clusters of ceil(V / 16384) CTAs of 256 threads x 8 vectors, three CTAs
// per SM (10 CTAs per row at V = 151936).  Measured at B = 128, k = 16, V = 151936 on B200, row
// pass alone: 0.365 ms, against 0.405 ms for 8 CTAs of 256 x 10 (two per SM), 0.438 ms for 16
// of 256 x 5 (four per SM), 0.431 ms for 11 of 256 x 7 and 0.450 ms for 4 of 512 x 10.
// Vocabularies whose slices would need more than 16 CTAs take 256 x 10.
constexpr int kSNT = 128, kSNV = 2, kSMB = 8;     //  2048 ids per CTA
constexpr int kLNT = 256, kLNV = 8, kLMB = 3;     // 16384 ids per CTA
// a length-head split of kHeadSplitCols columns stages in one chunk of this shape's staging area
static_assert(((kLNV * kLNT * 32 / (2 * (kHeadTileB + kHeadTileM)) - 8) & ~15) >= kHeadSplitCols,
              "head split width and staging area");
constexpr int kXNT = 256, kXNV = 10, kXMB = 2;    // 20480 ids per CTA

int next_pow2(int x) {
    int r = 1;
    while (r < x) r <<= 1;
    return r;
}

}  // namespace

bool row_geometry(int V, RowGeometry* g) {
    if (V < 1) return false;
    const int capS = kSNT * kSNV * 8, capL = kLNT * kLNV * 8, capX = kXNT * kXNV * 8;
    if (V <= 8 * capS) {
        g->variant = 0; g->threads = kSNT;
        g->cluster = next_pow2((V + capS - 1) / capS);
        g->smem = smem_fixed<kSNT, kSNV>();
    } else if (V <= 16 * capL) {
        g->variant = 1; g->threads = kLNT;
        g->cluster = (V + capL - 1) / capL;
        g->smem = smem_fixed<kLNT, kLNV>();
    } else {
        g->variant = 2; g->threads = kXNT;
        g->cluster = (V + capX - 1) / capX;
        g->smem = smem_fixed<kXNT, kXNV>();
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

namespace {

// Resident clusters of a row-pass kernel on the current device, for a launch with `smem` bytes of
// dynamic shared memory.  The function attributes are set once per (device, kernel) -- to the
// largest dynamic shared memory any batch size can ask for -- and the occupancy query once per
// (device, kernel, smem); both under a lock, so concurrent first calls from several host
// threads neither race on the cache nor on the attributes.
struct OccEntry {
    int dev;
    KernelFn fn;
    size_t smem;
    int clusters;
};
std::mutex g_occ_lock;
std::vector<OccEntry> g_occ;                     // occupancy per (device, kernel, smem)
std::vector<std::pair<int, KernelFn>> g_attr;    // (device, kernel) with attributes set

int resident_clusters(KernelFn fn, const RowGeometry& geo, size_t smem, cudaLaunchConfig_t cfg,
                      int* out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return static_cast<int>(err);
    std::lock_guard<std::mutex> guard(g_occ_lock);
    for (const OccEntry& e : g_occ) {
        if (e.dev == dev && e.fn == fn && e.smem == smem) {
            *out = e.clusters;
            return 0;
        }
    }
    bool attr_set = false;
    for (const auto& a : g_attr) attr_set = attr_set || (a.first == dev && a.second == fn);
    if (!attr_set) {
        err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   static_cast<int>(row_smem_bytes(geo, kCompactMaxB)));
        if (err != cudaSuccess) return static_cast<int>(err);
        // the same kernel serves vocabularies whose clusters exceed the portable size of 8
        err = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (err != cudaSuccess) return static_cast<int>(err);
        g_attr.emplace_back(dev, fn);
    }
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cfg.gridDim = dim3(geo.cluster * sms, 1, 1);
    int n = 0;
    err = cudaOccupancyMaxActiveClusters(&n, fn, &cfg);
    if (err != cudaSuccess || n < 1) {
        cudaGetLastError();
        n = sms / geo.cluster > 0 ? sms / geo.cluster : 1;
    }
    g_occ.push_back(OccEntry{dev, fn, smem, n});
    *out = n;
    return 0;
}

}  // namespace

int launch_row_pass(const RowParams& p, void* stream) {
    RowGeometry geo;
    if (!row_geometry(p.V, &geo)) return static_cast<int>(cudaErrorInvalidValue);
    const bool aligned = p.aligned != 0;
    KernelFn fn = geo.variant == 0 ? pick_kernel<kSNT, kSNV, kSMB>(p.flags, aligned)
                : geo.variant == 1 ? pick_kernel<kLNT, kLNV, kLMB>(p.flags, aligned)
                                   : pick_kernel<kXNT, kXNV, kXMB>(p.flags, aligned);
    const size_t smem = row_smem_bytes(geo, p.B);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = geo.cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.blockDim = dim3(geo.threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = static_cast<cudaStream_t>(stream);
    // persistent grid: as many clusters as can be resident at once
    int cache = 0;
    cudaError_t err = static_cast<cudaError_t>(resident_clusters(fn, geo, smem, cfg, &cache));
    if (err != cudaSuccess) return static_cast<int>(err);
    const long long max_items = static_cast<long long>(p.B) * (p.kt + p.k);
    int nclusters = cache;
    if (max_items < nclusters) nclusters = static_cast<int>(max_items > 0 ? max_items : 1);
    cfg.gridDim = dim3(geo.cluster * nclusters, 1, 1);
    // a programmatic dependent of the preceding kernel (the kernel waits for it first thing):
    // the launch latency overlaps that kernel's tail
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.numAttrs = 2;
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
    if (err != cudaSuccess) return static_cast<int>(err);
    // stochastic verification: the one drawn token per sequence, once its row is known
    if ((p.flags & kFlagStochastic) && (p.flags & kFlagVerify)) return launch_sample_fix(q, stream);
    return 0;
}

}  // namespace svd
