// svd_head_unit.cuh -- the length head as independent work units that any CTA can take, so the
// row pass can compute b_k itself, in its first microseconds, instead of waiting for a separate
// kernel.
//
// What it computes (AdaFlash; Pith review page "What carries the argument": a small network on
// the drafter's pooled hidden state predicts the block's acceptance rate; Axiom & Free-Parameter
// Ledger: a single scalar converted linearly to the verification length, gamma = 1.0; Referee
// Report minor comment 2: b_k = clamp(floor(bhat * k), 1, k), ceil by default here):
//     z_b = w2 . relu(W1 h_b + b1) + b2,   bhat_b = sigmoid(z_b),
//     b_k = clamp(round(gamma * bhat_b * k), 1, k)   (round = ceil or floor).
//
// Work units: (16-sequence tile bt) x (64-unit tile mt) x (K split kz).  A unit is one CTA (any
// multiple of 32 threads, at least 32): it stages its slices of h and W1 in shared memory with
// bulk copies, its warps take the eight 16 x 8 blocks of hidden units in turn and accumulate each
// over the split's K range on the tensor cores (mma.sync m16n8k16, bf16 operands, fp32
// accumulation), and the unit stores its block as a split partial.  The last unit of an
// output tile (atomic ticket, no waiting) adds the partials in split order, applies b1, ReLU and
// w2 and sums the tile's 64 units per sequence; the last tile of a sequence tile adds the tile
// sums in tile order and applies the sigmoid and the b_k map, then counts the sequence tile as
// done.  Every sum has a fixed order, and no unit ever waits for another, so the units can be
// handed out dynamically to whichever CTAs are running.
#pragma once

#include "svd_device.cuh"

namespace svd {

// D += A(16x16, row) * B(16x8, col), bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma_16816_bf16(float (&d)[4], const uint32_t (&a)[4],
                                               const uint32_t (&b)[2]) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Units of the head and the number of 16-sequence tiles that must finish.
__host__ __device__ inline int head_units(const HeadParams& p) {
    const int bt = (p.B + kHeadTileB - 1) / kHeadTileB, mt = (p.M + kHeadTileM - 1) / kHeadTileM;
    return bt * mt * p.nsplit;
}
__host__ __device__ inline int head_seq_tiles(const HeadParams& p) {
    return (p.B + kHeadTileB - 1) / kHeadTileB;
}

// Columns of one staged K chunk that fit in `smem_bytes` of shared memory: 16 rows of h and 64
// rows of W1, each padded by 8 bf16 (16 bytes) so that fragment reads hit distinct banks.
__host__ __device__ inline int head_chunk_cols(size_t smem_bytes) {
    const long cols = static_cast<long>(smem_bytes / (2 * (kHeadTileB + kHeadTileM))) - 8;
    return cols < 16 ? 0 : static_cast<int>(cols & ~15L);
}

// One unit, executed by all threads of the calling CTA (H a multiple of 16; h and W1 16-byte
// aligned).  The split's K range is staged in chunks: one bulk copy (1-D TMA, no multicast) per
// row of h and of W1, issued by the lanes of warp 0 in turn, into `stage` (smem_bytes of this
// CTA's shared memory), completing on the
// mbarrier `bar` (count 1; `phase` is its parity, flipped per chunk), then the warps take the
// eight 16 x 8 blocks of hidden units m0 + 8j .. m0 + 8j + 7 in turn and accumulate them over
// the chunk from shared memory.  A chunk costs one round trip to memory.  `flag` is one int of
// the CTA's shared memory.  The tickets live in p.tile_ticket: [bt * mt] output-tile tickets,
// then [bt] sequence-tile tickets; every ticket is back at zero once its last user has
// finished.  p.hdr->head_done counts finished sequence tiles.  With `standalone` (a kernel that
// only runs the head), the last sequence tile also puts head_done back to zero; inside the row
// pass the finalize pass does, after the rows have read it.  Returns false if a staging wait
// ran out (the status word then says SVD_ERR_TIMEOUT).
template <int NW>
__device__ __forceinline__ bool head_unit(const HeadParams& p, int u, int* flag, bool standalone,
                                          uint16_t* stage, size_t smem_bytes, uint64_t* bar,
                                          uint32_t& phase, uint64_t wait_limit_ns) {
    constexpr int nw = NW;                          // warps of the calling CTA
    constexpr int kPer = (kHeadTileM / 8 + NW - 1) / NW;   // 16 x 8 blocks per warp
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int BT = (p.B + kHeadTileB - 1) / kHeadTileB, MT = (p.M + kHeadTileM - 1) / kHeadTileM;
    const int kz = u % p.nsplit;
    const int tile = u / p.nsplit;
    const int mt = tile % MT, bt = tile / MT;
    const int b0 = bt * kHeadTileB, m0 = mt * kHeadTileM;
    const int g = lane >> 2, tq = lane & 3;
    const int k_lo = min(p.H, kz * p.ks), k_hi = min(p.H, k_lo + p.ks);
    const int nrow_h = min(kHeadTileB, p.B - b0), nrow_w = min(kHeadTileM, p.M - m0);
    const int cmax = head_chunk_cols(smem_bytes);
    const int nchunk = k_hi > k_lo ? (k_hi - k_lo + cmax - 1) / cmax : 0;
    const int cw = nchunk > 0 ? (((k_hi - k_lo + nchunk - 1) / nchunk) + 15) & ~15 : 0;
    const int ld = cw + 8;                              // row pitch in bf16
    uint16_t* hs = stage;
    uint16_t* ws = stage + kHeadTileB * ld;
    bool ok = true;

    // ------------------------------------------------ split partials, 16 x 8 blocks by warp
    // (a warp owns blocks warp, warp + nw, ...)
    float acc[kPer][4];
#pragma unroll
    for (int j = 0; j < kPer; ++j)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[j][q] = 0.f;
    // rows past the batch or the hidden size read as zeros
    for (int x = t; x < (kHeadTileB - nrow_h) * ld; x += blockDim.x) hs[nrow_h * ld + x] = 0;
    for (int x = t; x < (kHeadTileM - nrow_w) * ld; x += blockDim.x) ws[nrow_w * ld + x] = 0;
    for (int ch = 0; ch < nchunk; ++ch) {
        const int c0 = k_lo + ch * cw, c1 = min(k_hi, c0 + cw);
        __syncthreads();      // every read of the previous chunk (and the zero rows) is done
        if (warp == 0) {
            // lane 0 announces the chunk's bytes, then the 32 lanes issue its row copies
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            const uint32_t row_bytes = static_cast<uint32_t>(c1 - c0) * 2u;
            if (lane == 0) mbar_arrive_expect_tx(bar, row_bytes * static_cast<uint32_t>(nrow_h + nrow_w));
            __syncwarp();
            for (int r = lane; r < nrow_h + nrow_w; r += 32) {
                if (r < nrow_h)
                    bulk_load(hs + r * ld, p.h + static_cast<size_t>(b0 + r) * p.H + c0, row_bytes, bar);
                else
                    bulk_load(ws + (r - nrow_h) * ld, p.W1 + static_cast<size_t>(m0 + r - nrow_h) * p.H + c0,
                              row_bytes, bar);
            }
        }
        if (ok && !mbar_wait_bounded(bar, phase, wait_limit_ns)) {
            ok = false;
            set_device_error(&p.hdr->status, SVD_ERR_TIMEOUT);
        }
        phase ^= 1u;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int blk = warp + j * nw;
            if (blk >= kHeadTileM / 8) break;
            const uint16_t* wrow = ws + (blk * 8 + g) * ld;
            for (int kk = 0; kk < c1 - c0; kk += 16) {
                uint32_t a[4], bf[2];
                a[0] = *reinterpret_cast<const uint32_t*>(hs + g * ld + kk + 2 * tq);
                a[1] = *reinterpret_cast<const uint32_t*>(hs + (g + 8) * ld + kk + 2 * tq);
                a[2] = *reinterpret_cast<const uint32_t*>(hs + g * ld + kk + 2 * tq + 8);
                a[3] = *reinterpret_cast<const uint32_t*>(hs + (g + 8) * ld + kk + 2 * tq + 8);
                bf[0] = *reinterpret_cast<const uint32_t*>(wrow + kk + 2 * tq);
                bf[1] = *reinterpret_cast<const uint32_t*>(wrow + kk + 2 * tq + 8);
                mma_16816_bf16(acc[j], a, bf);
            }
        }
    }
    __syncthreads();          // the staging area is free again when this returns
    // accumulator layout: acc[j][0..1] = (row g, cols 2tq + {0,1}); acc[j][2..3] = row g + 8
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        const int blk = warp + j * nw;
        if (blk >= kHeadTileM / 8) break;
        float* part = p.part + static_cast<size_t>(kz) * p.B * p.M;
        const int m = m0 + blk * 8 + 2 * tq;
        const int rows[2] = {b0 + g, b0 + g + 8};
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            const int b = rows[h2];
            if (b < p.B) {
                if (m < p.M) part[static_cast<size_t>(b) * p.M + m] = acc[j][2 * h2];
                if (m + 1 < p.M) part[static_cast<size_t>(b) * p.M + m + 1] = acc[j][2 * h2 + 1];
            }
        }
    }
    // ------------------------------------------------ last split of the output tile
    __threadfence();
    __syncthreads();
    if (t == 0) {
        const uint32_t old = atomicAdd(&p.tile_ticket[bt * MT + mt], 1u);
        *flag = (old + 1u == static_cast<uint32_t>(p.nsplit)) ? 1 : 0;
    }
    __syncthreads();
    if (!*flag) return ok;
    __threadfence();
    // sixteen threads per row of the tile, four units each (m0 + l + 16 i): the split partials
    // of all four in flight eight splits at a time, added in split order; then b1, ReLU and w2,
    // and the row's sixteen threads combined by a fixed butterfly
    for (int o = t; o < kHeadTileB * 16; o += blockDim.x) {
        const int r = o >> 4, l = o & 15;
        const int b = b0 + r;
        float a[4] = {0.f, 0.f, 0.f, 0.f};
        if (b < p.B) {
            for (int z0 = 0; z0 < p.nsplit; z0 += 8) {
                float v[8][4];
#pragma unroll
                for (int z = 0; z < 8; ++z) {
                    const float* src = p.part + (static_cast<size_t>(z0 + z) * p.B + b) * p.M + m0 + l;
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        v[z][i] = (z0 + z < p.nsplit && m0 + l + 16 * i < p.M) ? __ldcg(src + 16 * i) : 0.f;
                }
#pragma unroll
                for (int z = 0; z < 8; ++z)
#pragma unroll
                    for (int i = 0; i < 4; ++i) a[i] += v[z][i];
            }
        }
        float zz = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int m = m0 + l + 16 * i;
            if (b < p.B && m < p.M) {
                float x = a[i];
                if (p.b1) x += __ldg(p.b1 + m);
                if (p.u_out) p.u_out[static_cast<size_t>(b) * p.M + m] = x;
                const float w2 = __uint_as_float(static_cast<uint32_t>(__ldg(p.w2 + m)) << 16);
                zz += w2 * fmaxf(x, 0.f);
            }
        }
#pragma unroll
        for (int o2 = 8; o2 > 0; o2 >>= 1) zz += __shfl_xor_sync(0xffffffffu, zz, o2);
        if (l == 0 && b < p.B) p.zpart[static_cast<size_t>(mt) * p.B + b] = zz;
    }
    if (t == 0) p.tile_ticket[bt * MT + mt] = 0u;
    // ------------------------------------------------ last tile of the sequence tile
    __threadfence();
    __syncthreads();
    if (t == 0) {
        const uint32_t old = atomicAdd(&p.tile_ticket[BT * MT + bt], 1u);
        *flag = (old + 1u == static_cast<uint32_t>(MT)) ? 2 : 0;
    }
    __syncthreads();
    if (*flag != 2) return ok;
    __threadfence();
    if (t < kHeadTileB && b0 + t < p.B) {
        const int b = b0 + t;
        float z = p.b2_dev ? *p.b2_dev : p.b2;
        // tile sums in tile order, eight loads in flight at a time
        for (int q0 = 0; q0 < MT; q0 += 8) {
            float v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                v[q] = q0 + q < MT ? __ldcg(p.zpart + static_cast<size_t>(q0 + q) * p.B + b) : 0.f;
#pragma unroll
            for (int q = 0; q < 8; ++q) z += v[q];
        }
        const float bhat = 1.f / (1.f + expf(-z));
        const float target = p.gamma * bhat * static_cast<float>(p.k);
        const float r = p.rnd == 0 ? ceilf(target) : floorf(target);
        int bk = static_cast<int>(fminf(fmaxf(r, 1.f), static_cast<float>(p.k)));
        if (!(r == r)) bk = 1;  // non-finite hidden states
        if (p.bhat) p.bhat[b] = bhat;
        if (p.bk) p.bk[b] = bk;
    }
    if (t == 0) p.tile_ticket[BT * MT + bt] = 0u;
    __threadfence();
    __syncthreads();
    if (t == 0) {
        const uint32_t old = atomicAdd(&p.hdr->head_done, 1u);
        if (standalone && old + 1u == static_cast<uint32_t>(BT)) p.hdr->head_done = 0u;
    }
    return ok;
}

}  // namespace svd
