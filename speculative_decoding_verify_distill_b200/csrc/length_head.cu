// length_head.cu -- the adaptive length head: bhat = sigmoid(w2 . relu(W1 h + b1) + b2) and the
// verification length b_k = clamp(round(gamma * bhat * k), 1, k).
//
// AdaFlash (Pith review page "What carries the argument": a small network on drafter hidden
// states predicts the block's acceptance rate; Axiom & Free-Parameter Ledger: a pooled
// representation is mapped to a single scalar and converted linearly to the verification length,
// gamma = 1.0; Referee Report minor comment 2: b_k = clamp(floor(bhat * k), 1, k)).
//
// The projection h [B,H] x W1^T [H,M] is a small dense contraction (2*B*H*M flops, e.g. 0.27
// GFLOP at B=128, H=4096, M=256), run on the tensor cores with bf16 operands and fp32
// accumulation.  Grid: one CTA per (16 sequences, 64 hidden units); the 8 warps of a CTA split
// the H axis and their 16x64 partial tiles are summed in shared memory in a fixed order.  Each
// CTA then applies bias, ReLU and its slice of w2, leaving one partial logit per sequence; the
// last CTA to finish (atomic ticket, no waiting) adds the partials in tile order, applies the
// sigmoid and the b_k map.
#include <cuda_runtime.h>

#include <cmath>

#include "svd_device.cuh"

namespace svd {

namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Two consecutive bf16 elements (row r, columns c, c+1) of a [rows, cols] matrix; zero outside.
__device__ __forceinline__ uint32_t load_pair(const uint16_t* m, int rows, int cols, int r, int c,
                                              bool vec_ok) {
    if (r >= rows) return 0u;
    const uint16_t* src = m + static_cast<size_t>(r) * cols + c;
    if (vec_ok && c + 1 < cols) return __ldg(reinterpret_cast<const uint32_t*>(src));
    const uint32_t lo = c < cols ? __ldg(src) : 0u;
    const uint32_t hi = c + 1 < cols ? __ldg(src + 1) : 0u;
    return lo | (hi << 16);
}

}  // namespace

__global__ void __launch_bounds__(kWarps * 32) length_head_kernel(const HeadParams p) {
    __shared__ float part[kWarps][kHeadTileB][kHeadTileM + 1];
    __shared__ float zrow[kHeadTileB][kWarps];
    __shared__ int is_last;

    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int b0 = blockIdx.x * kHeadTileB, m0 = blockIdx.y * kHeadTileM;
    const int g = lane >> 2, tq = lane & 3;
    // 32-bit fragment loads need even row lengths and 4-byte aligned bases
    const bool vec_ok = (p.H % 2 == 0) && ((reinterpret_cast<uintptr_t>(p.h) & 3) == 0) &&
                        ((reinterpret_cast<uintptr_t>(p.W1) & 3) == 0);

    float acc[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[n][q] = 0.f;

    const int ksteps = (p.H + 15) / 16;
    for (int s = warp; s < ksteps; s += kWarps) {
        const int k0 = s * 16 + 2 * tq;
        uint32_t a[4];
        a[0] = load_pair(p.h, p.B, p.H, b0 + g, k0, vec_ok);
        a[1] = load_pair(p.h, p.B, p.H, b0 + g + 8, k0, vec_ok);
        a[2] = load_pair(p.h, p.B, p.H, b0 + g, k0 + 8, vec_ok);
        a[3] = load_pair(p.h, p.B, p.H, b0 + g + 8, k0 + 8, vec_ok);
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            const int m = m0 + n * 8 + g;
            uint32_t bf[2];
            bf[0] = load_pair(p.W1, p.M, p.H, m, k0, vec_ok);
            bf[1] = load_pair(p.W1, p.M, p.H, m, k0 + 8, vec_ok);
            mma_bf16_16816(acc[n], a, bf);
        }
    }
    // accumulator layout: acc[n][0..1] = (row g, cols n*8 + 2tq + {0,1}); [2..3] = row g + 8
#pragma unroll
    for (int n = 0; n < 8; ++n) {
        part[warp][g][n * 8 + 2 * tq] = acc[n][0];
        part[warp][g][n * 8 + 2 * tq + 1] = acc[n][1];
        part[warp][g + 8][n * 8 + 2 * tq] = acc[n][2];
        part[warp][g + 8][n * 8 + 2 * tq + 1] = acc[n][3];
    }
    __syncthreads();

    // each warp owns two sequences of the tile; lanes cover the 64 hidden units in pairs
    for (int rb = warp * 2; rb < warp * 2 + 2; ++rb) {
        float zsum = 0.f;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            const int col = lane + 32 * h2;
            const int m = m0 + col;
            float a = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) a += part[w][rb][col];
            if (m < p.M) {
                if (p.b1) a += __ldg(p.b1 + m);
                const float hid = fmaxf(a, 0.f);
                const float w2 = __uint_as_float(static_cast<uint32_t>(__ldg(p.w2 + m)) << 16);
                zsum = fmaf(w2, hid, zsum);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) zsum += __shfl_xor_sync(0xffffffffu, zsum, o);
        if (lane == 0) zrow[rb][0] = zsum;
    }
    __syncthreads();
    if (t < kHeadTileB && b0 + t < p.B) p.zpart[static_cast<size_t>(blockIdx.y) * p.B + b0 + t] = zrow[t][0];

    // last CTA to finish combines the partial logits of every tile
    __threadfence();
    __syncthreads();
    if (t == 0) {
        const uint32_t total = gridDim.x * gridDim.y;
        const uint32_t old = atomicAdd(&p.hdr->head_ticket, 1u);
        is_last = (old + 1u == total) ? 1 : 0;
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    const int mtiles = gridDim.y;
    for (int b = t; b < p.B; b += blockDim.x) {
        float z = p.b2;
        for (int mt = 0; mt < mtiles; ++mt) z += __ldcg(p.zpart + static_cast<size_t>(mt) * p.B + b);
        const float bhat = 1.f / (1.f + expf(-z));
        const float target = p.gamma * bhat * static_cast<float>(p.k);
        float r = p.rnd == 0 ? ceilf(target) : floorf(target);
        int bk = static_cast<int>(fminf(fmaxf(r, 1.f), static_cast<float>(p.k)));
        if (!(r == r)) bk = 1;  // NaN guard (non-finite hidden states)
        if (p.bhat) p.bhat[b] = bhat;
        p.bk[b] = bk;
    }
    if (t == 0) p.hdr->head_ticket = 0u;
}

int launch_length_head(const HeadParams& p, void* stream) {
    dim3 grid((p.B + kHeadTileB - 1) / kHeadTileB, (p.M + kHeadTileM - 1) / kHeadTileM, 1);
    length_head_kernel<<<grid, kWarps * 32, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return static_cast<int>(cudaGetLastError());
}

// ------------------------------------------------------------------------------------------
// bounded-wait self test: one thread waits on a barrier that nothing completes
// ------------------------------------------------------------------------------------------
__global__ void wait_timeout_selftest_kernel(WsHeader* hdr, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // phase 0 never completes: its single expected arrival is never made
        if (!mbar_wait_bounded(&bar, 0, limit_ns)) set_device_error(&hdr->status, SVD_ERR_TIMEOUT);
    }
}

int launch_wait_timeout_selftest(WsHeader* hdr, uint64_t limit_ns, void* stream) {
    wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(hdr, limit_ns);
    return static_cast<int>(cudaGetLastError());
}

}  // namespace svd
