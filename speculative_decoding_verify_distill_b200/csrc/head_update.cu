// head_update.cu -- one online update step of the adaptive length head: the backward of
//   l = (1/B) sum_b (bhat_b - a*_b)^2,   bhat_b = sigmoid(w2 . relu(W1 h_b + b1) + b2),
// and an AdamW step on fp32 master weights, refreshing the bf16 copies the forward serves.
//
// AdaFlash trains its length head online on the squared error between the predicted and the
// observed acceptance rate (Pith verdict record, skeptic_critique.load_bearing_attack), with
// AdamW at learning rate 2e-4 (Pith review page, Axiom & Free-Parameter Ledger).  AdamW is
// Loshchilov & Hutter, "Decoupled Weight Decay Regularization" (ICLR 2019), in the order
// torch.optim.AdamW applies it: theta *= 1 - lr*wd, then the bias-corrected moment step.
//
// Kernels: the forward, with its pre-activations stored, is the length-head kernel; the whole
// backward and the AdamW steps are one kernel (head_back_kernel below): dl/dW1 = E^T h
// ([M,B] x [B,H], 0.27 GFLOP at B=128, H=4096, M=256) on the tensor cores (mma.sync m16n8k16,
// fp32 accumulation), with E formed on the fly from the stored pre-activations and fed as the
// sum of three bf16 operands (hi = RN(e), mid = RN(e - hi), lo = RN(e - hi - mid): e h to
// within 2^-24 relative, since h is exact in bf16); the w2, b1, b2 gradients and their AdamW
// steps in the last CTA.  Accuracy
// matters here because Adam's first step is lr * g / |g|: the sign of a small gradient decides
// the direction of the step.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <cmath>

#include "svd_internal.h"

namespace svd {

namespace {

constexpr int kTile = 64;        // back2 output tile: 64 units x 64 hidden columns

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}
__device__ __forceinline__ uint16_t f32_to_bf16_rne(float x) {
    __nv_bfloat16 r = __float2bfloat16_rn(x);
    return *reinterpret_cast<uint16_t*>(&r);
}

// One AdamW update of one parameter; returns the new value and updates the moments.
__device__ __forceinline__ float adamw(float theta, float g, float& m, float& v,
                                       const HeadUpdateParams& p) {
    theta *= 1.f - p.lr * p.wd;
    m = p.beta1 * m + (1.f - p.beta1) * g;
    v = p.beta2 * v + (1.f - p.beta2) * g * g;
    const float mhat = m / p.bc1, vhat = v / p.bc2;
    return theta - p.lr * mhat / (sqrtf(vhat) + p.eps);
}

__device__ __forceinline__ float delta_of(const HeadUpdateParams& p, int b) {
    const float bh = __ldg(p.bhat + b);
    return (2.f / static_cast<float>(p.B)) * (bh - __ldg(p.label + b)) * bh * (1.f - bh);
}

// One kernel for the whole backward.  CTA (jt, mt) owns the 64 x 64 block of W1 (units
// m0 .. m0 + 63, hidden columns j0 .. j0 + 63).  Per chunk of 64 sequences it forms
// e_bm = delta_b w2_m [u_bm > 0] for its units in shared memory (from the forward's stored
// pre-activations u, so no separate pass writes e), stages the matching h columns, and its
// eight warps add E^T h into four 16 x 8 tiles each on the tensor cores.  The AdamW step on its
// block of W1 follows, row by row (16-byte loads and stores).  The CTAs of column 0 also sum the w2 and b1
// gradients of their units over the sequences (four threads per unit, combined in order) into
// the workspace; the last CTA to finish (atomic ticket) applies AdamW to w2, b1 and b2 and forms
// the loss -- only then, because every CTA reads the forward's w2 to form e.
constexpr int kBC = 64;          // sequences per chunk
constexpr int kHLd = kTile + 8;  // bf16 row pitch of the staged h tile (16-byte rows)
constexpr int kELd = kTile + 4;  // fp32 row pitch of the e tile (fragment reads on distinct banks)

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               const uint32_t (&b)[2]) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// Two fp32 to bf16 with round-to-nearest-even, the first in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
    __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&r);
}

__global__ void __launch_bounds__(256) head_back_kernel(const HeadUpdateParams p) {
    __shared__ __align__(16) float se[kBC][kELd];         // e[b0 + r, m0 + c]
    __shared__ __align__(16) uint16_t sh[kBC][kHLd];      // h[b0 + r, j0 + c]
    __shared__ float sdelta[kBC];
    __shared__ float sg[2][4][kTile];                     // w2 / b1 gradient partials
    __shared__ int last;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    // tensor-core tiles: warp w owns hidden units m0 + 16 (w & 3) .. + 15 and columns
    // j0 + 32 (w >> 2) .. + 31, i.e. four 16 x 8 output tiles
    const int g = lane >> 2, tq = lane & 3;
    const int mb = (warp & 3) * 16, jb = (warp >> 2) * 32;
    const int j0 = blockIdx.x * kTile, m0 = blockIdx.y * kTile;
    const bool col0 = blockIdx.x == 0;
    // e-tile role: unit c = t % 64, rows r = t / 64, t / 64 + 4, ...
    const int ec = t & (kTile - 1), er = t >> 6;
    const bool ulive = m0 + ec < p.M;
    const float w2f = ulive ? bf16_to_f32(__ldg(p.w2 + m0 + ec)) : 0.f;   // the forward's weight
    const bool hvec = (p.H % 8 == 0) && ((reinterpret_cast<uintptr_t>(p.h) & 15) == 0) && (j0 + kTile <= p.H);
    // The epilogue's master weights and moments (3 x 64 rows x 256 bytes) and the second
    // chunk's operands go to L2 now, so that their loads later find them there instead of in HBM.
    for (int x = t; x < 3 * kTile * 2; x += 256) {
        const int arr = x / (kTile * 2), r = (x / 2) % kTile, half = x & 1;
        const int m = m0 + r;
        if (m < p.M && j0 + 32 * half < p.H) {
            const float* base = arr == 0 ? p.W1m : (arr == 1 ? p.mW1 : p.vW1);
            asm volatile("prefetch.global.L2 [%0];" ::"l"(base + static_cast<size_t>(m) * p.H + j0 + 32 * half));
        }
    }
    for (int b = kBC + t; b < p.B; b += 256) {
        asm volatile("prefetch.global.L2 [%0];" ::"l"(p.h + static_cast<size_t>(b) * p.H + j0));
        for (int c = 0; c < kTile && m0 + c < p.M; c += 32)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(p.u + static_cast<size_t>(b) * p.M + m0 + c));
    }
    float gw = 0.f, gb = 0.f;
    float acc[4][4];   // [tile nt][(g, 2tq), (g, 2tq + 1), (g + 8, 2tq), (g + 8, 2tq + 1)]
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) acc[i][jj] = 0.f;
    for (int b0 = 0; b0 < p.B; b0 += kBC) {
        const int nb = min(kBC, p.B - b0);
        if (t < kBC) sdelta[t] = t < nb ? delta_of(p, b0 + t) : 0.f;
        // h columns of the chunk: one 16-byte vector per (row, 8 columns)
        for (int x = t; x < kBC * (kTile / 8); x += 256) {
            const int r = x / (kTile / 8), c8 = (x % (kTile / 8)) * 8;
            const int b = b0 + r;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (b < p.B) {
                const uint16_t* src = p.h + static_cast<size_t>(b) * p.H + j0 + c8;
                if (hvec) {
                    v = __ldg(reinterpret_cast<const uint4*>(src));
                } else {
                    uint16_t e8[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) e8[q] = (j0 + c8 + q < p.H) ? __ldg(src + q) : uint16_t(0);
                    v = make_uint4(e8[0] | (uint32_t(e8[1]) << 16), e8[2] | (uint32_t(e8[3]) << 16),
                                   e8[4] | (uint32_t(e8[5]) << 16), e8[6] | (uint32_t(e8[7]) << 16));
                }
            }
            *reinterpret_cast<uint4*>(&sh[r][c8]) = v;
        }
        __syncthreads();
        // e of the chunk (and, in column 0, the w2 / b1 gradient partials in row order); the
        // thread's 16 pre-activations are loaded before any is used
        {
            constexpr int kRows = kBC / 4;
            float uu[kRows];
#pragma unroll
            for (int q = 0; q < kRows; ++q) {
                const int r = er + 4 * q;
                uu[q] = (r < nb && ulive) ? __ldcg(p.u + static_cast<size_t>(b0 + r) * p.M + m0 + ec) : 0.f;
            }
#pragma unroll
            for (int q = 0; q < kRows; ++q) {
                const int r = er + 4 * q;
                float ev = 0.f;
                if (r < nb && ulive) {
                    const float d = sdelta[r];
                    ev = uu[q] > 0.f ? d * w2f : 0.f;
                    if (col0) {
                        gw += d * fmaxf(uu[q], 0.f);
                        gb += ev;
                    }
                }
                se[r][ec] = ev;
            }
        }
        __syncthreads();
        // dW1 tile += E^T h over the chunk's sequences, 16 at a time, on the tensor cores
        // (mma.sync m16n8k16, fp32 accumulation).  E is fp32: it enters as the sum of three
        // bf16 operands, hi = RN(e), mid = RN(e - hi), lo = RN(e - hi - mid), whose products
        // with the exact bf16 h add up to e h within 2^-24 relative, as fine as e itself;
        // rows past the batch hold zeros.
        for (int kb = 0; kb < nb; kb += 16) {
            uint32_t ahi[4], amid[4], alo[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                // a0: (row g, k 2tq..2tq+1), a1: row g + 8, a2: k + 8, a3: both
                const int m = mb + g + ((q & 1) ? 8 : 0);
                const int r = kb + 2 * tq + ((q & 2) ? 8 : 0);
                const float e0 = se[r][m], e1 = se[r + 1][m];
                const uint32_t hi = pack_bf16x2_rn(e0, e1);
                const float r0 = e0 - __uint_as_float(hi << 16), r1 = e1 - __uint_as_float(hi & 0xffff0000u);
                const uint32_t mid = pack_bf16x2_rn(r0, r1);
                ahi[q] = hi;
                amid[q] = mid;
                alo[q] = pack_bf16x2_rn(r0 - __uint_as_float(mid << 16), r1 - __uint_as_float(mid & 0xffff0000u));
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int j = jb + nt * 8 + g;
                const int r = kb + 2 * tq;
                uint32_t bf[2];
                bf[0] = static_cast<uint32_t>(sh[r][j]) | (static_cast<uint32_t>(sh[r + 1][j]) << 16);
                bf[1] = static_cast<uint32_t>(sh[r + 8][j]) | (static_cast<uint32_t>(sh[r + 9][j]) << 16);
                // smallest part first, so the larger parts are added to an accumulator that
                // already holds the small corrections
                mma_bf16_16816(acc[nt], alo, bf);
                mma_bf16_16816(acc[nt], amid, bf);
                mma_bf16_16816(acc[nt], ahi, bf);
            }
        }
        __syncthreads();
    }
    // The gradient tile goes through shared memory (the e tile's buffer) so that the AdamW
    // epilogue walks whole rows of W1: each half-warp takes one row's 64 columns as 16-byte
    // vectors, 256 contiguous bytes of every master and moment array per row.
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int r = mb + g + 8 * half, c = jb + nt * 8 + 2 * tq;
            se[r][c] = acc[nt][2 * half];
            se[r][c + 1] = acc[nt][2 * half + 1];
        }
    }
    __syncthreads();
    const bool wvec = (p.H % 4 == 0) && (j0 + kTile <= p.H) &&
                      (((reinterpret_cast<uintptr_t>(p.W1m) | reinterpret_cast<uintptr_t>(p.mW1) |
                         reinterpret_cast<uintptr_t>(p.vW1)) & 15) == 0) &&
                      ((reinterpret_cast<uintptr_t>(p.W1) & 7) == 0);
    {
        const int c = (t & 15) * 4;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int r = (t >> 4) + 16 * q;
            const int m = m0 + r;
            if (m >= p.M) continue;
            const size_t o = static_cast<size_t>(m) * p.H + j0 + c;
            const float4 gv = *reinterpret_cast<const float4*>(&se[r][c]);
            if (wvec) {
                const float4 wm = *reinterpret_cast<const float4*>(p.W1m + o);
                float4 mm = *reinterpret_cast<const float4*>(p.mW1 + o);
                float4 vv = *reinterpret_cast<const float4*>(p.vW1 + o);
                float4 w;
                w.x = adamw(wm.x, gv.x, mm.x, vv.x, p);
                w.y = adamw(wm.y, gv.y, mm.y, vv.y, p);
                w.z = adamw(wm.z, gv.z, mm.z, vv.z, p);
                w.w = adamw(wm.w, gv.w, mm.w, vv.w, p);
                *reinterpret_cast<float4*>(p.W1m + o) = w;
                *reinterpret_cast<float4*>(p.mW1 + o) = mm;
                *reinterpret_cast<float4*>(p.vW1 + o) = vv;
                *reinterpret_cast<uint2*>(p.W1 + o) =
                    make_uint2(f32_to_bf16_rne(w.x) | (static_cast<uint32_t>(f32_to_bf16_rne(w.y)) << 16),
                               f32_to_bf16_rne(w.z) | (static_cast<uint32_t>(f32_to_bf16_rne(w.w)) << 16));
            } else {
                const float gg[4] = {gv.x, gv.y, gv.z, gv.w};
                for (int jj = 0; jj < 4; ++jj) {
                    if (j0 + c + jj >= p.H) break;
                    float mm = p.mW1[o + jj], vv = p.vW1[o + jj];
                    const float w = adamw(p.W1m[o + jj], gg[jj], mm, vv, p);
                    p.W1m[o + jj] = w;
                    p.mW1[o + jj] = mm;
                    p.vW1[o + jj] = vv;
                    p.W1[o + jj] = f32_to_bf16_rne(w);
                }
            }
        }
    }
    // column 0: this tile's units' w2 / b1 gradients (four row partials per unit, in order)
    if (col0) {
        sg[0][er][ec] = gw;
        sg[1][er][ec] = gb;
        __syncthreads();
        if (t < kTile && m0 + t < p.M) {
            float a = 0.f, c = 0.f;
            for (int q = 0; q < 4; ++q) { a += sg[0][q][t]; c += sg[1][q][t]; }
            p.e[m0 + t] = a;                 // workspace: [M] w2 gradient, then [M] b1 gradient
            p.e[p.M + m0 + t] = c;
        }
    }
    // the last CTA updates w2, b1, b2 (every CTA has read the forward's w2 by now)
    __threadfence();
    __syncthreads();
    if (t == 0) {
        const uint32_t old = atomicAdd(p.ticket, 1u);
        last = (old + 1u == gridDim.x * gridDim.y) ? 1 : 0;
    }
    __syncthreads();
    if (!last) return;
    __threadfence();
    for (int m = t; m < p.M; m += 256) {
        const float gwm = __ldcg(p.e + m), gbm = __ldcg(p.e + p.M + m);
        float mm = p.mw2[m], vv = p.vw2[m];
        const float w2n = adamw(p.w2m[m], gwm, mm, vv, p);
        p.w2m[m] = w2n;
        p.mw2[m] = mm;
        p.vw2[m] = vv;
        p.w2[m] = f32_to_bf16_rne(w2n);
        mm = p.mb1[m];
        vv = p.vb1[m];
        p.b1[m] = adamw(p.b1[m], gbm, mm, vv, p);
        p.mb1[m] = mm;
        p.vb1[m] = vv;
    }
    if (t < 32) {
        // loss and b2 gradient: lane l adds sequences l, l + 32, ... in order, then a butterfly
        float ls = 0.f, gs = 0.f;
#pragma unroll 4
        for (int b = t; b < p.B; b += 32) {
            const float e = __ldg(p.bhat + b) - __ldg(p.label + b);
            ls += e * e;
            gs += delta_of(p, b);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            ls += __shfl_xor_sync(0xffffffffu, ls, o);
            gs += __shfl_xor_sync(0xffffffffu, gs, o);
        }
        if (t == 0) {
            *p.loss = ls / static_cast<float>(p.B);
            float mm = *p.mb2, vv = *p.vb2;
            *p.b2 = adamw(*p.b2, gs, mm, vv, p);
            *p.mb2 = mm;
            *p.vb2 = vv;
            *p.ticket = 0u;
        }
    }
}

}  // namespace

int launch_head_update(const HeadUpdateParams& p, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    dim3 grid((p.H + kTile - 1) / kTile, (p.M + kTile - 1) / kTile);
    head_back_kernel<<<grid, 256, 0, st>>>(p);
    return static_cast<int>(cudaGetLastError());
}

}  // namespace svd
