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
// ([M,B] x [B,H], 0.27 GFLOP at B=128, H=4096, M=256) on fp32 CUDA cores with shared-memory
// tiles, each output summed over b in order, with E formed on the fly from the stored
// pre-activations; the w2, b1, b2 gradients and their AdamW steps in the last CTA.  fp32
// throughout: Adam's first step is lr * g / |g|, so the sign of small gradients matters, and the
// contraction is too small for tensor-core tiles to pay.
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
// pre-activations u, so no separate pass writes e), stages the matching h columns, and adds
// e_bm h_bj into its 4 x 4 outputs per thread, sequences in order.  The AdamW step on its block
// of W1 follows (16-byte loads and stores).  The CTAs of column 0 also sum the w2 and b1
// gradients of their units over the sequences (four threads per unit, combined in order) into
// the workspace; the last CTA to finish (atomic ticket) applies AdamW to w2, b1 and b2 and forms
// the loss -- only then, because every CTA reads the forward's w2 to form e.
constexpr int kBC = 64;          // sequences per chunk
constexpr int kHLd = kTile + 8;  // bf16 row pitch of the staged h tile (16-byte rows)

__global__ void __launch_bounds__(256) head_back_kernel(const HeadUpdateParams p) {
    __shared__ __align__(16) float se[kBC][kTile];        // e[b0 + r, m0 + c]
    __shared__ __align__(16) uint16_t sh[kBC][kHLd];      // h[b0 + r, j0 + c]
    __shared__ float sdelta[kBC];
    __shared__ float sg[2][4][kTile];                     // w2 / b1 gradient partials
    __shared__ int last;
    const int t = threadIdx.x;
    const int tx = t & 15, ty = t >> 4;         // outputs (m0 + 4ty + i, j0 + 4tx + jj)
    const int j0 = blockIdx.x * kTile, m0 = blockIdx.y * kTile;
    const bool col0 = blockIdx.x == 0;
    // e-tile role: unit c = t % 64, rows r = t / 64, t / 64 + 4, ...
    const int ec = t & (kTile - 1), er = t >> 6;
    const bool ulive = m0 + ec < p.M;
    const float w2f = ulive ? bf16_to_f32(__ldg(p.w2 + m0 + ec)) : 0.f;   // the forward's weight
    const bool hvec = (p.H % 8 == 0) && ((reinterpret_cast<uintptr_t>(p.h) & 15) == 0) && (j0 + kTile <= p.H);
    float gw = 0.f, gb = 0.f;
    float acc[4][4];
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
        for (int r = 0; r < nb; ++r) {   // sequences in order
            const float4 e4 = *reinterpret_cast<const float4*>(&se[r][4 * ty]);
            const uint2 h4 = *reinterpret_cast<const uint2*>(&sh[r][4 * tx]);
            const float ev[4] = {e4.x, e4.y, e4.z, e4.w};
            const float hv[4] = {__uint_as_float(h4.x << 16), __uint_as_float(h4.x & 0xffff0000u),
                                 __uint_as_float(h4.y << 16), __uint_as_float(h4.y & 0xffff0000u)};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) acc[i][jj] = fmaf(ev[i], hv[jj], acc[i][jj]);
        }
        __syncthreads();
    }
    // AdamW epilogue on this thread's 4 x 4 block of W1: every master weight and moment is
    // loaded before the first store
    const bool wvec = (p.H % 4 == 0) && (j0 + 4 * tx + 4 <= p.H) &&
                      (((reinterpret_cast<uintptr_t>(p.W1m) | reinterpret_cast<uintptr_t>(p.mW1) |
                         reinterpret_cast<uintptr_t>(p.vW1)) & 15) == 0) &&
                      ((reinterpret_cast<uintptr_t>(p.W1) & 7) == 0);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + 4 * ty + i;
        if (m >= p.M) continue;
        const size_t o = static_cast<size_t>(m) * p.H + j0 + 4 * tx;
        if (wvec) {
            float4 wm = *reinterpret_cast<const float4*>(p.W1m + o);
            float4 mm = *reinterpret_cast<const float4*>(p.mW1 + o);
            float4 vv = *reinterpret_cast<const float4*>(p.vW1 + o);
            float w[4] = {wm.x, wm.y, wm.z, wm.w}, m1[4] = {mm.x, mm.y, mm.z, mm.w},
                  v1[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) w[jj] = adamw(w[jj], acc[i][jj], m1[jj], v1[jj], p);
            *reinterpret_cast<float4*>(p.W1m + o) = make_float4(w[0], w[1], w[2], w[3]);
            *reinterpret_cast<float4*>(p.mW1 + o) = make_float4(m1[0], m1[1], m1[2], m1[3]);
            *reinterpret_cast<float4*>(p.vW1 + o) = make_float4(v1[0], v1[1], v1[2], v1[3]);
            const uint2 wb = make_uint2(f32_to_bf16_rne(w[0]) | (uint32_t(f32_to_bf16_rne(w[1])) << 16),
                                        f32_to_bf16_rne(w[2]) | (uint32_t(f32_to_bf16_rne(w[3])) << 16));
            *reinterpret_cast<uint2*>(p.W1 + o) = wb;
        } else {
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                if (j0 + 4 * tx + jj >= p.H) continue;
                float mm = p.mW1[o + jj], vv = p.vW1[o + jj];
                const float w = adamw(p.W1m[o + jj], acc[i][jj], mm, vv, p);
                p.W1m[o + jj] = w;
                p.mW1[o + jj] = mm;
                p.vW1[o + jj] = vv;
                p.W1[o + jj] = f32_to_bf16_rne(w);
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
    if (t == 0) {
        // loss and b2 gradient over the sequences in order
        float ls = 0.f, gs = 0.f;
        for (int b = 0; b < p.B; ++b) {
            const float e = __ldg(p.bhat + b) - __ldg(p.label + b);
            ls += e * e;
            gs += delta_of(p, b);
        }
        *p.loss = ls / static_cast<float>(p.B);
        float mm = *p.mb2, vv = *p.vb2;
        *p.b2 = adamw(*p.b2, gs, mm, vv, p);
        *p.mb2 = mm;
        *p.vb2 = vv;
        *p.ticket = 0u;
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
