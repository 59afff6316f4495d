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
// Kernels (the forward, with its pre-activations stored, is the length-head kernel):
//   back1: per sequence delta_b = (2/B)(bhat_b - a*_b) bhat_b (1 - bhat_b), staged in shared
//          memory by chunks; per unit m the gradients of w2 and b1 and e_bm = delta_b w2_m
//          [u_bm > 0] (32 units per CTA, 8 warps over the sequences, partials added in a fixed
//          order); CTA 0 also forms the loss and the b2 gradient.  AdamW on w2, b1, b2.
//   back2: dl/dW1 = E^T h ([M,B] x [B,H], 0.27 GFLOP at B=128, H=4096, M=256) on fp32 CUDA
//          cores with shared-memory tiles, each output summed over b in order; AdamW on W1 in
//          the epilogue.  Too small and too precision-sensitive (Adam's first step is
//          lr * g / |g|) for bf16 tensor-core operands.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <cmath>

#include "svd_internal.h"

namespace svd {

namespace {

constexpr int kBack1Threads = 256;
constexpr int kTile = 64;        // back2 output tile: 64 units x 64 hidden columns
constexpr int kBChunk = 32;      // sequences staged per round

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

// One CTA per 32 hidden units (lane = unit); its 8 warps take every 8th sequence, so each thread
// walks B/8 sequences with independent loads, and the warps' partial sums are added in order.
__global__ void __launch_bounds__(kBack1Threads) head_back1_kernel(const HeadUpdateParams p) {
    constexpr int kW = kBack1Threads / 32;
    constexpr int kChunk = 1024;
    __shared__ float sdelta[kChunk];                 // delta_b for a chunk of sequences
    __shared__ float sred[2][kW][32];
    __shared__ float sloss[2][kW];
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int m = blockIdx.x * 32 + lane;
    const bool live = m < p.M;
    const float w2 = live ? bf16_to_f32(p.w2[m]) : 0.f;   // the forward's weight
    float gw = 0.f, gb = 0.f, l = 0.f, g2 = 0.f;
    for (int b0 = 0; b0 < p.B; b0 += kChunk) {
        const int nb = min(kChunk, p.B - b0);
        for (int r = t; r < nb; r += kBack1Threads) {
            const int b = b0 + r;
            const float d = delta_of(p, b);
            sdelta[r] = d;
            if (blockIdx.x == 0) {          // loss and b2 gradient: fixed per-thread strides
                const float e = __ldg(p.bhat + b) - __ldg(p.label + b);
                l += e * e;
                g2 += d;
            }
        }
        __syncthreads();
        if (live) {
            // this warp's sequences in order, kGroup at a time: the group's loads are all issued
            // before its stores (which the compiler may not move loads across)
            constexpr int kGroup = 8;
            for (int r0 = warp; r0 < nb; r0 += kW * kGroup) {
                float u[kGroup];
#pragma unroll
                for (int q = 0; q < kGroup; ++q) {
                    const int r = r0 + q * kW;
                    u[q] = r < nb ? p.u[static_cast<size_t>(b0 + r) * p.M + m] : 0.f;
                }
#pragma unroll
                for (int q = 0; q < kGroup; ++q) {
                    const int r = r0 + q * kW;
                    if (r < nb) {
                        const float d = sdelta[r];
                        const float ev = u[q] > 0.f ? d * w2 : 0.f;
                        gw += d * fmaxf(u[q], 0.f);
                        gb += ev;
                        p.e[static_cast<size_t>(b0 + r) * p.M + m] = ev;
                    }
                }
            }
        }
        __syncthreads();
    }
    sred[0][warp][lane] = gw;
    sred[1][warp][lane] = gb;
    if (blockIdx.x == 0) {
        // fixed-order reduction of the loss / b2 partials: warp butterflies, then warps in order
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            l += __shfl_xor_sync(0xffffffffu, l, o);
            g2 += __shfl_xor_sync(0xffffffffu, g2, o);
        }
        if (lane == 0) { sloss[0][warp] = l; sloss[1][warp] = g2; }
    }
    __syncthreads();
    if (blockIdx.x == 0 && t == 0) {
        float ls = 0.f, gs = 0.f;
        for (int q = 0; q < kW; ++q) { ls += sloss[0][q]; gs += sloss[1][q]; }
        *p.loss = ls / static_cast<float>(p.B);
        float mm = *p.mb2, vv = *p.vb2;
        *p.b2 = adamw(*p.b2, gs, mm, vv, p);
        *p.mb2 = mm;
        *p.vb2 = vv;
    }
    if (warp != 0 || !live) return;
    gw = 0.f;
    gb = 0.f;
    for (int q = 0; q < kW; ++q) { gw += sred[0][q][lane]; gb += sred[1][q][lane]; }
    float mm = p.mw2[m], vv = p.vw2[m];
    const float w2n = adamw(p.w2m[m], gw, mm, vv, p);
    p.w2m[m] = w2n;
    p.mw2[m] = mm;
    p.vw2[m] = vv;
    p.w2[m] = f32_to_bf16_rne(w2n);
    mm = p.mb1[m];
    vv = p.vb1[m];
    p.b1[m] = adamw(p.b1[m], gb, mm, vv, p);
    p.mb1[m] = mm;
    p.vb1[m] = vv;
}

__global__ void __launch_bounds__(256) head_back2_kernel(const HeadUpdateParams p) {
    __shared__ float se[kBChunk][kTile];        // e[b, m0 + i]
    __shared__ float sh[kBChunk][kTile + 1];    // h[b, j0 + j]
    const int t = threadIdx.x;
    const int tx = t & 15, ty = t >> 4;         // outputs (m0 + 4ty + i, j0 + 4tx + jj)
    const int j0 = blockIdx.x * kTile, m0 = blockIdx.y * kTile;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) acc[i][jj] = 0.f;
    for (int b0 = 0; b0 < p.B; b0 += kBChunk) {
        for (int x = t; x < kBChunk * kTile; x += 256) {
            const int r = x / kTile, c = x % kTile;
            const int b = b0 + r;
            se[r][c] = (b < p.B && m0 + c < p.M) ? p.e[static_cast<size_t>(b) * p.M + m0 + c] : 0.f;
            sh[r][c] = (b < p.B && j0 + c < p.H) ? bf16_to_f32(__ldg(p.h + static_cast<size_t>(b) * p.H + j0 + c)) : 0.f;
        }
        __syncthreads();
        const int nb = min(kBChunk, p.B - b0);
        for (int r = 0; r < nb; ++r) {   // sequences in order
            float ev[4], hv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) ev[i] = se[r][4 * ty + i];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) hv[jj] = sh[r][4 * tx + jj];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) acc[i][jj] = fmaf(ev[i], hv[jj], acc[i][jj]);
        }
        __syncthreads();
    }
    // AdamW epilogue on this thread's 4 x 4 block of W1: every master weight and moment is
    // loaded before the first store, so the 48 loads are in flight together
    float wm[4][4], mm[4][4], vv[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + 4 * ty + i;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const int j = j0 + 4 * tx + jj;
            const bool in = m < p.M && j < p.H;
            const size_t o = static_cast<size_t>(m) * p.H + j;
            wm[i][jj] = in ? p.W1m[o] : 0.f;
            mm[i][jj] = in ? p.mW1[o] : 0.f;
            vv[i][jj] = in ? p.vW1[o] : 0.f;
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + 4 * ty + i;
        if (m >= p.M) continue;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const int j = j0 + 4 * tx + jj;
            if (j >= p.H) continue;
            const size_t o = static_cast<size_t>(m) * p.H + j;
            const float w = adamw(wm[i][jj], acc[i][jj], mm[i][jj], vv[i][jj], p);
            p.W1m[o] = w;
            p.mW1[o] = mm[i][jj];
            p.vW1[o] = vv[i][jj];
            p.W1[o] = f32_to_bf16_rne(w);
        }
    }
}

}  // namespace

int launch_head_update(const HeadUpdateParams& p, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    head_back1_kernel<<<(p.M + 31) / 32, kBack1Threads, 0, st>>>(p);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return static_cast<int>(err);
    dim3 grid((p.H + kTile - 1) / kTile, (p.M + kTile - 1) / kTile);
    head_back2_kernel<<<grid, 256, 0, st>>>(p);
    return static_cast<int>(cudaGetLastError());
}

}  // namespace svd
