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
// within 2^-24 relative, since h is exact in bf16); the w2 and b1 gradients and their AdamW
// steps in the CTAs of column 0, b2 and the loss in CTA (0, 0).  Accuracy
// matters here because Adam's first step is lr * g / |g|: the sign of a small gradient decides
// the direction of the step.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>
#include <mutex>
#include <vector>

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

// One AdamW update of one parameter; returns the new value and updates the moments.  The bias
// corrections are folded into two per-step constants, as torch.optim.AdamW folds them:
// theta - (lr / bc1) m / (sqrt(v) / sqrt(bc2) + eps), one division per parameter.
__device__ __forceinline__ float adamw(float theta, float g, float& m, float& v,
                                       const HeadUpdateParams& p) {
    theta *= 1.f - p.lr * p.wd;
    m = p.beta1 * m + (1.f - p.beta1) * g;
    v = p.beta2 * v + (1.f - p.beta2) * g * g;
    return theta - p.step_size * m / (sqrtf(v) * p.rsqrt_bc2 + p.eps);
}

__device__ __forceinline__ float delta_of(const HeadUpdateParams& p, int b) {
    const float bh = __ldg(p.bhat + b);
    return (2.f / static_cast<float>(p.B)) * (bh - __ldg(p.label + b)) * bh * (1.f - bh);
}

// One kernel for the whole backward.  CTA (jt, mt) owns the 64 x 64 block of W1 (units
// m0 .. m0 + 63, hidden columns j0 .. j0 + 63).  It stages the h columns and pre-activations u
// of a chunk of 128 sequences in shared memory by asynchronous 16-byte copies, and once the
// first chunk has landed it starts the copies of its block of the fp32 master weights and both
// moments, which fly while the tensor cores run.  Per chunk its eight warps add E^T h on the
// tensor cores (each warp 16 units x 64 columns over half of the sequences), forming
// e_bm = delta_b w2_m [u_bm > 0] from the staged u as they build their operand fragments; the
// two halves are added, and the AdamW step on the block of W1 follows, row by row, from the
// staged masters and moments.  The CTAs of column 0 also sum the w2 and b1 gradients of their
// units over the sequences (in the same fragments; per warp the four lanes of a unit combined
// by a fixed butterfly, then the two halves) and step the fp32 masters and moments of w2 and
// b1 themselves (nothing else in the kernel reads them); only the bf16 w2, which every CTA
// reads to form e, waits for the last CTA to take an atomic ticket (taken after the MMA, before
// the W1 stores), which copies it in.  CTA (0, 0) forms the loss and steps b2 while its first
// copies are in flight.
constexpr int kBC = 128;         // sequences per chunk (one chunk up to B = 128)
constexpr int kHLd = kTile + 8;  // bf16 row pitch of the staged h tile (16-byte rows)
constexpr int kELd = kTile + 4;  // fp32 row pitch of the u tile (fragment reads on distinct banks)
constexpr size_t kBackSmem = sizeof(float) * kBC * kELd + sizeof(uint16_t) * kBC * kHLd +
                             sizeof(float) * 3 * kTile * kTile;

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
// 16-byte asynchronous global -> shared copy; src_bytes = 0 fills the 16 bytes with zeros.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
// Four transposed 8 x 8 bf16 matrices from shared memory (lane l names row l % 8 of matrix l / 8).
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], const void* row) {
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(row));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(a));
}

__global__ void __launch_bounds__(256, 2) head_back_kernel(const HeadUpdateParams p) {
    // dynamic shared memory: u[b0 + r, m0 + c] fp32, h[b0 + r, j0 + c] bf16, then the
    // W1 block's fp32 master, first and second moment [3][64][64]
    extern __shared__ __align__(16) unsigned char back_smem[];
    float (*se)[kELd] = reinterpret_cast<float (*)[kELd]>(back_smem);
    uint16_t (*sh)[kHLd] = reinterpret_cast<uint16_t (*)[kHLd]>(back_smem + sizeof(float) * kBC * kELd);
    float (*sw)[kTile][kTile] = reinterpret_cast<float (*)[kTile][kTile]>(
        back_smem + sizeof(float) * kBC * kELd + sizeof(uint16_t) * kBC * kHLd);
    __shared__ float sdelta[kBC];
    __shared__ float sg[2][2][kTile];                     // [half][w2 / b1] gradients of the units
    __shared__ float sp[6][kTile];                        // column 0: w2 / b1 masters and moments
    __shared__ int last;
    // launched as a programmatic dependent of the preceding kernel: nothing is read before it
    // has finished
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    // tensor-core tiles: warp w owns hidden units m0 + 16 (w & 3) .. + 15 and all 64 columns,
    // i.e. eight 16 x 8 output tiles, over half of the sequences (16-row steps kh, kh + 2, ...
    // with kh = w >> 2); the two halves are added at the end.  Every e operand is thus split
    // into its bf16 parts once.
    const int g = lane >> 2, tq = lane & 3;
    const int mb = (warp & 3) * 16, kh = warp >> 2;
    const int j0 = blockIdx.x * kTile, m0 = blockIdx.y * kTile;
    const bool col0 = blockIdx.x == 0;
    const bool hvec = (p.H % 8 == 0) && ((reinterpret_cast<uintptr_t>(p.h) & 15) == 0) && (j0 + kTile <= p.H);
    const bool uvec = (p.M % 4 == 0) && ((reinterpret_cast<uintptr_t>(p.u) & 15) == 0) && (m0 + kTile <= p.M);
    const bool wvec = (p.H % 4 == 0) && (j0 + kTile <= p.H) &&
                      (((reinterpret_cast<uintptr_t>(p.W1m) | reinterpret_cast<uintptr_t>(p.mW1) |
                         reinterpret_cast<uintptr_t>(p.vW1)) & 15) == 0) &&
                      ((reinterpret_cast<uintptr_t>(p.W1) & 7) == 0);

    // h and u of a chunk into shared memory: asynchronous copies where the rows are whole
    // 16-byte vectors, plain loads otherwise; rows past the batch are zeros
    auto stage_chunk = [&](int b0) {
        for (int x = t; x < kBC * (kTile / 8); x += 256) {
            const int r = x / (kTile / 8), c8 = (x % (kTile / 8)) * 8;
            const int b = b0 + r;
            const uint16_t* src = p.h + static_cast<size_t>(b < p.B ? b : 0) * p.H + j0 + c8;
            if (hvec) {
                cp_async16(&sh[r][c8], src, b < p.B ? 16u : 0u);
            } else {
                uint16_t e8[8];
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    e8[q] = (b < p.B && j0 + c8 + q < p.H) ? __ldg(src + q) : uint16_t(0);
                *reinterpret_cast<uint4*>(&sh[r][c8]) =
                    make_uint4(e8[0] | (uint32_t(e8[1]) << 16), e8[2] | (uint32_t(e8[3]) << 16),
                               e8[4] | (uint32_t(e8[5]) << 16), e8[6] | (uint32_t(e8[7]) << 16));
            }
        }
        for (int x = t; x < kBC * (kTile / 4); x += 256) {
            const int r = x / (kTile / 4), c4 = (x % (kTile / 4)) * 4;
            const int b = b0 + r;
            const float* src = p.u + static_cast<size_t>(b < p.B ? b : 0) * p.M + m0 + c4;
            if (uvec) {
                cp_async16(&se[r][c4], src, b < p.B ? 16u : 0u);
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    se[r][c4 + q] = (b < p.B && m0 + c4 + q < p.M) ? __ldcg(src + q) : 0.f;
            }
        }
        cp_async_commit();
    };
    stage_chunk(0);
    // delta of the first chunk's sequences while its copies fly
    for (int r = t; r < kBC; r += 256) sdelta[r] = r < min(kBC, p.B) ? delta_of(p, r) : 0.f;
    if (col0 && t < kTile && m0 + t < p.M) {
        // column 0: its units' w2 and b1 masters and moments, for the AdamW steps after the MMA
        const int m = m0 + t;
        sp[0][t] = p.w2m[m];
        sp[1][t] = p.mw2[m];
        sp[2][t] = p.vw2[m];
        sp[3][t] = p.b1[m];
        sp[4][t] = p.mb1[m];
        sp[5][t] = p.vb1[m];
    }
    // the forward's w2 of this thread's two fragment units (rows g and g + 8 of its tiles)
    const float w2a = m0 + mb + g < p.M ? bf16_to_f32(__ldg(p.w2 + m0 + mb + g)) : 0.f;
    const float w2b = m0 + mb + g + 8 < p.M ? bf16_to_f32(__ldg(p.w2 + m0 + mb + g + 8)) : 0.f;
    if (blockIdx.x == 0 && blockIdx.y == 0 && warp == 0) {
        // loss and b2 gradient: lane l adds sequences l, l + 32, ... in order, then a butterfly
        float ls = 0.f, gs = 0.f;
#pragma unroll 4
        for (int b = lane; b < p.B; b += 32) {
            const float e = __ldg(p.bhat + b) - __ldg(p.label + b);
            ls += e * e;
            gs += delta_of(p, b);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            ls += __shfl_xor_sync(0xffffffffu, ls, o);
            gs += __shfl_xor_sync(0xffffffffu, gs, o);
        }
        if (lane == 0) {
            *p.loss = ls / static_cast<float>(p.B);
            float mm = *p.mb2, vv = *p.vb2;
            *p.b2 = adamw(*p.b2, gs, mm, vv, p);
            *p.mb2 = mm;
            *p.vb2 = vv;
        }
    }
    // column 0: w2 / b1 gradient partials of units mb + g and mb + g + 8 over the warp's rows
    float gw[2] = {0.f, 0.f}, gb[2] = {0.f, 0.f};
    float acc[8][4];   // [tile nt][(g, 2tq), (g, 2tq + 1), (g + 8, 2tq), (g + 8, 2tq + 1)]
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) acc[i][jj] = 0.f;
    for (int b0 = 0; b0 < p.B; b0 += kBC) {
        const int nb = min(kBC, p.B - b0);
        if (b0 > 0) {
            stage_chunk(b0);
            for (int r = t; r < kBC; r += 256) sdelta[r] = r < nb ? delta_of(p, b0 + r) : 0.f;
            cp_async_wait<0>();   // (the W1 block, committed earlier, has landed too)
        } else {
            cp_async_wait<0>();
            if (wvec) {
                // this CTA's block of the masters and moments, for the epilogue
                for (int x = t; x < 3 * kTile * (kTile / 4); x += 256) {
                    const int a = x / (kTile * (kTile / 4)), r = (x / (kTile / 4)) % kTile;
                    const int c4 = (x % (kTile / 4)) * 4;
                    const int m = m0 + r;
                    const float* base = a == 0 ? p.W1m : (a == 1 ? p.mW1 : p.vW1);
                    cp_async16(&sw[a][r][c4], base + static_cast<size_t>(m < p.M ? m : 0) * p.H + j0 + c4,
                               m < p.M ? 16u : 0u);
                }
            }
            cp_async_commit();    // in flight while the tensor cores run
        }
        __syncthreads();
        // dW1 tile += E^T h over the chunk's sequences, 16 at a time, on the tensor cores
        // (mma.sync m16n8k16, fp32 accumulation).  e_bm = delta_b w2_m [u_bm > 0] is formed
        // from the staged u as the fragments are built.  E is fp32: it enters as the sum of three
        // bf16 operands, hi = RN(e), mid = RN(e - hi), lo = RN(e - hi - mid), whose products
        // with the exact bf16 h add up to e h within 2^-24 relative, as fine as e itself;
        // rows past the batch hold zeros.  The h operand comes from the [b][j] tile by
        // transposing 8 x 8 loads: b0 = h[kb + 2tq .. + 1][j], b1 = h[kb + 8 + 2tq .. + 1][j].
        for (int kb = 16 * kh; kb < nb; kb += 32) {
            uint32_t ahi[4], amid[4], alo[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                // a0: (row g, k 2tq..2tq+1), a1: row g + 8, a2: k + 8, a3: both
                const int m = mb + g + ((q & 1) ? 8 : 0);
                const int r = kb + 2 * tq + ((q & 2) ? 8 : 0);
                const float u0 = se[r][m], u1 = se[r + 1][m];
                const float d0 = sdelta[r], d1 = sdelta[r + 1];
                const float w2m = (q & 1) ? w2b : w2a;
                const float e0 = u0 > 0.f ? d0 * w2m : 0.f, e1 = u1 > 0.f ? d1 * w2m : 0.f;
                if (col0) {
                    gw[q & 1] += d0 * fmaxf(u0, 0.f) + d1 * fmaxf(u1, 0.f);
                    gb[q & 1] += e0 + e1;
                }
                const uint32_t hi = pack_bf16x2_rn(e0, e1);
                const float r0 = e0 - __uint_as_float(hi << 16), r1 = e1 - __uint_as_float(hi & 0xffff0000u);
                const uint32_t mid = pack_bf16x2_rn(r0, r1);
                ahi[q] = hi;
                amid[q] = mid;
                alo[q] = pack_bf16x2_rn(r0 - __uint_as_float(mid << 16), r1 - __uint_as_float(mid & 0xffff0000u));
            }
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                // matrices: rows kb .. kb + 7 / kb + 8 .. kb + 15 of column groups 2np, 2np + 1
                const int mat = lane >> 3;
                uint32_t bq[4];
                ldsm_x4_trans(bq, &sh[kb + (lane & 7) + 8 * (mat & 1)][(2 * np + (mat >> 1)) * 8]);
                const uint32_t b_lo[2] = {bq[0], bq[1]}, b_hi[2] = {bq[2], bq[3]};
                // smallest part first, so the larger parts are added to an accumulator that
                // already holds the small corrections
                mma_bf16_16816(acc[2 * np], alo, b_lo);
                mma_bf16_16816(acc[2 * np + 1], alo, b_hi);
                mma_bf16_16816(acc[2 * np], amid, b_lo);
                mma_bf16_16816(acc[2 * np + 1], amid, b_hi);
                mma_bf16_16816(acc[2 * np], ahi, b_lo);
                mma_bf16_16816(acc[2 * np + 1], ahi, b_hi);
            }
        }
        __syncthreads();
    }
    // column 0: this tile's units' w2 / b1 gradients, summed over the sequences in a fixed
    // order, and the AdamW steps of their fp32 masters and moments; the new w2 goes to the
    // workspace until every CTA has read the old one
    if (col0) {
        // the four lanes of a unit (tq = 0..3) hold disjoint rows of the warp's half
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            gw[i] += __shfl_xor_sync(0xffffffffu, gw[i], 1);
            gw[i] += __shfl_xor_sync(0xffffffffu, gw[i], 2);
            gb[i] += __shfl_xor_sync(0xffffffffu, gb[i], 1);
            gb[i] += __shfl_xor_sync(0xffffffffu, gb[i], 2);
        }
        if (tq == 0) {
            sg[kh][0][mb + g] = gw[0];
            sg[kh][0][mb + g + 8] = gw[1];
            sg[kh][1][mb + g] = gb[0];
            sg[kh][1][mb + g + 8] = gb[1];
        }
        __syncthreads();
        if (t < kTile && m0 + t < p.M) {
            const int m = m0 + t;
            const float a = sg[0][0][t] + sg[1][0][t], c = sg[0][1][t] + sg[1][1][t];
            float mm = sp[1][t], vv = sp[2][t];
            const float w2n = adamw(sp[0][t], a, mm, vv, p);
            float mb = sp[4][t], vb = sp[5][t];
            const float b1n = adamw(sp[3][t], c, mb, vb, p);
            p.w2m[m] = w2n;
            p.mw2[m] = mm;
            p.vw2[m] = vv;
            p.b1[m] = b1n;
            p.mb1[m] = mb;
            p.vb1[m] = vb;
            p.e[m] = w2n;                    // workspace: the new w2 master, [M]
        }
    }
    // the ticket, before this CTA's W1 stores, so that the fence waits only for the column-0
    // writes above; every CTA has read the forward's w2 by now.  The atomic is in flight while
    // the epilogue runs, and the last CTA to take it publishes the new bf16 w2.
    __syncthreads();
    uint32_t ticket_old = 0u;
    if (t == 0) {
        __threadfence();
        ticket_old = atomicAdd(p.ticket, 1u);
    }
    // The gradient tile goes through shared memory (the u tile's buffer) so that the AdamW
    // epilogue walks whole rows of W1: each half-warp takes one row's 64 columns as 16-byte
    // vectors, 256 contiguous bytes of every master and moment array per row.  The second half
    // of the sequences is stored first, and the first half's warps add theirs to it.
    if (kh == 1) {
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int r = mb + g + 8 * half, c = nt * 8 + 2 * tq;
                *reinterpret_cast<float2*>(&se[r][c]) = make_float2(acc[nt][2 * half], acc[nt][2 * half + 1]);
            }
    }
    __syncthreads();
    if (kh == 0) {
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int r = mb + g + 8 * half, c = nt * 8 + 2 * tq;
                float2* d = reinterpret_cast<float2*>(&se[r][c]);
                const float2 o = *d;
                *d = make_float2(acc[nt][2 * half] + o.x, acc[nt][2 * half + 1] + o.y);
            }
    }
    cp_async_wait<0>();
    __syncthreads();
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
                const float4 wm = *reinterpret_cast<const float4*>(&sw[0][r][c]);
                float4 mm = *reinterpret_cast<const float4*>(&sw[1][r][c]);
                float4 vv = *reinterpret_cast<const float4*>(&sw[2][r][c]);
                float4 w;
                w.x = adamw(wm.x, gv.x, mm.x, vv.x, p);
                w.y = adamw(wm.y, gv.y, mm.y, vv.y, p);
                w.z = adamw(wm.z, gv.z, mm.z, vv.z, p);
                w.w = adamw(wm.w, gv.w, mm.w, vv.w, p);
                __stcg(reinterpret_cast<float4*>(p.W1m + o), w);
                __stcg(reinterpret_cast<float4*>(p.mW1 + o), mm);
                __stcg(reinterpret_cast<float4*>(p.vW1 + o), vv);
                *reinterpret_cast<uint2*>(p.W1 + o) =
                    make_uint2(f32_to_bf16_rne(w.x) | (static_cast<uint32_t>(f32_to_bf16_rne(w.y)) << 16),
                               f32_to_bf16_rne(w.z) | (static_cast<uint32_t>(f32_to_bf16_rne(w.w)) << 16));
            } else {
                const float gg[4] = {gv.x, gv.y, gv.z, gv.w};
                for (int jj = 0; jj < 4; ++jj) {
                    if (j0 + c + jj >= p.H) break;
                    float mmv = p.mW1[o + jj], vvv = p.vW1[o + jj];
                    const float w = adamw(p.W1m[o + jj], gg[jj], mmv, vvv, p);
                    p.W1m[o + jj] = w;
                    p.mW1[o + jj] = mmv;
                    p.vW1[o + jj] = vvv;
                    p.W1[o + jj] = f32_to_bf16_rne(w);
                }
            }
        }
    }
    if (t == 0) last = (ticket_old + 1u == gridDim.x * gridDim.y) ? 1 : 0;
    __syncthreads();
    if (!last) return;
    __threadfence();
    for (int m = t; m < p.M; m += 256) p.w2[m] = f32_to_bf16_rne(__ldcg(p.e + m));
    if (t == 0) *p.ticket = 0u;
}

}  // namespace

int launch_head_update(const HeadUpdateParams& p, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    constexpr size_t kSmem = kBackSmem;
    {
        // the dynamic shared-memory attribute, once per device (under a lock)
        static std::mutex lock;
        static std::vector<int> done;
        int dev = 0;
        cudaError_t err = cudaGetDevice(&dev);
        if (err != cudaSuccess) return static_cast<int>(err);
        std::lock_guard<std::mutex> guard(lock);
        if (std::find(done.begin(), done.end(), dev) == done.end()) {
            err = cudaFuncSetAttribute(head_back_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmem));
            if (err != cudaSuccess) return static_cast<int>(err);
            done.push_back(dev);
        }
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    // a programmatic dependent of the preceding kernel (it waits for that grid first thing):
    // the launch latency overlaps that kernel's tail
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3((p.H + kTile - 1) / kTile, (p.M + kTile - 1) / kTile, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = st;
    return static_cast<int>(cudaLaunchKernelEx(&cfg, head_back_kernel, p));
}

}  // namespace svd
