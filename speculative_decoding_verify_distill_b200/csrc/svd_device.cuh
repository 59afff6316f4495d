// svd_device.cuh -- device-side building blocks for sm_100a: mbarriers and bulk (TMA) copies,
// cluster barriers and distributed shared memory, bf16 unpacking, exp2, Philox4x32-10.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "svd_internal.h"

namespace svd {

// ------------------------------------------------------------------------------------------
// shared-memory addresses, mbarriers, bulk copies
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

// Makes barrier initialisation visible to the async (bulk-copy) proxy and the cluster.
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// Waiting threads are suspended by the hardware until the phase completes or the hint (in ns)
// runs out, so a wait costs no issue slots that other warps on the SM could use.
constexpr uint32_t kSuspendHintNs = 1000000;

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Waits for phase `parity` of `bar` to complete, for at most `limit_ns` nanoseconds of
// wall-clock time.  Returns false if the limit ran out (the caller records SVD_ERR_TIMEOUT and
// carries on, so no thread ever spins without bound).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (global_timer_ns() - t0 > limit_ns) return false;
    }
}

// Same wait with cluster-scope acquire: for barriers completed by other CTAs' st.async.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    return done != 0;
}
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint64_t* bar, uint32_t parity,
                                                          uint64_t limit_ns) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if (global_timer_ns() - t0 > limit_ns) return false;
    }
}

// One-dimensional bulk copy global -> this CTA's shared memory, completing on `bar`.
// Both addresses 16-byte aligned, bytes a multiple of 16.  No multicast.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_addr(smem_dst)), "l"(gsrc), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// ------------------------------------------------------------------------------------------
// clusters and distributed shared memory
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t num_clusters_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}

// Full cluster barrier (every thread of every CTA of the cluster), release/acquire.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of the same shared variable in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t dsmem_map(const void* local, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(local)), "r"(rank));
    return r;
}
__device__ __forceinline__ uint32_t dsmem_ld_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ void dsmem_st_f32(uint32_t a, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}
__device__ __forceinline__ void dsmem_st_u32(uint32_t a, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
// Asynchronous 16-byte store into another CTA's shared memory (cluster addresses from
// dsmem_map), counted as transaction bytes on that CTA's mbarrier `bar`.
__device__ __forceinline__ void st_async_v4(uint32_t a, const uint4& v, uint32_t bar) {
    asm volatile(
        "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1,%2,%3,%4}, [%5];"
        ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "r"(bar)
        : "memory");
}

// Warp-wide max / min in one instruction (f32 form: sm_100a).
__device__ __forceinline__ float redux_max_f32(float v) {
    float r;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
    return r;
}
__device__ __forceinline__ uint32_t redux_min_u32(uint32_t v) {
    uint32_t r;
    asm volatile("redux.sync.min.u32 %0, %1, 0xffffffff;" : "=r"(r) : "r"(v));
    return r;
}

// Three-input maximum (sm_100a form of max.f32; same NaN rule as fmaxf).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Packed pairs of fp32 (sm_100a f32x2 forms; each half rounds exactly like the scalar op).
__device__ __forceinline__ unsigned long long f2_bits(float2 a) {
    return *reinterpret_cast<unsigned long long*>(&a);
}
__device__ __forceinline__ float2 f2_from(unsigned long long b) {
    return *reinterpret_cast<float2*>(&b);
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    unsigned long long r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)), "l"(f2_bits(c)));
    return f2_from(r);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    unsigned long long r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)));
    return f2_from(r);
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    unsigned long long r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)));
    return f2_from(r);
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    unsigned long long r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)));
    return f2_from(r);
}

// ------------------------------------------------------------------------------------------
// arithmetic helpers
// ------------------------------------------------------------------------------------------
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// 2^x with the MUFU.EX2 unit (PTX ex2.approx; ex2(-inf) = +0, ex2(0) = 1).
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Two bf16 packed in one 32-bit word -> two fp32 (exact).
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Maximum of the eight bf16 values of a 16-byte vector (exact, packed compares).
__device__ __forceinline__ float max8_bf16(const uint4& v) {
    __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&v.x);
    __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&v.y);
    __nv_bfloat162 c = *reinterpret_cast<const __nv_bfloat162*>(&v.z);
    __nv_bfloat162 d = *reinterpret_cast<const __nv_bfloat162*>(&v.w);
    __nv_bfloat162 m = __hmax2(__hmax2(a, b), __hmax2(c, d));
    return fmaxf(__low2float(m), __high2float(m));
}

__device__ __forceinline__ void unpack8(const uint4& v, float (&x)[8]) {
    x[0] = bf_lo(v.x); x[1] = bf_hi(v.x);
    x[2] = bf_lo(v.y); x[3] = bf_hi(v.y);
    x[4] = bf_lo(v.z); x[5] = bf_hi(v.z);
    x[6] = bf_lo(v.w); x[7] = bf_hi(v.w);
}

// Round-to-nearest-even pack of two fp32 into one bf16x2 word (lo in the low half).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&r);
}

// Load with acquire semantics at GPU scope (pairs with a release by another CTA: a
// __threadfence before the writer's atomic).
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Record the first device-side error in the workspace status word.
__device__ __forceinline__ void set_device_error(uint32_t* status, uint32_t code) {
    atomicCAS(status, 0u, code);
}

// ------------------------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw: "Parallel random numbers: as easy as 1, 2, 3",
// SC'11): ten rounds of the 4x32 S-box built from two 32x32 -> 64-bit products; the key is
// bumped by the two Weyl increments before every round after the first.
// ------------------------------------------------------------------------------------------
struct PhiloxOut {
    uint32_t w[4];
};

__device__ __forceinline__ PhiloxOut philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2,
                                                   uint32_t c3, uint32_t k0, uint32_t k1) {
    constexpr uint32_t kMulA = 0xD2511F53u, kMulB = 0xCD9E8D57u;
    constexpr uint32_t kWeylA = 0x9E3779B9u, kWeylB = 0xBB67AE85u;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k0 += kWeylA;
            k1 += kWeylB;
        }
        const uint32_t lo_a = kMulA * c0, hi_a = __umulhi(kMulA, c0);
        const uint32_t lo_b = kMulB * c2, hi_b = __umulhi(kMulB, c2);
        const uint32_t n0 = hi_b ^ c1 ^ k0;
        const uint32_t n2 = hi_a ^ c3 ^ k1;
        c0 = n0;
        c1 = lo_b;
        c2 = n2;
        c3 = lo_a;
    }
    PhiloxOut o;
    o.w[0] = c0; o.w[1] = c1; o.w[2] = c2; o.w[3] = c3;
    return o;
}

// Words for (position, sequence, step) under key = seed: counter = (pos, seq, step_lo, step_hi).
__device__ __forceinline__ PhiloxOut philox_words(uint64_t seed, uint64_t step, uint32_t seq,
                                                  uint32_t pos) {
    return philox4x32_10(pos, seq, static_cast<uint32_t>(step), static_cast<uint32_t>(step >> 32),
                         static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
}

// Uniform in [0,1) from the top 24 bits (exact in fp32).
__device__ __forceinline__ float uniform24(uint32_t w) {
    return static_cast<float>(w >> 8) * (1.0f / 16777216.0f);
}

// ------------------------------------------------------------------------------------------
// row arithmetic shared by the fused row pass and the vocab-sharded passes
// ------------------------------------------------------------------------------------------
// Position (0..7) of the first element of a bf16 vector equal to R (7 if none: never used then).
__device__ __forceinline__ int first_pos(const uint4& v, float R) {
    float x[8];
    unpack8(v, x);
    int l = 7;
#pragma unroll
    for (int q = 6; q >= 0; --q) l = (x[q] == R) ? q : l;
    return l;
}
// The four bf16 pairs of a 16-byte vector as packed fp32 pairs (exact).
__device__ __forceinline__ void unpack8x2(const uint4& v, float2 (&x)[4]) {
    x[0] = make_float2(bf_lo(v.x), bf_hi(v.x));
    x[1] = make_float2(bf_lo(v.y), bf_hi(v.y));
    x[2] = make_float2(bf_lo(v.z), bf_hi(v.z));
    x[3] = make_float2(bf_lo(v.w), bf_hi(v.w));
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
// Factor that moves a sum taken relative to reference round(m k2) onto round(M k2) (exactly 1
// when m == M).  Maxima at or below -1e38 mark empty sums (all -inf, or the staging sentinel).
__device__ __forceinline__ float rescale(float m, float M, float k2) {
    return m > -1e38f ? fast_exp2(__fsub_rn(__fmul_rn(m, k2), __fmul_rn(M, k2))) : 0.f;
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


__device__ __forceinline__ void warp_inclusive_scan_u64(unsigned long long& x) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
}

}  // namespace svd
