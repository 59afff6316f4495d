// length_head.cu -- the adaptive length head: bhat = sigmoid(w2 . relu(W1 h + b1) + b2) and the
// verification length b_k = clamp(round(gamma * bhat * k), 1, k).
//
// AdaFlash (Pith review page "What carries the argument": a small network on drafter hidden
// states predicts the block's acceptance rate; Axiom & Free-Parameter Ledger: a pooled
// representation is mapped to a single scalar and converted linearly to the verification length,
// gamma = 1.0; Referee Report minor comment 2: b_k = clamp(floor(bhat * k), 1, k)).
//
// The projection h [B,H] x W1^T [H,M] is a small dense contraction (2*B*H*M flops, 0.27 GFLOP
// at B=128, H=4096, M=256) on the tensor cores: bf16 operands, fp32 accumulation.  Two forms:
//   * units (H a multiple of 16, 16-byte aligned h and W1): the work units of svd_head_unit.cuh,
//     one CTA each -- the same units the fused verify-and-distill call runs inside its row pass,
//     so both give the same bhat and b_k;
//   * split (any shape): grid (16-sequence tiles) x (64-unit tiles) x (K splits); each CTA stages
//     its operand slices in shared memory with element-wise 16-byte loads and its 8 warps each
//     accumulate one 16x8 output tile.  Split partials land in the workspace; the last CTA of an
//     output tile (atomic ticket, no waiting) adds them in split order, applies bias, ReLU and
//     w2, and the last tile adds the per-tile logits in tile order and applies the sigmoid and
//     the b_k map.
// Every sum has a fixed order in both.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <mutex>
#include <vector>

#include "svd_device.cuh"
#include "svd_head_unit.cuh"

namespace svd {

namespace {

constexpr int kWarps = 8;
constexpr int kKC = 256;          // K chunk staged in shared memory
constexpr int kPad = 8;           // row padding (16 bytes): conflict-free fragment reads
constexpr int kLd = kKC + kPad;

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// rows x kKC tile of a [nrows, ncols] bf16 matrix into padded shared memory; zero outside
// [0, nrows) x [c0, c1).
__device__ __forceinline__ void stage_tile(uint16_t* dst, const uint16_t* src, int rows, int r0,
                                           int nrows, int ncols, int c0, int c1, bool vec_ok) {
    const int vecs = rows * (kKC / 8);
    for (int v = threadIdx.x; v < vecs; v += blockDim.x) {
        const int r = v / (kKC / 8), cv = (v % (kKC / 8)) * 8;
        const int gr = r0 + r, gc = c0 + cv;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (gr < nrows) {
            const uint16_t* s = src + static_cast<size_t>(gr) * ncols + gc;
            if (vec_ok && gc + 8 <= c1) {
                val = __ldg(reinterpret_cast<const uint4*>(s));
            } else {
                uint16_t e[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) e[q] = (gc + q < c1) ? __ldg(s + q) : uint16_t(0);
                val = make_uint4(e[0] | (uint32_t(e[1]) << 16), e[2] | (uint32_t(e[3]) << 16),
                                 e[4] | (uint32_t(e[5]) << 16), e[6] | (uint32_t(e[7]) << 16));
            }
        }
        *reinterpret_cast<uint4*>(dst + r * kLd + cv) = val;
    }
}

}  // namespace

__global__ void __launch_bounds__(kWarps * 32) length_head_kernel(const HeadParams p) {
    __shared__ __align__(16) uint16_t hs[kHeadTileB * kLd];
    __shared__ __align__(16) uint16_t ws[kHeadTileM * kLd];
    __shared__ float pre[kHeadTileB][kHeadTileM + 1];
    __shared__ int flag;

    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int bt = blockIdx.x, mt = blockIdx.y, kz = blockIdx.z;
    const int b0 = bt * kHeadTileB, m0 = mt * kHeadTileM;
    const int g = lane >> 2, tq = lane & 3;
    const int k_lo = min(p.H, kz * p.ks), k_hi = min(p.H, k_lo + p.ks);
    const bool vec_ok = (p.H % 8 == 0) && ((reinterpret_cast<uintptr_t>(p.h) & 15) == 0) &&
                        ((reinterpret_cast<uintptr_t>(p.W1) & 15) == 0);

    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int c0 = k_lo; c0 < k_hi; c0 += kKC) {
        const int c1 = min(k_hi, c0 + kKC);
        stage_tile(hs, p.h, kHeadTileB, b0, p.B, p.H, c0, c1, vec_ok);
        stage_tile(ws, p.W1, kHeadTileM, m0, p.M, p.H, c0, c1, vec_ok);
        __syncthreads();
        const uint16_t* wrow = ws + (warp * 8 + g) * kLd;
#pragma unroll 4
        for (int kk = 0; kk < kKC; kk += 16) {
            if (c0 + kk >= c1) break;
            uint32_t a[4], bf[2];
            a[0] = *reinterpret_cast<const uint32_t*>(hs + g * kLd + kk + 2 * tq);
            a[1] = *reinterpret_cast<const uint32_t*>(hs + (g + 8) * kLd + kk + 2 * tq);
            a[2] = *reinterpret_cast<const uint32_t*>(hs + g * kLd + kk + 2 * tq + 8);
            a[3] = *reinterpret_cast<const uint32_t*>(hs + (g + 8) * kLd + kk + 2 * tq + 8);
            bf[0] = *reinterpret_cast<const uint32_t*>(wrow + kk + 2 * tq);
            bf[1] = *reinterpret_cast<const uint32_t*>(wrow + kk + 2 * tq + 8);
            mma_bf16_16816(acc, a, bf);
        }
        __syncthreads();
    }
    // accumulator layout: acc[0..1] = (row g, cols 2tq + {0,1}); acc[2..3] = row g + 8
    {
        float* part = p.part + static_cast<size_t>(kz) * p.B * p.M;
        const int m = m0 + warp * 8 + 2 * tq;
        const int rows[2] = {b0 + g, b0 + g + 8};
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            const int b = rows[h2];
            if (b < p.B) {
                if (m < p.M) part[static_cast<size_t>(b) * p.M + m] = acc[2 * h2];
                if (m + 1 < p.M) part[static_cast<size_t>(b) * p.M + m + 1] = acc[2 * h2 + 1];
            }
        }
    }
    // last split of this output tile reduces the partials in split order
    __threadfence();
    __syncthreads();
    if (t == 0) {
        const uint32_t old = atomicAdd(&p.tile_ticket[bt * gridDim.y + mt], 1u);
        flag = (old + 1u == gridDim.z) ? 1 : 0;
    }
    __syncthreads();
    if (!flag) return;
    __threadfence();
    for (int o = t; o < kHeadTileB * kHeadTileM; o += blockDim.x) {
        const int r = o / kHeadTileM, col = o % kHeadTileM;
        const int b = b0 + r, m = m0 + col;
        float a = 0.f;
        if (b < p.B && m < p.M) {
            for (int z = 0; z < static_cast<int>(gridDim.z); ++z)
                a += __ldcg(p.part + (static_cast<size_t>(z) * p.B + b) * p.M + m);
            if (p.b1) a += __ldg(p.b1 + m);
            if (p.u_out) p.u_out[static_cast<size_t>(b) * p.M + m] = a;
            const float w2 = __uint_as_float(static_cast<uint32_t>(__ldg(p.w2 + m)) << 16);
            a = w2 * fmaxf(a, 0.f);
        }
        pre[r][col] = a;
    }
    __syncthreads();
    // per-sequence sum over this tile's 64 units (warp w: rows 2w, 2w+1; fixed shuffle order)
    for (int r = warp * 2; r < warp * 2 + 2; ++r) {
        float z = pre[r][lane] + pre[r][lane + 32];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        if (lane == 0 && b0 + r < p.B) p.zpart[static_cast<size_t>(mt) * p.B + b0 + r] = z;
    }
    if (t == 0) p.tile_ticket[bt * gridDim.y + mt] = 0u;
    // last output tile combines the per-tile logits of every sequence
    __threadfence();
    __syncthreads();
    if (t == 0) {
        const uint32_t total = gridDim.x * gridDim.y;
        const uint32_t old = atomicAdd(&p.hdr->head_ticket, 1u);
        flag = (old + 1u == total) ? 2 : 0;
    }
    __syncthreads();
    if (flag != 2) return;
    __threadfence();
    const int mtiles = gridDim.y;
    for (int b = t; b < p.B; b += blockDim.x) {
        float z = p.b2_dev ? *p.b2_dev : p.b2;
        for (int q = 0; q < mtiles; ++q) z += __ldcg(p.zpart + static_cast<size_t>(q) * p.B + b);
        const float bhat = 1.f / (1.f + expf(-z));
        const float target = p.gamma * bhat * static_cast<float>(p.k);
        const float r = p.rnd == 0 ? ceilf(target) : floorf(target);
        int bk = static_cast<int>(fminf(fmaxf(r, 1.f), static_cast<float>(p.k)));
        if (!(r == r)) bk = 1;  // non-finite hidden states
        if (p.bhat) p.bhat[b] = bhat;
        if (p.bk) p.bk[b] = bk;
    }
    if (t == 0) p.hdr->head_ticket = 0u;
}

namespace {
constexpr uint64_t kHeadWaitNs = 1000000000ull;   // 1 s bound on a unit's staging wait
}  // namespace

// The head as independent work units (svd_head_unit.cuh), one CTA per unit: the same units the
// fused verify-and-distill pass runs inside its row pass, so both give the same bhat and b_k.
// Dynamic shared memory: the unit's staged K chunk, then its mbarrier.
__global__ void __launch_bounds__(kWarps * 32) length_head_units_kernel(const HeadParams p,
                                                                       uint32_t stage_bytes) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem_raw + stage_bytes);
    __shared__ int flag;
    // launched as a programmatic dependent of the preceding kernel: nothing is read before it
    // has finished; the kernel after this one may be scheduled at once (it waits likewise)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    uint32_t phase = 0;
    head_unit<kWarps>(p, static_cast<int>(blockIdx.x), &flag, true, reinterpret_cast<uint16_t*>(smem_raw),
                      stage_bytes, bar, phase, kHeadWaitNs);
}

// Shared memory for a unit whose split of ks columns is staged in one chunk.
size_t head_unit_stage_bytes(int ks) {
    return static_cast<size_t>(kHeadTileB + kHeadTileM) * (ks + 8) * 2;
}

int launch_length_head(const HeadParams& p, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // units need H a multiple of 16 and 16-byte aligned rows (bulk copies); otherwise the
    // split form with element-wise staging
    const bool units_form = (p.H % 16 == 0) && ((reinterpret_cast<uintptr_t>(p.h) & 15) == 0) &&
                            ((reinterpret_cast<uintptr_t>(p.W1) & 15) == 0);
    if (!units_form) {
        dim3 grid((p.B + kHeadTileB - 1) / kHeadTileB, (p.M + kHeadTileM - 1) / kHeadTileM, p.nsplit);
        length_head_kernel<<<grid, kWarps * 32, 0, st>>>(p);
        return static_cast<int>(cudaGetLastError());
    }
    // one chunk per unit when it fits in 100 KB, else chunks of what does
    constexpr size_t kMaxStage = 100 * 1024;
    size_t stage = head_unit_stage_bytes(p.ks);
    if (stage > kMaxStage) stage = kMaxStage;
    stage = (stage + 127) & ~size_t(127);
    const size_t smem = stage + 16;
    {
        // the dynamic shared-memory limit, raised to the largest stage once per device
        static std::mutex lock;
        static std::vector<int> done;
        int dev = 0;
        cudaError_t err = cudaGetDevice(&dev);
        if (err != cudaSuccess) return static_cast<int>(err);
        std::lock_guard<std::mutex> guard(lock);
        if (std::find(done.begin(), done.end(), dev) == done.end()) {
            err = cudaFuncSetAttribute(length_head_units_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kMaxStage + 16));
            if (err != cudaSuccess) return static_cast<int>(err);
            done.push_back(dev);
        }
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(head_units(p)), 1, 1);
    cfg.blockDim = dim3(kWarps * 32, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    return static_cast<int>(cudaLaunchKernelEx(&cfg, length_head_units_kernel, p, static_cast<uint32_t>(stage)));
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
