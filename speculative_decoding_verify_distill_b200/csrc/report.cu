// report.cu -- speedup reporter for one verification step: the measured tokens per target
// verification, the pooled and per-position acceptance rates, and the speculative-decoding
// model E[tau] = (1 - Acc^(k+1)) / (1 - Acc), eta = E[tau] / (rho*k + 1) (Pith review page,
// Referee Report minor comment 1, their Eq. 1; the Axiom ledger's standard acceptance formula).
//
// One CTA: per-position counts from warp ballots, exact integer sums, fp64 results.
#include <cuda_runtime.h>

#include <cmath>

#include "svd_internal.h"

namespace svd {

namespace {

constexpr int kReportThreads = 256;

__device__ __forceinline__ unsigned long long warp_sum_ull(unsigned long long v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__global__ void __launch_bounds__(kReportThreads) speedup_report_kernel(
    const int32_t* accept_len, const int32_t* bk, const int32_t* n_emitted, int B, int k,
    double rho, double* out) {
    __shared__ unsigned long long s_sum[4];   // emitted, accepted, decided, verified
    __shared__ unsigned int s_acc[32], s_tst[32];
    const int t = threadIdx.x, lane = t & 31;
    if (t < 4) s_sum[t] = 0ull;
    if (t < 32) { s_acc[t] = 0u; s_tst[t] = 0u; }
    __syncthreads();
    unsigned long long se = 0, sa = 0, st = 0, sn = 0;
    for (int base = 0; base < B; base += kReportThreads) {
        const int b = base + t;
        const bool valid = b < B;
        const int a = valid ? __ldg(accept_len + b) : 0;
        const int n = valid ? __ldg(bk + b) : 0;
        if (valid) {
            se += static_cast<unsigned long long>(__ldg(n_emitted + b));
            sa += static_cast<unsigned long long>(a);
            sn += static_cast<unsigned long long>(n);
            st += static_cast<unsigned long long>(a + 1 < n ? a + 1 : n);   // decisions taken
        }
        for (int i = 0; i < k; ++i) {
            const unsigned acc_m = __ballot_sync(0xffffffffu, valid && a > i);
            const unsigned tst_m = __ballot_sync(0xffffffffu, valid && a >= i && n > i);
            if (lane == 0) {
                atomicAdd(&s_acc[i], static_cast<unsigned>(__popc(acc_m)));
                atomicAdd(&s_tst[i], static_cast<unsigned>(__popc(tst_m)));
            }
        }
    }
    se = warp_sum_ull(se);
    sa = warp_sum_ull(sa);
    st = warp_sum_ull(st);
    sn = warp_sum_ull(sn);
    if (lane == 0) {
        atomicAdd(&s_sum[0], se);
        atomicAdd(&s_sum[1], sa);
        atomicAdd(&s_sum[2], st);
        atomicAdd(&s_sum[3], sn);
    }
    __syncthreads();
    if (t == 0) {
        const double nb = static_cast<double>(B);
        const double acc = static_cast<double>(s_sum[1]) / static_cast<double>(s_sum[2]);
        const double model = acc == 1.0 ? static_cast<double>(k + 1)
                                        : (1.0 - pow(acc, static_cast<double>(k + 1))) / (1.0 - acc);
        const double denom = rho * static_cast<double>(k) + 1.0;
        out[0] = static_cast<double>(s_sum[0]) / nb;
        out[1] = acc;
        out[2] = model;
        out[3] = model / denom;
        out[4] = out[0] / denom;
        out[5] = static_cast<double>(s_sum[3]) / nb;
        out[6] = static_cast<double>(s_sum[1]) / nb;
        out[7] = nb;
    }
    if (t < k) {
        out[8 + t] = s_tst[t] > 0u ? static_cast<double>(s_acc[t]) / static_cast<double>(s_tst[t])
                                   : __longlong_as_double(0x7ff8000000000000ll);
    }
}

}  // namespace

int launch_speedup_report(const int32_t* accept_len, const int32_t* bk, const int32_t* n_emitted,
                          int B, int k, double rho, double* out, void* stream) {
    speedup_report_kernel<<<1, kReportThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        accept_len, bk, n_emitted, B, k, rho, out);
    return static_cast<int>(cudaGetLastError());
}

}  // namespace svd
