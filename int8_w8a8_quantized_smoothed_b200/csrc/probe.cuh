// Measurement and self-test aids (not part of the W8A8 path).
//
// Tensor-core throughput probe: measures the dense INT8 rate of tcgen05.mma kind::i8 on this
// device, the denominator of the GEMM roofline. One CTA per SM; one thread issues `iters`
// back-to-back 128 x N x 32 MMAs on zero-filled shared-memory operands into a TMEM
// accumulator, then waits for them through tcgen05.commit. Not part of the W8A8 path.
#pragma once

#include "ptx.cuh"

namespace w8a8 {

template <int N>
__global__ void __launch_bounds__(128, 1) mma_i8_probe_kernel(long long iters,
                                                              unsigned long long limit_ns)
{
    constexpr int kABytes = 128 * 128, kBBytes = N * 128;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sA = smem_u32(smem), sB = sA + kABytes;
    const uint32_t bar = sB + kBBytes;
    uint32_t *tslot_ptr = reinterpret_cast<uint32_t *>(smem + kABytes + kBBytes + 16);
    for (int i = threadIdx.x; i < (kABytes + kBBytes) / 4; i += blockDim.x)
        reinterpret_cast<uint32_t *>(smem)[i] = 0u;
    fence_proxy_async_smem();
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    constexpr uint32_t kCols = N < 32 ? 32 : N; // allocation: a power of two >= 32
    if (threadIdx.x < 32) {
        tmem_alloc(smem_u32(tslot_ptr), kCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(tslot_ptr);
    if (threadIdx.x == 0) {
        constexpr uint32_t idesc = idesc_i8(128, N);
        for (long long i = 0; i < iters; ++i) {
            const uint32_t k = static_cast<uint32_t>(i & 3) * 32u;
            umma_i8(tmem, sw128_kmajor_desc(sA + k), sw128_kmajor_desc(sB + k), idesc,
                    i > 0 ? 1u : 0u);
        }
        umma_commit(bar);
        mbar_wait(bar, 0, limit_ns);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        tc_fence_after();
        tmem_dealloc(tmem, kCols);
    }
}

// Binary64 FMA throughput probe (the denominator of the GPTQ kernels' roofline): every thread
// runs 8 independent chains of `iters` fused multiply-adds; the sums are written so that the
// work is kept.
__global__ void __launch_bounds__(256) fma_f64_probe_kernel(long long iters, double *out)
{
    double a[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
        a[i] = 1.0 + 1e-9 * (threadIdx.x + i);
    const double m = 0.999999999, c = 1e-12;
    for (long long it = 0; it < iters; ++it)
#pragma unroll
        for (int i = 0; i < 8; ++i)
            a[i] = fma(a[i], m, c);
    double s = 0.0;
#pragma unroll
    for (int i = 0; i < 8; ++i)
        s += a[i];
    out[static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x] = s;
}

// Failure-path self-test: one CTA whose waits can never be satisfied -- thread 0 on an
// mbarrier nobody arrives at, thread 32 on a flag word nobody sets -- each bounded by
// limit_ns, so both give up, raise the device status word and return. Shows that a wait that
// runs out ends the kernel cleanly and leaves the context usable.
__device__ unsigned int g_never_set_flag;

__global__ void __launch_bounds__(64, 1) wait_timeout_selftest_kernel(unsigned long long limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0)
        mbar_wait(smem_u32(&bar), 0, limit_ns); // flags the timeout itself
    if (threadIdx.x == 32) {
        const volatile unsigned int *f = &g_never_set_flag;
        const uint64_t t0 = globaltimer_ns();
        while (*f == 0u) {
            if (globaltimer_ns() - t0 > limit_ns) {
                flag_timeout();
                break;
            }
        }
    }
}

} // namespace w8a8
