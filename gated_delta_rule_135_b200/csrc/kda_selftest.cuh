// kda_selftest.cuh -- the bounded-wait recovery path, exercised on purpose.
//
// Every kernel of the library waits on mbarriers with a wall-clock limit.  When a wait runs out
// it records KDA_DEVERR_TIMEOUT, lets its own in-flight tensor-core work finish (again with a
// limit), frees its TMEM and returns, so the device stays usable.  This kernel walks that path
// without any fault: it allocates TMEM, puts one MMA in flight, waits on a barrier that no
// thread ever arrives at, and then winds down exactly as the product kernels do.
#pragma once

#include "kda_common.cuh"
#include "umma.cuh"

namespace kda {
namespace selftest {

using namespace umma;

__global__ void __launch_bounds__(128, 1) wait_timeout_kernel(uint64_t limit_ns, unsigned int* observed) {
    // A (128 rows) and B (64 rows) in the 128-byte-swizzled K-major layout: 128-byte rows, of
    // which the single K = 16 slice uses the first 32 bytes
    __shared__ __align__(1024) unsigned char tiles[128 * 128 + 64 * 128];
    __shared__ uint64_t bars[2];   // 0: the MMA's commit; 1: never arrived at
    __shared__ uint32_t tmem_base;
    const int tid = threadIdx.x;
    for (int i = tid; i < (int)(sizeof(tiles) / 16); i += 128)
        reinterpret_cast<uint4*>(tiles)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async();
    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_init_fence();
    }
    if (tid < 32) {
        tmem_alloc(&tmem_base, 64);
        tmem_relinquish();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tb = tmem_base;
    if (tid == 0) {
        // one MMA in flight (zeros), committed to bars[0]
        const uint32_t a0 = smem_u32(tiles), b0 = smem_u32(tiles + 128 * 128);
        mma_f16(tb, desc_kmajor(a0, 128, 0), desc_kmajor(b0, 64, 0), idesc_f16(128, 64, true, false, false), 0u);
        mma_commit(&bars[0]);
        // the wait that runs out: nothing arrives at bars[1]
        const bool ok = mbar_wait_bounded(&bars[1], 0u, limit_ns);
        if (!ok) record_error(KDA_DEVERR_TIMEOUT);
        // wind-down: the MMA of this thread must be complete before TMEM is released
        const bool drained = mbar_wait_bounded(&bars[0], 0u);
        if (observed) {
            observed[0] = ok ? 0u : 1u;
            observed[1] = drained ? 1u : 0u;
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (tid < 32) tmem_dealloc(tb, 64);
}

}  // namespace selftest

cudaError_t launch_wait_timeout_selftest(uint64_t limit_ns, unsigned int* observed, cudaStream_t stream) {
    selftest::wait_timeout_kernel<<<1, 128, 0, stream>>>(limit_ns, observed);
    return cudaGetLastError();
}

}  // namespace kda
