// umma_probe.cu -- test-only kernel: one tcgen05 MMA chain on a small tile, to
// check the library's shared-memory descriptors, instruction descriptors and
// TMEM read-back layout against a host matmul.  Not part of the library.
//
// D[M][N] = A[M][K] * B[N][K]^T (negated when neg_b), fp32 accumulation.
// A, B arrive as fp32 values that 16-bit floats represent exactly.  With a_tmem, A is
// written to tensor memory (row m in lane m, elements 2j and 2j+1 packed into column j)
// and the MMA reads it from there.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../gated_delta_rule_135_b200/csrc/umma.cuh"

using namespace kda::umma;

namespace {

constexpr int kMaxM = 128, kMaxN = 256, kMaxK = 128;

__global__ void __launch_bounds__(128) probe_kernel(const float* A, const float* B, float* D,
                                                    int M, int N, int K, int a_mn, int b_mn,
                                                    int bf16, int neg_b, int a_tmem, int* status) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* sA = smem;                                   // up to 128 x 128 x 2 = 32 KB
    unsigned char* sB = smem + kMaxM * kMaxK * 2;               // up to 256 x 128 x 2 = 64 KB
    __shared__ uint64_t bar;
    __shared__ uint32_t tmem_base;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    for (int x = tid; x < M * K; x += blockDim.x) {
        const int m = x / K, k = x % K;
        const uint32_t off = a_mn ? sw128_off(k, m, K) : sw128_off(m, k, M);
        if (bf16) *reinterpret_cast<__nv_bfloat16*>(sA + off) = __float2bfloat16_rn(A[x]);
        else *reinterpret_cast<__half*>(sA + off) = __float2half_rn(A[x]);
    }
    for (int x = tid; x < N * K; x += blockDim.x) {
        const int n = x / K, k = x % K;
        const uint32_t off = b_mn ? sw128_off(k, n, K) : sw128_off(n, k, N);
        if (bf16) *reinterpret_cast<__nv_bfloat16*>(sB + off) = __float2bfloat16_rn(B[x]);
        else *reinterpret_cast<__half*>(sB + off) = __float2half_rn(B[x]);
    }
    fence_proxy_async();
    if (tid == 0) {
        mbar_init(&bar, 1);
        mbar_init_fence();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base, 512);
        tmem_relinquish();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = tmem_base;
    constexpr uint32_t kAcol = 256;   // A's columns in TMEM (D uses 0 .. N-1)
    if (a_tmem) {
        // row 32 * warp + lane of A into lane quarter `warp`, two 16-bit elements per column
        const int m = warp * 32 + lane;
        for (int c0 = 0; c0 < K / 2; c0 += 16) {
            uint32_t r[16];
            for (int j = 0; j < 16; ++j) {
                const float lo = A[m * K + 2 * (c0 + j)], hi = A[m * K + 2 * (c0 + j) + 1];
                uint32_t w;
                if (bf16) {
                    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
                    w = *reinterpret_cast<uint32_t*>(&v);
                } else {
                    __half2 v = __floats2half2_rn(lo, hi);
                    w = *reinterpret_cast<uint32_t*>(&v);
                }
                r[j] = w;
            }
            tmem_st16(taddr(tbase, warp, kAcol + c0), r);
        }
        tmem_wait_st();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (tid == 0) {
        const uint32_t idesc = idesc_f16(M, N, bf16 != 0, a_mn != 0, b_mn != 0, neg_b != 0);
        const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
        for (int ks = 0; ks < K / 16; ++ks) {
            const uint64_t bd = b_mn ? desc_mnmajor(b0, K, ks) : desc_kmajor(b0, N, ks);
            if (a_tmem) {
                mma_f16_ts(tbase, tbase + kAcol + (uint32_t)ks * 8u, bd, idesc, ks > 0 ? 1u : 0u);
            } else {
                const uint64_t ad = a_mn ? desc_mnmajor(a0, K, ks) : desc_kmajor(a0, M, ks);
                mma_f16(tbase, ad, bd, idesc, ks > 0 ? 1u : 0u);
            }
        }
        mma_commit(&bar);
    }
    __syncwarp();
    const bool ok = mbar_wait_bounded(&bar, 0);
    if (!ok && tid == 0) atomicExch(status, 1);
    fence_after_sync();
    if (ok) {
        // lane quarter `warp` holds D rows 32*warp.. (M=128) or 16*warp.. in its lanes 0-15 (M=64)
        for (int c0 = 0; c0 < N; c0 += 16) {
            uint32_t r[16];
            tmem_ld16(taddr(tbase, warp, c0), r);
            tmem_wait_ld();
            int row = -1;
            if (M == 128) row = warp * 32 + lane;
            else if (lane < 16) row = warp * 16 + lane;
            if (row >= 0)
                for (int j = 0; j < 16; ++j) D[row * N + c0 + j] = __uint_as_float(r[j]);
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 512);
}

}  // namespace

extern "C" int umma_probe(const float* A, const float* B, float* D, int M, int N, int K, int a_mn,
                          int b_mn, int bf16, int neg_b, int a_tmem, int* status) {
    if (!(M == 64 || M == 128) || N < 16 || N > kMaxN || N % 16 || K < 16 || K > kMaxK || K % 16)
        return -1;
    if (a_tmem && (M != 128 || a_mn)) return -1;   // a TMEM operand is 128 lanes, one row per lane
    const int smem = kMaxM * kMaxK * 2 + kMaxN * kMaxK * 2 + 1024;
    if (cudaFuncSetAttribute(probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
        return -2;
    probe_kernel<<<1, 128, smem>>>(A, B, D, M, N, K, a_mn, b_mn, bf16, neg_b, a_tmem, status);
    if (cudaGetLastError() != cudaSuccess) return -3;
    return cudaDeviceSynchronize() == cudaSuccess ? 0 : -4;
}
