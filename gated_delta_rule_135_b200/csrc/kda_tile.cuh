// kda_tile.cuh -- register-tiled fp32 block products on shared-memory operands.
//
// The staged kernels (forward fallback and backward) are small dense products of
// 64 x 128 and 128 x 128 tiles held in shared memory.  One accumulator per thread
// makes every FMA wait on a shared-memory load; a TM x TN tile of accumulators per
// thread gives TM * TN independent FMAs per TM + TN loads instead.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace kda {

// acc[i][j] += sum_{k0 <= k < k1} A(r0 + i RS, k) * B(k, c0 + j CS)
// with A(r, k) = a[r AR + k AK] and B(k, c) = b[k BK + c BC] (all strides in floats).
template <int TM, int TN, int RS, int CS, int AR, int AK, int BK, int BC>
__device__ __forceinline__ void tile_fma(float (&acc)[TM][TN], const float* __restrict__ a,
                                         const float* __restrict__ b, int r0, int c0, int k0, int k1) {
#pragma unroll 4
    for (int k = k0; k < k1; ++k) {
        float av[TM], bv[TN];
#pragma unroll
        for (int i = 0; i < TM; ++i) av[i] = a[(r0 + i * RS) * AR + k * AK];
#pragma unroll
        for (int j = 0; j < TN; ++j) bv[j] = b[k * BK + (c0 + j * CS) * BC];
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
}

template <int TM, int TN>
__device__ __forceinline__ void tile_zero(float (&acc)[TM][TN]) {
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;
}

// ---------------------------------------------------------------------------
// Staging of token-major tiles into shared memory.  Every thread first issues all of
// its 16-byte global loads (ROWS x COLS / NT / elements-per-vector of them), then
// converts and stores: the loads of a thread are in flight together instead of one
// at a time.  Row r of the tile starts at src + r * ld (16-byte aligned); rows >= len
// are stored as 0, rows < len as f(r, c, value).
template <typename T>
struct Vec16;
template <>
struct Vec16<float> {
    using type = float4;
    static constexpr int n = 4;
    __device__ static void unpack(const float4& v, float* o) { o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w; }
};
template <>
struct Vec16<__nv_bfloat16> {
    using type = uint4;
    static constexpr int n = 8;
    __device__ static void unpack(const uint4& v, float* o) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            o[2 * i] = __uint_as_float(w[i] << 16);
            o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};

template <int ROWS, int COLS, int NT, typename T, typename F>
__device__ __forceinline__ void stage(float* __restrict__ dst, int pitch, const T* __restrict__ src, int64_t ld,
                                      int len, F f) {
    using V = Vec16<T>;
    constexpr int VPR = COLS / V::n, TOTAL = ROWS * VPR;
    static_assert(TOTAL % NT == 0, "tile must divide among the threads");
    constexpr int PER = TOTAL / NT;
    typename V::type v[PER];
#pragma unroll
    for (int m = 0; m < PER; ++m) {
        const int x = threadIdx.x + NT * m, r = x / VPR, cv = x % VPR;
        if (r < len) v[m] = *reinterpret_cast<const typename V::type*>(src + r * ld + cv * V::n);
        else v[m] = typename V::type{};
    }
#pragma unroll
    for (int m = 0; m < PER; ++m) {
        const int x = threadIdx.x + NT * m, r = x / VPR, cv = x % VPR;
        float o[V::n];
        V::unpack(v[m], o);
#pragma unroll
        for (int e = 0; e < V::n; ++e)
            dst[r * pitch + cv * V::n + e] = r < len ? f(r, cv * V::n + e, o[e]) : 0.f;
    }
}

// Two sources at the same positions: fp32 (16-byte loads) and bf16 (8-byte loads); stores
// f(r, c, fp32 value, bf16 value).
template <int ROWS, int COLS, int NT, typename F>
__device__ __forceinline__ void stage2(float* __restrict__ dst, int pitch, const float* __restrict__ srcf,
                                       const __nv_bfloat16* __restrict__ srcb, int64_t ld, int len, F f) {
    constexpr int VPR = COLS / 4, TOTAL = ROWS * VPR;
    static_assert(TOTAL % NT == 0, "tile must divide among the threads");
    constexpr int PER = TOTAL / NT;
    float4 vf[PER];
    uint2 vb[PER];
#pragma unroll
    for (int m = 0; m < PER; ++m) {
        const int x = threadIdx.x + NT * m, r = x / VPR, cv = x % VPR;
        if (r < len) {
            vf[m] = *reinterpret_cast<const float4*>(srcf + r * ld + cv * 4);
            vb[m] = *reinterpret_cast<const uint2*>(srcb + r * ld + cv * 4);
        } else {
            vf[m] = float4{};
            vb[m] = uint2{};
        }
    }
#pragma unroll
    for (int m = 0; m < PER; ++m) {
        const int x = threadIdx.x + NT * m, r = x / VPR, cv = x % VPR;
        const float of[4] = {vf[m].x, vf[m].y, vf[m].z, vf[m].w};
        const float ob[4] = {__uint_as_float(vb[m].x << 16), __uint_as_float(vb[m].x & 0xffff0000u),
                             __uint_as_float(vb[m].y << 16), __uint_as_float(vb[m].y & 0xffff0000u)};
#pragma unroll
        for (int e = 0; e < 4; ++e)
            dst[r * pitch + cv * 4 + e] = r < len ? f(r, cv * 4 + e, of[e], ob[e]) : 0.f;
    }
}

// Pulls `rows` rows of `row_bytes` bytes, row r at base + r * ld_bytes, into L2: one
// prefetch per 128-byte line, spread over the block.  The serial chunk scans call it for the
// next chunk so that its staging loads hit L2.
__device__ __forceinline__ void prefetch_rows_l2(const void* base, int64_t ld_bytes, int rows, int row_bytes,
                                                 int nthreads) {
    const int lines = (row_bytes + 127) / 128;
    for (int x = threadIdx.x; x < rows * lines; x += nthreads) {
        const char* ptr = static_cast<const char*>(base) + (int64_t)(x / lines) * ld_bytes + (x % lines) * 128;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
    }
}

// ---- split-bf16 operands of the tensor-core stages ----
// x = hi + lo with hi = bf16(x) and lo = bf16(x - hi), both rounded to nearest even: a product
// taken as hi.hi + hi.lo + lo.hi (fp32 accumulation) keeps about 16 mantissa bits.
__device__ __forceinline__ void split_bf16(float x, uint16_t& hi, uint16_t& lo) {
    const __nv_bfloat16 hb = __float2bfloat16_rn(x);
    hi = __bfloat16_as_ushort(hb);
    lo = __bfloat16_as_ushort(__float2bfloat16_rn(x - __bfloat162float(hb)));
}
// Eight values -> the high and the low parts as two 16-byte chunks (element 0 in the low half).
__device__ __forceinline__ void split_bf16x8(const float (&x)[8], uint4& hi, uint4& lo) {
    uint16_t a[8], b[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) split_bf16(x[i], a[i], b[i]);
    hi = make_uint4(a[0] | ((uint32_t)a[1] << 16), a[2] | ((uint32_t)a[3] << 16), a[4] | ((uint32_t)a[5] << 16),
                    a[6] | ((uint32_t)a[7] << 16));
    lo = make_uint4(b[0] | ((uint32_t)b[1] << 16), b[2] | ((uint32_t)b[3] << 16), b[4] | ((uint32_t)b[5] << 16),
                    b[6] | ((uint32_t)b[7] << 16));
}
// Eight consecutive fp32 values (16-byte aligned source).
__device__ __forceinline__ void load8_f32(const float* src, float (&x)[8]) {
    const float4 a = *reinterpret_cast<const float4*>(src), b = *reinterpret_cast<const float4*>(src + 4);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
// Eight consecutive bf16 values widened to fp32 (16-byte aligned source).
__device__ __forceinline__ void load8_bf16(const __nv_bfloat16* src, float (&x)[8]) {
    const uint4 v = *reinterpret_cast<const uint4*>(src);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

struct Identity {
    __device__ float operator()(int, int, float v) const { return v; }
};

}  // namespace kda
