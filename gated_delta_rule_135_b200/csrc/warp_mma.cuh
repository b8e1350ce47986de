// warp_mma.cuh -- 16x16x16 fp32 block products for one warp on the warp-level
// tensor-core path (mma.sync m16n8k8, tf32 operands, fp32 accumulation), with
// each operand split as hi + lo (both tf32) and the three significant cross
// products summed ("3xTF32"), which keeps the result at fp32-level accuracy.
//
// Fragments of mma.m16n8k8 .tf32 (g = lane / 4, t = lane % 4):
//   A 16x8 row-major: a0 (g, t), a1 (g+8, t), a2 (g, t+4), a3 (g+8, t+4)
//   B 8x8 col-major:  b0 (t, g), b1 (t+4, g)
//   D 16x8:           d0 (g, 2t), d1 (g, 2t+1), d2 (g+8, 2t), d3 (g+8, 2t+1)
#pragma once

#include <stdint.h>

namespace kda {
namespace warpmma {

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// acc[nh][*] += P[0:16][0:16] * Q[0:16][0:16] (row-major fp32 with pitches pp, qp);
// acc[nh] holds output columns 8 nh .. 8 nh + 7 in the D fragment layout.
__device__ __forceinline__ void mm16_acc(const float* P, int pp, const float* Q, int qp, float (&acc)[2][4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        const float af[4] = {P[g * pp + 8 * ks + t], P[(g + 8) * pp + 8 * ks + t],
                             P[g * pp + 8 * ks + t + 4], P[(g + 8) * pp + 8 * ks + t + 4]};
        uint32_t ahi[4], alo[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            ahi[i] = to_tf32(af[i]);
            alo[i] = to_tf32(af[i] - __uint_as_float(ahi[i]));
        }
#pragma unroll
        for (int nh = 0; nh < 2; ++nh) {
            const float bf[2] = {Q[(8 * ks + t) * qp + 8 * nh + g], Q[(8 * ks + t + 4) * qp + 8 * nh + g]};
            uint32_t bhi[2], blo[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                bhi[i] = to_tf32(bf[i]);
                blo[i] = to_tf32(bf[i] - __uint_as_float(bhi[i]));
            }
            mma_tf32(acc[nh], alo, bhi);
            mma_tf32(acc[nh], ahi, blo);
            mma_tf32(acc[nh], ahi, bhi);
        }
    }
}

// D[0:16][0:16] = sign * acc (row-major fp32 with pitch dp).
__device__ __forceinline__ void store16(float* D, int dp, const float (&acc)[2][4], float sign) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
        *reinterpret_cast<float2*>(D + g * dp + 8 * nh + 2 * t) = make_float2(sign * acc[nh][0], sign * acc[nh][1]);
        *reinterpret_cast<float2*>(D + (g + 8) * dp + 8 * nh + 2 * t) =
            make_float2(sign * acc[nh][2], sign * acc[nh][3]);
    }
}

// ---- single-pass fp16 variant: mma.sync m16n8k16, f16 operands, fp32 accumulation ----
// Fragments (g = lane / 4, t = lane % 4; each register holds two f16, lower index in the low half):
//   A 16x16 row-major: a0 (g, 2t..2t+1), a1 (g+8, 2t..2t+1), a2 (g, 2t+8..2t+9), a3 (g+8, 2t+8..2t+9)
//   B 16x8 col-major:  b0 (2t..2t+1, g), b1 (2t+8..2t+9, g)
//   D 16x8: as for m16n8k8.
__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// acc[nh][*] += P[0:16][0:16] * Q[0:16][0:16] with both operands rounded to fp16.
__device__ __forceinline__ void mm16_acc_h(const float* P, int pp, const float* Q, int qp, float (&acc)[2][4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const float2 p0 = *reinterpret_cast<const float2*>(P + g * pp + 2 * t);
    const float2 p1 = *reinterpret_cast<const float2*>(P + (g + 8) * pp + 2 * t);
    const float2 p2 = *reinterpret_cast<const float2*>(P + g * pp + 2 * t + 8);
    const float2 p3 = *reinterpret_cast<const float2*>(P + (g + 8) * pp + 2 * t + 8);
    const uint32_t a[4] = {pack_half2(p0.x, p0.y), pack_half2(p1.x, p1.y), pack_half2(p2.x, p2.y),
                           pack_half2(p3.x, p3.y)};
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
        const int c = 8 * nh + g;
        const uint32_t b[2] = {pack_half2(Q[(2 * t) * qp + c], Q[(2 * t + 1) * qp + c]),
                               pack_half2(Q[(2 * t + 8) * qp + c], Q[(2 * t + 9) * qp + c])};
        mma_f16_16816(acc[nh], a, b);
    }
}

}  // namespace warpmma
}  // namespace kda
