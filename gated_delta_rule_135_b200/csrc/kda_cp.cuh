// kda_cp.cuh -- the state fold of the context-parallel prefill.
//
// The recurrence is affine in the state a segment starts from: after a segment,
// S_out = A S_in + B with A = the segment's final state from S_in = I and v = 0, and
// B = its final state from S_in = 0.  Splitting one long sequence over ranks, rank r
// starts from S_r = A_{r-1} S_{r-1} + B_{r-1}.  This kernel applies one such step per
// head: out_h = A_h S_h + B_h, all [128][128] fp32, A_h acting on the key dimension.
#pragma once

#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {
namespace cp {

constexpr int kTile = 32;

// One CTA per (head, 32 x 32 output tile); fp32 FMAs in a fixed order (deterministic).
__global__ void __launch_bounds__(kTile * 8) state_affine_kernel(const float* __restrict__ A,
                                                                 const float* __restrict__ S,
                                                                 const float* __restrict__ B,
                                                                 float* __restrict__ out) {
    __shared__ float sA[kTile][kTile + 1];
    __shared__ float sS[kTile][kTile + 1];
    const int h = blockIdx.z;
    const int i0 = blockIdx.y * kTile, j0 = blockIdx.x * kTile;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8 threads, 4 rows each
    const int64_t base = (int64_t)h * kHeadDim * kHeadDim;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int c0 = 0; c0 < kHeadDim; c0 += kTile) {
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
            const int r = ty * 4 + rr;
            sA[r][tx] = A[base + (int64_t)(i0 + r) * kHeadDim + c0 + tx];
            sS[r][tx] = S[base + (int64_t)(c0 + r) * kHeadDim + j0 + tx];
        }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < kTile; ++c)
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) acc[rr] = fmaf(sA[ty * 4 + rr][c], sS[c][tx], acc[rr]);
        __syncthreads();
    }
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
        const int64_t o = base + (int64_t)(i0 + ty * 4 + rr) * kHeadDim + j0 + tx;
        out[o] = acc[rr] + B[o];
    }
}

// Boundaries of the segments of one sequence of T tokens: cu[r] = min(r step, T), r = 0..R.
__global__ void segment_offsets_kernel(int32_t* cu, int R, int64_t step, int64_t T) {
    for (int r = threadIdx.x; r <= R; r += blockDim.x) cu[r] = (int32_t)(r * step < T ? r * step : T);
}

// Segment length for R pieces of T tokens, a whole number of 64-token chunks.
inline int64_t segment_step(int64_t T, int R) {
    const int64_t step = (T + R - 1) / R;
    return (step + kChunk - 1) / kChunk * kChunk;
}
inline int segment_count(int64_t T, int R) {
    const int64_t step = segment_step(T, R);
    return (int)((T + step - 1) / step);
}

}  // namespace cp

// The segment count for one long sequence with H heads on n_sm SMs.  The fused forward runs one
// CTA per (sequence, head) and a CTA takes its units in turn, so a pass costs about
// ceil(R H / n_sm) rounds of ceil(T / R / 64) chunks; segments take three passes (the two maps of
// every segment, then every segment from its folded state) and each fold step about 0.6
// chunk-times.  Returns the R (non-empty pieces) of least estimated time; 1 = the plain forward.
// Sequences shorter than 128 chunks run unsplit: there the launches and the workspace of the
// split cost about what it saves.
constexpr int64_t kMinSegmentedTokens = 128 * kChunk;
inline int choose_segments(int64_t T, int H, int n_sm, int max_segments = 64) {
    if (T < kMinSegmentedTokens || H <= 0 || n_sm <= 0) return 1;
    double best_cost = 0.0;
    int best = 1;
    for (int R = 1; R <= max_segments; ++R) {
        const int R_eff = cp::segment_count(T, R);
        const int64_t step = cp::segment_step(T, R);
        const int64_t longest = step < T ? step : T;
        const int64_t rounds = ((int64_t)R_eff * H + n_sm - 1) / n_sm;
        const int passes = R_eff == 1 ? 1 : 3;
        const double cost = (double)passes * (double)rounds * (double)((longest + kChunk - 1) / kChunk) +
                            0.6 * (double)(R_eff - 1);
        if (R == 1 || cost < best_cost) {
            best_cost = cost;
            best = R;
        }
    }
    return cp::segment_count(T, best);
}

cudaError_t launch_state_affine(const float* A, const float* S, const float* B, float* out, int H,
                                cudaStream_t stream) {
    if (H == 0) return cudaSuccess;
    const dim3 grid(kHeadDim / cp::kTile, kHeadDim / cp::kTile, (unsigned)H);
    cp::state_affine_kernel<<<grid, cp::kTile * 8, 0, stream>>>(A, S, B, out);
    return cudaGetLastError();
}

}  // namespace kda
