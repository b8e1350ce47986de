// kda_common.cuh -- shared device helpers of the KDA library (not the oracle).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/kda.h"

namespace kda {

constexpr int kHeadDim = 128;   // K = V = 128 (the only supported head size)
constexpr int kChunk = 64;      // tokens per chunk

// Device error word: kernels OR bits into it instead of faulting.  The library
// is a single translation unit (kda_api.cu), so this is its only definition.
__device__ unsigned int g_device_error = 0;

__device__ __forceinline__ void record_error(unsigned int bits) {
    atomicOr(&g_device_error, bits);
}

// Gate: log a = max(-exp(A_log) * softplus(x), lower_bound), softplus written
// as max(x, 0) + log1p(exp(-|x|)) so that it never overflows.
__device__ __forceinline__ float gate_log_decay(float x, float neg_exp_alog, float lower_bound) {
    float sp = fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
    return fmaxf(neg_exp_alog * sp, lower_bound);
}

// Sequence n's token range, read from cu_seqlens (or the fixed layout).
// Offsets outside [0, Ttot] or decreasing are recorded and treated as empty.
__device__ __forceinline__ void seq_range(const int32_t* cu_seqlens, int n, int64_t seqlen,
                                          int64_t total_tokens, int64_t* begin, int64_t* end) {
    if (cu_seqlens == nullptr) {
        *begin = (int64_t)n * seqlen;
        *end = *begin + seqlen;
        return;
    }
    int64_t b = cu_seqlens[n], e = cu_seqlens[n + 1];
    if (b < 0 || e < b || e > total_tokens) {
        record_error(KDA_DEVERR_BAD_OFFSETS);
        *begin = 0;
        *end = 0;
        return;
    }
    *begin = b;
    *end = e;
}

}  // namespace kda
