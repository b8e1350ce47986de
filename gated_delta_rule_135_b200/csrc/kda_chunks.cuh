// kda_chunks.cuh -- chunk bookkeeping shared by the serial chunk scans (staged forward and
// backward).
#pragma once

#include "kda_common.cuh"

namespace kda {

// Global chunk index of sequence n's first chunk: the chunks of the sequences before it
// (one block computes it; every thread gets the value).
__device__ inline int64_t first_chunk_id(const int32_t* cu_seqlens, int n, int64_t seqlen, int64_t total_tokens) {
    __shared__ int64_t warp_part[32];
    __shared__ int64_t result;
    int64_t part = 0;
    for (int m = threadIdx.x; m < n; m += blockDim.x) {
        int64_t mb, me;
        seq_range(cu_seqlens, m, seqlen, total_tokens, &mb, &me);
        part += (me - mb + kChunk - 1) / kChunk;
    }
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if ((threadIdx.x & 31) == 0) warp_part[threadIdx.x >> 5] = part;
    __syncthreads();
    if (threadIdx.x == 0) {
        int64_t s = 0;
        for (int x = 0; x < (int)(blockDim.x >> 5); ++x) s += warp_part[x];
        result = s;
    }
    __syncthreads();
    return result;
}

}  // namespace kda
