// kda_decode.cuh -- one recurrent KDA step per sequence (decode), in place on the state.
//
// For every sequence b and head h, with the fp32 state S (K x V, rows = key channels):
//   log a = max(-exp(A_log) * softplus(g + dt_bias), lower_bound)       (per channel)
//   w     = sum_c a_c k_c S[c, :]                                         (= (a * k)^T S)
//   S'    = Diag(a) S + beta k (v - w)^T       i.e. (I - beta k k^T) Diag(a) S + beta k v^T
//   o     = scale * S'^T q
// The step reads and writes the whole state once: it is bound by HBM bandwidth
// (2 x 64 KiB per sequence-head), so the kernel streams S through registers:
// one CTA per (sequence, head), thread j owns state column j (128 rows in
// registers), and every row access is one coalesced 512-byte segment per CTA.
#pragma once

#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {
namespace decode {

constexpr int kThreads = kHeadDim;   // one thread per state column

// kScalar: the scalar-gate variant, with g [B*H] and dt_bias [H] (one decay for all channels).
template <bool kScalar>
__global__ void __launch_bounds__(kThreads) kda_decode_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, const float* __restrict__ g, const float* __restrict__ beta,
    const float* __restrict__ A_log, const float* __restrict__ dt_bias, float lower_bound, float scale,
    float* __restrict__ state, __nv_bfloat16* __restrict__ out, int H) {
    const int bh = blockIdx.x;               // sequence * H + head
    const int h = bh % H;
    const int tid = threadIdx.x;
    __shared__ float s_ak[kHeadDim];         // a_c k_c
    __shared__ float s_a[kHeadDim];          // a_c
    __shared__ float s_k[kHeadDim];          // k_c
    __shared__ float s_q[kHeadDim];          // q_c
    {
        const int64_t idx = (int64_t)bh * kHeadDim + tid;   // channel c = tid
        const float gin = kScalar ? g[bh] + dt_bias[h] : g[idx] + dt_bias[h * kHeadDim + tid];
        const float la = gate_log_decay(gin, -expf(A_log[h]), lower_bound);
        const float a = expf(la);
        const float kc = __bfloat162float(k[idx]);
        s_a[tid] = a;
        s_k[tid] = kc;
        s_ak[tid] = a * kc;
        s_q[tid] = __bfloat162float(q[idx]);
    }
    __syncthreads();
    float* S = state + (int64_t)bh * kHeadDim * kHeadDim;   // [c][j]
    const int j = tid;
    float col[kHeadDim];
#pragma unroll
    for (int c = 0; c < kHeadDim; ++c) col[c] = S[c * kHeadDim + j];
    float w = 0.f;
#pragma unroll
    for (int c = 0; c < kHeadDim; ++c) w = fmaf(s_ak[c], col[c], w);
    const float u = beta[bh] * (__bfloat162float(v[(int64_t)bh * kHeadDim + j]) - w);
    float o = 0.f;
#pragma unroll
    for (int c = 0; c < kHeadDim; ++c) {
        const float s_new = fmaf(s_a[c], col[c], s_k[c] * u);
        S[c * kHeadDim + j] = s_new;
        o = fmaf(s_q[c], s_new, o);
    }
    out[(int64_t)bh * kHeadDim + j] = __float2bfloat16_rn(scale * o);
}

}  // namespace decode

cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* g, const float* beta,
                          const float* A_log, const float* dt_bias, float lower_bound, float scale,
                          float* state, void* out, int batch, int H, cudaStream_t stream, bool scalar_gate) {
    const int64_t blocks = (int64_t)batch * H;
    if (blocks == 0) return cudaSuccess;
    auto kernel = scalar_gate ? decode::kda_decode_kernel<true> : decode::kda_decode_kernel<false>;
    kernel<<<(unsigned)blocks, decode::kThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), g, beta, A_log, dt_bias, lower_bound, scale, state,
        static_cast<__nv_bfloat16*>(out), H);
    return cudaGetLastError();
}

}  // namespace kda
