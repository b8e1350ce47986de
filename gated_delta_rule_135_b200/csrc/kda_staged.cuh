// kda_staged.cu -- the KDA chunked prefill forward as four separate kernels.
//
// fp32 CUDA-core arithmetic, every intra-chunk decay exp(Gamma_r - Gamma_i)
// formed pair by pair (never as a product of two exponentials), so the path
// is exact for any gate, including an unclamped one.  It is the fallback of
// kda_fwd for gates too steep for the fused kernel's factored decays, and its
// workspace exposes every stage's output for checking.
//
// Chunk algebra (the WY / UT form of the recurrence; restated in the oracle):
// with Gamma_r = sum_{i<=r in chunk} log a_i and gamma = exp(Gamma),
//   A_ri = beta_r sum_c k_rc k_ic e^{Gamma_rc - Gamma_ic}   (i < r)
//   P_ri =        sum_c q_rc k_ic e^{Gamma_rc - Gamma_ic}   (i <= r)
//   T = (I + A)^-1,  W = T diag(beta)(gamma * K),  U~ = T diag(beta) V
//   U = U~ - W S,  O = scale ((gamma * Q) S + P U)
//   S' = Diag(gamma_last) S + Khat^T U,  Khat_i = k_i * e^{Gamma_last - Gamma_i}.

#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

namespace {

constexpr int kPitch = kHeadDim + 1;   // padded fp32 row pitch (bank spread)
constexpr int kPitchC = kChunk + 1;

__device__ __forceinline__ float bf16_to_f32(const __nv_bfloat16 x) { return __bfloat162float(x); }

// ---------------------------------------------------------------------------
// chunk plan: table[i] = (seq, t0, len, j) for chunk j of each sequence, in
// sequence order; count = number of chunks.  One block.
__global__ void __launch_bounds__(1024) plan_chunks_kernel(
    const int32_t* __restrict__ cu_seqlens, int N, int64_t seqlen, int64_t total_tokens,
    int4* __restrict__ table, int32_t* __restrict__ count, int64_t max_chunks) {
    __shared__ int warp_sums[32];
    __shared__ int64_t carry;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int base = 0; base < N; base += blockDim.x) {
        int n = base + threadIdx.x;
        int64_t b = 0, e = 0;
        int nch = 0;
        if (n < N) {
            seq_range(cu_seqlens, n, seqlen, total_tokens, &b, &e);
            nch = (int)((e - b + kChunk - 1) / kChunk);
        }
        // inclusive scan of nch over the block
        int x = nch;
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_sums[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int s = (lane < (int)(blockDim.x >> 5)) ? warp_sums[lane] : 0;
            for (int o = 1; o < 32; o <<= 1) {
                int y = __shfl_up_sync(0xffffffffu, s, o);
                if (lane >= o) s += y;
            }
            warp_sums[lane] = s;
        }
        __syncthreads();
        int64_t off = carry + (warp > 0 ? warp_sums[warp - 1] : 0) + x - nch;
        for (int j = 0; j < nch; ++j) {
            int64_t idx = off + j;
            if (idx >= max_chunks) { record_error(KDA_DEVERR_BOUNDS); break; }
            int64_t t0 = b + (int64_t)j * kChunk;
            int64_t len = e - t0 < kChunk ? e - t0 : kChunk;
            table[idx] = make_int4(n, (int)t0, (int)len, j);
        }
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) carry = off + nch;
        __syncthreads();
    }
    if (threadIdx.x == 0) *count = (int32_t)(carry < max_chunks ? carry : max_chunks);
}

// ---------------------------------------------------------------------------
// (a) gate pre-pass: Gamma[t,h,c] = sum over the chunk's tokens up to t of log a.
// grid (max_chunks, H), 128 threads (one channel each).
__global__ void __launch_bounds__(128) gate_cumsum_kernel(
    const float* __restrict__ g, const float* __restrict__ A_log, const float* __restrict__ dt_bias,
    float lower_bound, const int4* __restrict__ table, const int32_t* __restrict__ count, int H,
    float* __restrict__ gamma) {
    const int ci = blockIdx.x;
    if (ci >= *count) return;
    const int4 e = table[ci];
    const int h = blockIdx.y, c = threadIdx.x;
    const float nexp = -expf(A_log[h]);
    const float db = dt_bias[h * kHeadDim + c];
    float acc = 0.0f;
    for (int r = 0; r < e.z; ++r) {
        const int64_t idx = (((int64_t)e.y + r) * H + h) * kHeadDim + c;
        acc += gate_log_decay(g[idx] + db, nexp, lower_bound);
        gamma[idx] = acc;
    }
}

// ---------------------------------------------------------------------------
// (b) intra-chunk WY: A, P, T = (I + A)^-1, W, U~.  grid (max_chunks, H), 256 threads.
constexpr int kIntraThreads = 256;
constexpr size_t kIntraSmem =
    sizeof(float) * (3 * kChunk * kPitch + 3 * kChunk * kPitchC + kChunk);

__global__ void __launch_bounds__(kIntraThreads) intra_chunk_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, const float* __restrict__ beta,
    const float* __restrict__ gamma, const int4* __restrict__ table,
    const int32_t* __restrict__ count, int H,
    float* __restrict__ w_out, float* __restrict__ ut_out, float* __restrict__ p_out) {
    const int ci = blockIdx.x;
    if (ci >= *count) return;
    const int4 e = table[ci];
    const int h = blockIdx.y, tid = threadIdx.x;
    const int len = e.z;
    extern __shared__ float sm[];
    float* sk = sm;                          // [64][129] k
    float* sq = sk + kChunk * kPitch;        // [64][129] q, later beta*gamma*k
    float* sG = sq + kChunk * kPitch;        // [64][129] Gamma, later beta*v
    float* sA = sG + kChunk * kPitch;        // [64][65]
    float* sP = sA + kChunk * kPitchC;       // [64][65]
    float* sT = sP + kChunk * kPitchC;       // [64][65]
    float* sb = sT + kChunk * kPitchC;       // [64] beta

    for (int x = tid; x < kChunk * kHeadDim; x += kIntraThreads) {
        const int r = x / kHeadDim, c = x % kHeadDim;
        float kv = 0.f, qv = 0.f, gv = 0.f;
        if (r < len) {
            const int64_t idx = (((int64_t)e.y + r) * H + h) * kHeadDim + c;
            kv = bf16_to_f32(k[idx]);
            qv = bf16_to_f32(q[idx]);
            gv = gamma[idx];
        }
        sk[r * kPitch + c] = kv;
        sq[r * kPitch + c] = qv;
        sG[r * kPitch + c] = gv;
    }
    for (int x = tid; x < kChunk * kPitchC; x += kIntraThreads) { sA[x] = 0.f; sP[x] = 0.f; sT[x] = 0.f; }
    if (tid < kChunk) sb[tid] = tid < len ? beta[((int64_t)e.y + tid) * H + h] : 0.f;
    __syncthreads();

    // lower-triangle pairs (r, i), i <= r, enumerated row-major
    constexpr int kPairs = kChunk * (kChunk + 1) / 2;
    for (int p = tid; p < kPairs; p += kIntraThreads) {
        int r = (int)((sqrtf(8.f * p + 1.f) - 1.f) * 0.5f);
        while (r * (r + 1) / 2 > p) --r;
        while ((r + 1) * (r + 2) / 2 <= p) ++r;
        const int i = p - r * (r + 1) / 2;
        if (r >= len) continue;
        const float* kr = sk + r * kPitch;
        const float* ki = sk + i * kPitch;
        const float* qr = sq + r * kPitch;
        const float* Gr = sG + r * kPitch;
        const float* Gi = sG + i * kPitch;
        float acc_a = 0.f, acc_p = 0.f;
        for (int cc = 0; cc < kHeadDim; ++cc) {
            const int c = (cc + tid) & (kHeadDim - 1);
            const float dec = expf(Gr[c] - Gi[c]);   // <= 1: Gamma is non-increasing in r
            const float kd = ki[c] * dec;
            acc_a = fmaf(kr[c], kd, acc_a);
            acc_p = fmaf(qr[c], kd, acc_p);
        }
        if (i < r) sA[r * kPitchC + i] = sb[r] * acc_a;
        sP[r * kPitchC + i] = acc_p;
    }
    __syncthreads();

    // T = (I + A)^-1 by forward substitution, one column per thread
    if (tid < kChunk) {
        const int j = tid;
        for (int r = j; r < kChunk; ++r) {
            float s = (r == j) ? 1.f : 0.f;
            for (int i = j; i < r; ++i) s = fmaf(-sA[r * kPitchC + i], sT[i * kPitchC + j], s);
            sT[r * kPitchC + j] = s;
        }
    }
    __syncthreads();
    // sq <- beta * gamma * k ; sG <- beta * v   (Gamma is consumed first)
    for (int x = tid; x < kChunk * kHeadDim; x += kIntraThreads) {
        const int r = x / kHeadDim, c = x % kHeadDim;
        sq[r * kPitch + c] = sb[r] * expf(sG[r * kPitch + c]) * sk[r * kPitch + c];
    }
    __syncthreads();
    for (int x = tid; x < kChunk * kHeadDim; x += kIntraThreads) {
        const int r = x / kHeadDim, c = x % kHeadDim;
        float vv = 0.f;
        if (r < len) vv = bf16_to_f32(v[(((int64_t)e.y + r) * H + h) * kHeadDim + c]);
        sG[r * kPitch + c] = sb[r] * vv;
    }
    __syncthreads();
    // W = T (beta gamma K), U~ = T (beta V): column c = tid % 128, rows tid/128 + 2m
    {
        const int c = tid % kHeadDim;
        for (int r = tid / kHeadDim; r < len; r += kIntraThreads / kHeadDim) {
            float aw = 0.f, au = 0.f;
            for (int i = 0; i <= r; ++i) {
                const float t = sT[r * kPitchC + i];
                aw = fmaf(t, sq[i * kPitch + c], aw);
                au = fmaf(t, sG[i * kPitch + c], au);
            }
            const int64_t idx = (((int64_t)e.y + r) * H + h) * kHeadDim + c;
            w_out[idx] = aw;
            ut_out[idx] = au;
        }
    }
    for (int x = tid; x < len * kChunk; x += kIntraThreads) {
        const int r = x / kChunk, i = x % kChunk;
        p_out[(((int64_t)e.y + r) * H + h) * kChunk + i] = sP[r * kPitchC + i];
    }
}

// ---------------------------------------------------------------------------
// (c) inter-chunk state propagation, serial over a sequence's chunks.
// grid (N, H, 128 / kSlab), 256 threads; each block owns a 128 x kSlab column slab of S.
constexpr int kSlab = 32;
constexpr int kStateThreads = 256;
constexpr size_t kStateSmem =
    sizeof(float) * (kHeadDim * (kSlab + 1) + 2 * kChunk * kPitch + kChunk * (kSlab + 1) + kHeadDim);

__global__ void __launch_bounds__(kStateThreads) state_prop_kernel(
    const __nv_bfloat16* __restrict__ k, const float* __restrict__ gamma,
    const float* __restrict__ w, const float* __restrict__ ut,
    const float* __restrict__ initial_state, const int32_t* __restrict__ cu_seqlens,
    int64_t seqlen, int64_t total_tokens, int H,
    float* __restrict__ u_out, float* __restrict__ chunk_states, int64_t max_chunks,
    float* __restrict__ final_state) {
    const int n = blockIdx.x, h = blockIdx.y, slab = blockIdx.z, tid = threadIdx.x;
    const int j0 = slab * kSlab;
    extern __shared__ float sm[];
    float* sS = sm;                                  // [128][33]
    float* sW = sS + kHeadDim * (kSlab + 1);         // [64][129] W, later Khat
    float* sK = sW + kChunk * kPitch;                // [64][129] k -> Khat
    float* sU = sK + kChunk * kPitch;                // [64][33]
    float* sgC = sU + kChunk * (kSlab + 1);          // [128] gamma_last
    __shared__ int64_t s_first_chunk;

    int64_t b, e;
    seq_range(cu_seqlens, n, seqlen, total_tokens, &b, &e);
    // global chunk id of this sequence's first chunk: sum over earlier sequences
    {
        int64_t part = 0;
        for (int m = tid; m < n; m += kStateThreads) {
            int64_t mb, me;
            seq_range(cu_seqlens, m, seqlen, total_tokens, &mb, &me);
            part += (me - mb + kChunk - 1) / kChunk;
        }
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        __shared__ int64_t warp_part[kStateThreads / 32];
        if ((tid & 31) == 0) warp_part[tid >> 5] = part;
        __syncthreads();
        if (tid == 0) {
            int64_t s = 0;
            for (int x = 0; x < kStateThreads / 32; ++x) s += warp_part[x];
            s_first_chunk = s;
        }
        __syncthreads();
    }
    for (int x = tid; x < kHeadDim * kSlab; x += kStateThreads) {
        const int c = x / kSlab, j = x % kSlab;
        sS[c * (kSlab + 1) + j] = initial_state
            ? initial_state[(((int64_t)n * H + h) * kHeadDim + c) * kHeadDim + j0 + j] : 0.f;
    }
    __syncthreads();
    int64_t chunk_id = s_first_chunk;
    for (int64_t t0 = b; t0 < e; t0 += kChunk, ++chunk_id) {
        const int len = (int)(e - t0 < kChunk ? e - t0 : kChunk);
        // stage W and k/Gamma of the chunk
        for (int x = tid; x < kChunk * kHeadDim; x += kStateThreads) {
            const int r = x / kHeadDim, c = x % kHeadDim;
            float wv = 0.f, kv = 0.f;
            if (r < len) {
                const int64_t idx = ((t0 + r) * H + h) * kHeadDim + c;
                wv = w[idx];
                kv = bf16_to_f32(k[idx]);
            }
            sW[r * kPitch + c] = wv;
            sK[r * kPitch + c] = kv;
        }
        if (tid < kHeadDim) sgC[tid] = gamma[((t0 + len - 1) * H + h) * kHeadDim + tid];
        __syncthreads();
        // Khat_ic = k_ic e^{Gamma_last,c - Gamma_ic}
        for (int x = tid; x < len * kHeadDim; x += kStateThreads) {
            const int r = x / kHeadDim, c = x % kHeadDim;
            const float G = gamma[((t0 + r) * H + h) * kHeadDim + c];
            sK[r * kPitch + c] *= expf(sgC[c] - G);
        }
        // record the chunk's starting state
        if (chunk_id < max_chunks) {
            for (int x = tid; x < kHeadDim * kSlab; x += kStateThreads) {
                const int c = x / kSlab, j = x % kSlab;
                chunk_states[((chunk_id * H + h) * kHeadDim + c) * kHeadDim + j0 + j] =
                    sS[c * (kSlab + 1) + j];
            }
        } else if (tid == 0) {
            record_error(KDA_DEVERR_BOUNDS);
        }
        __syncthreads();
        // U = U~ - W S   (rows r, slab columns j)
        {
            const int j = tid % kSlab;
            for (int r = tid / kSlab; r < kChunk; r += kStateThreads / kSlab) {
                float acc = 0.f;
                if (r < len) {
                    acc = ut[((t0 + r) * H + h) * kHeadDim + j0 + j];
                    for (int c = 0; c < kHeadDim; ++c)
                        acc = fmaf(-sW[r * kPitch + c], sS[c * (kSlab + 1) + j], acc);
                    u_out[((t0 + r) * H + h) * kHeadDim + j0 + j] = acc;
                }
                sU[r * (kSlab + 1) + j] = acc;
            }
        }
        __syncthreads();
        // S = Diag(gamma_last) S + Khat^T U
        {
            const int j = tid % kSlab;
            for (int c = tid / kSlab; c < kHeadDim; c += kStateThreads / kSlab) {
                float acc = expf(sgC[c]) * sS[c * (kSlab + 1) + j];
                for (int r = 0; r < len; ++r)
                    acc = fmaf(sK[r * kPitch + c], sU[r * (kSlab + 1) + j], acc);
                sS[c * (kSlab + 1) + j] = acc;
            }
        }
        __syncthreads();
    }
    if (final_state) {
        for (int x = tid; x < kHeadDim * kSlab; x += kStateThreads) {
            const int c = x / kSlab, j = x % kSlab;
            final_state[(((int64_t)n * H + h) * kHeadDim + c) * kHeadDim + j0 + j] =
                sS[c * (kSlab + 1) + j];
        }
    }
}

// ---------------------------------------------------------------------------
// (d) output: O = scale ((gamma * Q) S_c + P U), bf16.  grid (max_chunks, H), 256 threads.
constexpr int kOutThreads = 256;
constexpr size_t kOutSmem =
    sizeof(float) * (kChunk * kPitch + kHeadDim * kPitch + kChunk * kPitchC + kChunk * kPitch);

__global__ void __launch_bounds__(kOutThreads) chunk_out_kernel(
    const __nv_bfloat16* __restrict__ q, const float* __restrict__ gamma,
    const float* __restrict__ chunk_states, const float* __restrict__ p,
    const float* __restrict__ u, const int4* __restrict__ table,
    const int32_t* __restrict__ count, int H, float scale, __nv_bfloat16* __restrict__ out) {
    const int ci = blockIdx.x;
    if (ci >= *count) return;
    const int4 e = table[ci];
    const int h = blockIdx.y, tid = threadIdx.x, len = e.z;
    extern __shared__ float sm[];
    float* sQ = sm;                          // [64][129] gamma * q
    float* sS = sQ + kChunk * kPitch;        // [128][129]
    float* sP = sS + kHeadDim * kPitch;      // [64][65]
    float* sU = sP + kChunk * kPitchC;       // [64][129]
    for (int x = tid; x < kChunk * kHeadDim; x += kOutThreads) {
        const int r = x / kHeadDim, c = x % kHeadDim;
        float qv = 0.f, uv = 0.f;
        if (r < len) {
            const int64_t idx = (((int64_t)e.y + r) * H + h) * kHeadDim + c;
            qv = bf16_to_f32(q[idx]) * expf(gamma[idx]);
            uv = u[idx];
        }
        sQ[r * kPitch + c] = qv;
        sU[r * kPitch + c] = uv;
    }
    for (int x = tid; x < kHeadDim * kHeadDim; x += kOutThreads) {
        const int c = x / kHeadDim, j = x % kHeadDim;
        sS[c * kPitch + j] = chunk_states[(((int64_t)ci * H + h) * kHeadDim + c) * kHeadDim + j];
    }
    for (int x = tid; x < kChunk * kChunk; x += kOutThreads) {
        const int r = x / kChunk, i = x % kChunk;
        sP[r * kPitchC + i] = r < len ? p[(((int64_t)e.y + r) * H + h) * kChunk + i] : 0.f;
    }
    __syncthreads();
    const int j = tid % kHeadDim;
    for (int r = tid / kHeadDim; r < len; r += kOutThreads / kHeadDim) {
        float acc = 0.f;
        for (int c = 0; c < kHeadDim; ++c) acc = fmaf(sQ[r * kPitch + c], sS[c * kPitch + j], acc);
        for (int i = 0; i <= r; ++i) acc = fmaf(sP[r * kPitchC + i], sU[i * kPitch + j], acc);
        out[(((int64_t)e.y + r) * H + h) * kHeadDim + j] = __float2bfloat16_rn(scale * acc);
    }
}

}  // namespace

// ---------------------------------------------------------------------------
// host side

StagedLayout staged_layout(int64_t total_tokens, int H, int N) {
    StagedLayout L{};
    auto align = [](size_t x) { return (x + 255) & ~size_t(255); };
    L.max_chunks = (total_tokens + kChunk - 1) / kChunk + N;
    size_t off = 0;
    L.chunk_table = off;
    off = align(off + sizeof(int4) * (size_t)L.max_chunks + sizeof(int32_t));
    const size_t tok = (size_t)total_tokens * (size_t)H;
    L.gamma = off;   off = align(off + sizeof(float) * tok * kHeadDim);
    L.w = off;       off = align(off + sizeof(float) * tok * kHeadDim);
    L.u_tilde = off; off = align(off + sizeof(float) * tok * kHeadDim);
    L.p = off;       off = align(off + sizeof(float) * tok * kChunk);
    L.u = off;       off = align(off + sizeof(float) * tok * kHeadDim);
    L.chunk_states = off;
    off = align(off + sizeof(float) * (size_t)L.max_chunks * H * kHeadDim * kHeadDim);
    L.total = off;
    return L;
}

cudaError_t launch_staged(const StagedArgs& a, char* ws, const StagedLayout& L, cudaStream_t stream) {
    static bool attrs_set = false;
    if (!attrs_set) {
        cudaError_t err;
        if ((err = cudaFuncSetAttribute(intra_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)kIntraSmem)) != cudaSuccess) return err;
        if ((err = cudaFuncSetAttribute(state_prop_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)kStateSmem)) != cudaSuccess) return err;
        if ((err = cudaFuncSetAttribute(chunk_out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)kOutSmem)) != cudaSuccess) return err;
        attrs_set = true;
    }
    int4* table = reinterpret_cast<int4*>(ws + L.chunk_table);
    int32_t* count = reinterpret_cast<int32_t*>(ws + L.chunk_table + sizeof(int4) * L.max_chunks);
    float* gamma = reinterpret_cast<float*>(ws + L.gamma);
    float* w = reinterpret_cast<float*>(ws + L.w);
    float* ut = reinterpret_cast<float*>(ws + L.u_tilde);
    float* p = reinterpret_cast<float*>(ws + L.p);
    float* u = reinterpret_cast<float*>(ws + L.u);
    float* cs = reinterpret_cast<float*>(ws + L.chunk_states);
    const int H = a.H;
    const auto* q = static_cast<const __nv_bfloat16*>(a.q);
    const auto* k = static_cast<const __nv_bfloat16*>(a.k);
    const auto* v = static_cast<const __nv_bfloat16*>(a.v);

    plan_chunks_kernel<<<1, 1024, 0, stream>>>(a.cu_seqlens, a.N, a.seqlen, a.total_tokens,
                                                table, count, L.max_chunks);
    if (L.max_chunks > 0) {
        dim3 gc((unsigned)L.max_chunks, (unsigned)H);
        gate_cumsum_kernel<<<gc, 128, 0, stream>>>(a.g, a.A_log, a.dt_bias, a.lower_bound, table,
                                                   count, H, gamma);
        intra_chunk_kernel<<<gc, kIntraThreads, kIntraSmem, stream>>>(q, k, v, a.beta, gamma, table,
                                                                      count, H, w, ut, p);
    }
    if (a.N > 0) {
        dim3 gs((unsigned)a.N, (unsigned)H, kHeadDim / kSlab);
        state_prop_kernel<<<gs, kStateThreads, kStateSmem, stream>>>(
            k, gamma, w, ut, a.initial_state, a.cu_seqlens, a.seqlen, a.total_tokens, H, u, cs,
            L.max_chunks, a.final_state);
    }
    if (L.max_chunks > 0 && a.out) {   // the backward runs the forward for its intermediates only
        dim3 gc((unsigned)L.max_chunks, (unsigned)H);
        chunk_out_kernel<<<gc, kOutThreads, kOutSmem, stream>>>(
            q, gamma, cs, p, u, table, count, H, a.scale, static_cast<__nv_bfloat16*>(a.out));
    }
    return cudaGetLastError();
}

}  // namespace kda
