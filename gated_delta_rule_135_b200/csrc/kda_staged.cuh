// kda_staged.cu -- the KDA chunked prefill forward as four separate kernels.
//
// fp32 CUDA-core arithmetic, every intra-chunk decay exp(Gamma_r - Gamma_i)
// formed pair by pair (never as a product of two exponentials), so the path
// is exact for any gate, including an unclamped one.  The state propagation
// runs on the tensor cores with split-bf16 operands (about 16 mantissa bits
// per product) and the state in fp32 TMEM.  It is the fallback of
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
#include "kda_tile.cuh"
#include "kda_chunks.cuh"
#include "umma.cuh"

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
// (b) intra-chunk WY: A, P, T = (I + A)^-1, W, U~.  grid (max_chunks, H), 512 threads.
constexpr int kIntraThreads = 512;
constexpr size_t kIntraSmem =
    sizeof(float) * (3 * kChunk * kPitch + 3 * kChunk * kPitchC + kChunk);

__global__ void __launch_bounds__(kIntraThreads) intra_chunk_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, const float* __restrict__ beta,
    const float* __restrict__ gamma, const int4* __restrict__ table,
    const int32_t* __restrict__ count, int H,
    float* __restrict__ w_out, float* __restrict__ ut_out, float* __restrict__ p_out,
    float* __restrict__ t_out) {
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

    const int64_t base = ((int64_t)e.y * H + h) * kHeadDim, ld = (int64_t)H * kHeadDim;
    stage<kChunk, kHeadDim, kIntraThreads>(sk, kPitch, k + base, ld, len, Identity{});
    stage<kChunk, kHeadDim, kIntraThreads>(sq, kPitch, q + base, ld, len, Identity{});
    stage<kChunk, kHeadDim, kIntraThreads>(sG, kPitch, gamma + base, ld, len, Identity{});
    for (int x = tid; x < kChunk * kPitchC; x += kIntraThreads) { sA[x] = 0.f; sP[x] = 0.f; sT[x] = 0.f; }
    if (tid < kChunk) sb[tid] = tid < len ? beta[((int64_t)e.y + tid) * H + h] : 0.f;
    __syncthreads();

    // A and P on 2 x 2 tiles of (r, i) pairs, tiles (tr, ti) with ti <= tr enumerated row-major:
    // rows 2 tr + {0, 1}, columns 2 ti + {0, 1}; every decay formed pair by pair.  Thread t takes
    // tile t over all channels; the tiles past the thread count go one per warp, its lanes
    // splitting the channels (reduced by shuffles, in a fixed order).
    constexpr int kTiles = (kChunk / 2) * (kChunk / 2 + 1) / 2;
    static_assert(kTiles <= kIntraThreads + kIntraThreads / 32, "pair tiles exceed one round");
    auto tile_coords = [](int p, int& tr, int& ti) {
        tr = (int)((sqrtf(8.f * p + 1.f) - 1.f) * 0.5f);
        while (tr * (tr + 1) / 2 > p) --tr;
        while ((tr + 1) * (tr + 2) / 2 <= p) ++tr;
        ti = p - tr * (tr + 1) / 2;
    };
    auto pair_sums = [&](int r0, int i0, int c_begin, int c_step, int n_c, float (&aa)[2][2], float (&ap)[2][2]) {
        for (int m = 0; m < n_c; ++m) {
            const int c = (c_begin + m * c_step) & (kHeadDim - 1);
            const float kr[2] = {sk[r0 * kPitch + c], sk[(r0 + 1) * kPitch + c]};
            const float qr[2] = {sq[r0 * kPitch + c], sq[(r0 + 1) * kPitch + c]};
            const float Gr[2] = {sG[r0 * kPitch + c], sG[(r0 + 1) * kPitch + c]};
            const float ki[2] = {sk[i0 * kPitch + c], sk[(i0 + 1) * kPitch + c]};
            const float Gi[2] = {sG[i0 * kPitch + c], sG[(i0 + 1) * kPitch + c]};
#pragma unroll
            for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int b2 = 0; b2 < 2; ++b2) {
                    // e^{Gamma_r - Gamma_i} <= 1 for i <= r (Gamma is non-increasing); the pairs
                    // above the diagonal of a diagonal tile are discarded below
                    const float kd = ki[b2] * expf(fminf(Gr[a] - Gi[b2], 0.f));
                    aa[a][b2] = fmaf(kr[a], kd, aa[a][b2]);
                    ap[a][b2] = fmaf(qr[a], kd, ap[a][b2]);
                }
        }
    };
    auto store_tile = [&](int r0, int i0, const float (&aa)[2][2], const float (&ap)[2][2]) {
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int b2 = 0; b2 < 2; ++b2) {
                const int r = r0 + a, i = i0 + b2;
                if (r >= len || i > r) continue;
                if (i < r) sA[r * kPitchC + i] = sb[r] * aa[a][b2];
                sP[r * kPitchC + i] = ap[a][b2];
            }
    };
    if (tid < kTiles) {
        int tr, ti;
        tile_coords(tid, tr, ti);
        if (2 * tr < len) {
            float aa[2][2] = {}, ap[2][2] = {};
            pair_sums(2 * tr, 2 * ti, tid, 1, kHeadDim, aa, ap);
            store_tile(2 * tr, 2 * ti, aa, ap);
        }
    }
    {
        const int p = kIntraThreads + tid / 32, lane = tid % 32;
        int tr = 0, ti = 0;
        if (p < kTiles) tile_coords(p, tr, ti);
        if (p < kTiles && 2 * tr < len) {           // uniform across the warp
            float aa[2][2] = {}, ap[2][2] = {};
            pair_sums(2 * tr, 2 * ti, lane, 32, kHeadDim / 32, aa, ap);
#pragma unroll
            for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int b2 = 0; b2 < 2; ++b2)
                    for (int o = 16; o > 0; o >>= 1) {
                        aa[a][b2] += __shfl_xor_sync(0xffffffffu, aa[a][b2], o);
                        ap[a][b2] += __shfl_xor_sync(0xffffffffu, ap[a][b2], o);
                    }
            if (lane == 0) store_tile(2 * tr, 2 * ti, aa, ap);
        }
    }
    __syncthreads();

    // T = (I + A)^-1 in 16 x 16 blocks.  Level 0: the diagonal blocks by forward substitution,
    // one column per thread.  Level d = 1..3: blocks (j + d, j) as T_ij = -T_ii sum_{j<=m<i} A_im T_mj,
    // the sum into scratch (sq: q is consumed) and then the product with T_ii.
    if (tid < kChunk) {
        const int o = tid & ~15, j = tid & 15;
        for (int r = 0; r < 16; ++r) {
            float acc = (r == j) ? 1.f : 0.f;
            for (int i = j; i < r; ++i) acc = fmaf(-sA[(o + r) * kPitchC + o + i], sT[(o + i) * kPitchC + o + j], acc);
            if (r >= j) sT[(o + r) * kPitchC + o + j] = acc;
        }
    }
    __syncthreads();
    float* scratch = sq;
    for (int d = 1; d < 4; ++d) {
        const int n = (4 - d) * 256;
        for (int x = tid; x < n; x += kIntraThreads) {
            const int bj = x / 256, bi = bj + d, r = (x / 16) % 16, cc = x % 16;
            float acc = 0.f;
            for (int m = 16 * bj; m < 16 * bi; ++m)
                acc = fmaf(sA[(16 * bi + r) * kPitchC + m], sT[m * kPitchC + 16 * bj + cc], acc);
            scratch[x] = acc;
        }
        __syncthreads();
        for (int x = tid; x < n; x += kIntraThreads) {
            const int bj = x / 256, bi = bj + d, r = (x / 16) % 16, cc = x % 16;
            float acc = 0.f;
            for (int m = 0; m <= r; ++m)
                acc = fmaf(sT[(16 * bi + r) * kPitchC + 16 * bi + m], scratch[bj * 256 + m * 16 + cc], acc);
            sT[(16 * bi + r) * kPitchC + 16 * bj + cc] = -acc;
        }
        __syncthreads();
    }
    // sq <- beta * gamma * k ; sG <- beta * v   (Gamma is consumed first)
    for (int x = tid; x < kChunk * kHeadDim; x += kIntraThreads) {
        const int r = x / kHeadDim, c = x % kHeadDim;
        sq[r * kPitch + c] = sb[r] * expf(sG[r * kPitch + c]) * sk[r * kPitch + c];
    }
    __syncthreads();
    stage<kChunk, kHeadDim, kIntraThreads>(sG, kPitch, v + base, ld, len, [sb](int r, int, float x) { return sb[r] * x; });
    __syncthreads();
    // W = T (beta gamma K), U~ = T (beta V): 2 x 8 register tiles, rows ty + 32 ii, columns tx + 16 jj
    {
        const int tx = tid % 16, ty = tid / 16;
        float aw[2][8], au[2][8];
        tile_zero(aw);
        tile_zero(au);
        tile_fma<2, 8, 32, 16, kPitchC, 1, kPitch, 1>(aw, sT, sq, ty, tx, 0, len);
        tile_fma<2, 8, 32, 16, kPitchC, 1, kPitch, 1>(au, sT, sG, ty, tx, 0, len);
#pragma unroll
        for (int ii = 0; ii < 2; ++ii) {
            const int r = ty + 32 * ii;
            if (r >= len) continue;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const int64_t idx = base + (int64_t)r * ld + tx + 16 * jj;
                w_out[idx] = aw[ii][jj];
                ut_out[idx] = au[ii][jj];
            }
        }
    }
    for (int x = tid; x < len * kChunk; x += kIntraThreads) {
        const int r = x / kChunk, i = x % kChunk;
        p_out[(((int64_t)e.y + r) * H + h) * kChunk + i] = sP[r * kPitchC + i];
    }
    if (t_out) {   // kept for the backward
        float* dst = t_out + ((int64_t)ci * H + h) * kChunk * kChunk;
        for (int x = tid; x < kChunk * kChunk; x += kIntraThreads) dst[x] = sT[(x / kChunk) * kPitchC + x % kChunk];
    }
}

// ---------------------------------------------------------------------------
// (c) inter-chunk state propagation on the tensor cores, serial over a sequence's chunks.  grid (N, H), 256 threads, one sequence and
// head per CTA with the fp32 state transposed in TMEM (lane j = state column, column c = state
// row).  Per chunk:
//   1. one pass over the TMEM state writes the chunk-start state, writes its split-bf16 copy
//      (the MN-major A operand S^T) and scales the TMEM state by gamma_C;
//   2. U^T = U~^T - S^T W^T         (M = 128 state columns j, N = 64 tokens, K = 128 rows c);
//   3. U = U~ + (that product) is written out and staged split-bf16 as the A operand U^T;
//   4. S^T += U^T Khat              (M = 128, N = 128 state rows c, K = 64 tokens).
// Operands are bf16 high and low parts of the fp32 values (hi.hi + hi.lo + lo.hi, fp32
// accumulation): about 16 mantissa bits per product, the state itself kept in fp32.
namespace stc {
using namespace umma;
constexpr uint32_t SH = 0, SL = 32768, WH = 65536, WL = 81920, UH = 98304, UL = 114688, KH = 131072,
                   KL = 147456, GC = 163840, BAR = GC + 512, TSLOT = BAR + 8, ABORT = BAR + 12;
constexpr uint32_t BYTES = BAR + 16;
constexpr uint32_t ALLOC = BYTES + 1008;
constexpr uint32_t TM_S = 0, TM_U = 128, TM_COLS = 256;
constexpr uint32_t IDESC_U = idesc_f16(128, 64, true, true, false);
constexpr uint32_t IDESC_S = idesc_f16(128, 128, true, true, true);
constexpr int kThreads = 256;

}  // namespace stc

__global__ void __launch_bounds__(stc::kThreads, 1) state_prop_tc_kernel(
    const __nv_bfloat16* __restrict__ k, const float* __restrict__ gamma,
    const float* __restrict__ w, const float* __restrict__ ut,
    const float* __restrict__ initial_state, const int32_t* __restrict__ cu_seqlens,
    int64_t seqlen, int64_t total_tokens, int H,
    float* __restrict__ u_out, float* __restrict__ chunk_states, int64_t max_chunks,
    float* __restrict__ final_state) {
    using namespace stc;
    const int n = blockIdx.x, h = blockIdx.y, tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + BAR);
    uint32_t* slot = reinterpret_cast<uint32_t*>(sm + TSLOT);
    volatile uint32_t* sAbort = reinterpret_cast<volatile uint32_t*>(sm + ABORT);
    float* sGC = reinterpret_cast<float*>(sm + GC);            // [128] e^{Gamma_last}
    int64_t b, e;
    seq_range(cu_seqlens, n, seqlen, total_tokens, &b, &e);
    const int64_t first = first_chunk_id(cu_seqlens, n, seqlen, total_tokens);
    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init_fence();
        *sAbort = 0u;
    }
    if (warp == 0) {
        tmem_alloc(slot, TM_COLS);
        tmem_relinquish();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *slot;
    // thread -> state column j (TMEM lane) and a half of the 128 state rows
    const int q = warp & 3, j = q * 32 + lane, c_half = warp >> 2;   // rows c in [64 c_half, 64 c_half + 64)
    const int64_t st_base = ((int64_t)n * H + h) * kHeadDim * kHeadDim;
    // the initial state into TMEM: S^T[j][c] = S[c][j]
#pragma unroll 1
    for (int cb = 0; cb < 4; ++cb) {
        uint32_t v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int c = 64 * c_half + 16 * cb + i;
            v[i] = __float_as_uint(initial_state ? initial_state[st_base + (int64_t)c * kHeadDim + j] : 0.f);
        }
        tmem_st16(taddr(tbase, q, TM_S + 64 * c_half + 16 * cb), v);
    }
    tmem_wait_st();
    uint32_t phase = 0u;
    bool aborted = false;
    const int64_t ld = (int64_t)H * kHeadDim;
    int64_t chunk_id = first;
    for (int64_t t0 = b; t0 < e && !aborted; t0 += kChunk, ++chunk_id) {
        const int len = (int)(e - t0 < kChunk ? e - t0 : kChunk);
        const int64_t base = (t0 * H + h) * kHeadDim;
        if (tid < kHeadDim) sGC[tid] = expf(gamma[base + (int64_t)(len - 1) * ld + tid]);
        // -W (K-major B of step 2: rows r, columns c) and Khat (MN-major B of step 4: rows r, columns c)
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int x = tid + kThreads * m, r = x >> 4, ch = x & 15;   // 64 rows x 16 chunks of 8
            float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, kk[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (r < len) {
                const int64_t off = base + (int64_t)r * ld + 8 * ch;
                const float4 w0 = *reinterpret_cast<const float4*>(w + off), w1 = *reinterpret_cast<const float4*>(w + off + 4);
                const float4 g0 = *reinterpret_cast<const float4*>(gamma + off), g1 = *reinterpret_cast<const float4*>(gamma + off + 4);
                const uint4 kb = *reinterpret_cast<const uint4*>(k + off);
                const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                const uint32_t kw[4] = {kb.x, kb.y, kb.z, kb.w};
                const float* gl = gamma + base + (int64_t)(len - 1) * ld + 8 * ch;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float kv = __uint_as_float((i & 1) ? (kw[i >> 1] & 0xffff0000u) : (kw[i >> 1] << 16));
                    a[i] = -wv[i];
                    kk[i] = kv * expf(gl[i] - gv[i]);
                }
            }
            uint4 hi, lo;
            split_bf16x8(a, hi, lo);
            *reinterpret_cast<uint4*>(sm + WH + sw128_chunk_off(r, ch, 64)) = hi;
            *reinterpret_cast<uint4*>(sm + WL + sw128_chunk_off(r, ch, 64)) = lo;
            split_bf16x8(kk, hi, lo);
            *reinterpret_cast<uint4*>(sm + KH + sw128_chunk_off(r, ch, 64)) = hi;
            *reinterpret_cast<uint4*>(sm + KL + sw128_chunk_off(r, ch, 64)) = lo;
        }
        __syncthreads();   // sGC
        // 1. the chunk-start state: out, split copy (MN-major A: rows c, columns j), scaled in TMEM
        const bool store_cs = chunk_id < max_chunks;
        if (!store_cs && tid == 0) record_error(KDA_DEVERR_BOUNDS);
#pragma unroll 1
        for (int cb = 0; cb < 4; ++cb) {
            uint32_t v[16];
            const uint32_t col = TM_S + 64 * c_half + 16 * cb;
            tmem_ld16(taddr(tbase, q, col), v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int c = 64 * c_half + 16 * cb + i;
                const float sv = __uint_as_float(v[i]);
                if (store_cs) chunk_states[(chunk_id * H + h) * kHeadDim * kHeadDim + (int64_t)c * kHeadDim + j] = sv;
                uint16_t hi, lo;
                split_bf16(sv, hi, lo);
                *reinterpret_cast<uint16_t*>(sm + SH + sw128_off(c, j, 128)) = hi;
                *reinterpret_cast<uint16_t*>(sm + SL + sw128_off(c, j, 128)) = lo;
                v[i] = __float_as_uint(sv * sGC[c]);
            }
            tmem_st16(taddr(tbase, q, col), v);
        }
        tmem_wait_st();
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        // 2. U^T (columns TM_U..) = S^T (-W)^T
        if (tid == 0) {
            fence_after_sync();
            const uint32_t sh = smem_u32(sm + SH), sl = smem_u32(sm + SL), wh = smem_u32(sm + WH),
                           wl = smem_u32(sm + WL);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                mma_f16(tbase + TM_U, desc_mnmajor(sh, 128, ks), desc_kmajor(wh, 64, ks), IDESC_U, ks > 0 ? 1u : 0u);
                mma_f16(tbase + TM_U, desc_mnmajor(sh, 128, ks), desc_kmajor(wl, 64, ks), IDESC_U, 1u);
                mma_f16(tbase + TM_U, desc_mnmajor(sl, 128, ks), desc_kmajor(wh, 64, ks), IDESC_U, 1u);
            }
            mma_commit(bar);
            if (!mbar_wait_bounded(bar, phase)) {
                record_error(KDA_DEVERR_TIMEOUT);
                *sAbort = 1u;
            }
        }
        __syncthreads();
        fence_after_sync();
        if (*sAbort != 0u) { aborted = true; break; }
        phase ^= 1u;
        // 3. U = U~ + U^T^T: out, and split as the MN-major A of step 4 (rows r, columns j)
#pragma unroll 1
        for (int rb = 0; rb < 2; ++rb) {
            uint32_t v[16];
            const int r0 = 32 * c_half + 16 * rb;                  // warps 0-3: r 0-31, warps 4-7: r 32-63
            tmem_ld16(taddr(tbase, q, TM_U + r0), v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = r0 + i;
                float uv = 0.f;
                if (r < len) {
                    const int64_t idx = base + (int64_t)r * ld + j;
                    uv = ut[idx] + __uint_as_float(v[i]);
                    u_out[idx] = uv;
                }
                uint16_t hi, lo;
                split_bf16(uv, hi, lo);
                *reinterpret_cast<uint16_t*>(sm + UH + sw128_off(r, j, 64)) = hi;
                *reinterpret_cast<uint16_t*>(sm + UL + sw128_off(r, j, 64)) = lo;
            }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        // 4. S^T += U^T Khat
        if (tid == 0) {
            fence_after_sync();
            const uint32_t uh = smem_u32(sm + UH), ul = smem_u32(sm + UL), kh = smem_u32(sm + KH),
                           kl = smem_u32(sm + KL);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                mma_f16(tbase + TM_S, desc_mnmajor(uh, 64, ks), desc_mnmajor(kh, 64, ks), IDESC_S, 1u);
                mma_f16(tbase + TM_S, desc_mnmajor(uh, 64, ks), desc_mnmajor(kl, 64, ks), IDESC_S, 1u);
                mma_f16(tbase + TM_S, desc_mnmajor(ul, 64, ks), desc_mnmajor(kh, 64, ks), IDESC_S, 1u);
            }
            mma_commit(bar);
            if (!mbar_wait_bounded(bar, phase)) {
                record_error(KDA_DEVERR_TIMEOUT);
                *sAbort = 1u;
            }
        }
        __syncthreads();
        fence_after_sync();
        if (*sAbort != 0u) { aborted = true; break; }
        phase ^= 1u;
    }
    if (aborted) {
        // the MMAs may still be running: give them (bounded) time before TMEM is released
        if (tid == 0) mbar_wait_bounded(bar, phase);
        fence_before_sync();
        __syncthreads();
    } else if (final_state) {
#pragma unroll 1
        for (int cb = 0; cb < 4; ++cb) {
            uint32_t v[16];
            tmem_ld16(taddr(tbase, q, TM_S + 64 * c_half + 16 * cb), v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i)
                final_state[st_base + (int64_t)(64 * c_half + 16 * cb + i) * kHeadDim + j] = __uint_as_float(v[i]);
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tbase, TM_COLS);
    }
}

// ---------------------------------------------------------------------------
// (d) output: O = scale ((gamma * Q) S_c + P U), bf16.  grid (max_chunks, H), 512 threads.
constexpr int kOutThreads = 512;
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
    const int64_t base = ((int64_t)e.y * H + h) * kHeadDim, ld = (int64_t)H * kHeadDim;
    stage<kHeadDim, kHeadDim, kOutThreads>(sS, kPitch, chunk_states + ((int64_t)ci * H + h) * kHeadDim * kHeadDim,
                                           kHeadDim, kHeadDim, Identity{});
    stage2<kChunk, kHeadDim, kOutThreads>(sQ, kPitch, gamma + base, q + base, ld, len,
                                          [](int, int, float G, float qv) { return qv * expf(G); });
    stage<kChunk, kHeadDim, kOutThreads>(sU, kPitch, u + base, ld, len, Identity{});
    stage<kChunk, kChunk, kOutThreads>(sP, kPitchC, p + ((int64_t)e.y * H + h) * kChunk, (int64_t)H * kChunk, len,
                                       Identity{});
    __syncthreads();
    // 2 x 8 register tiles: rows ty + 32 ii, columns tx + 16 jj
    const int tx = tid % 16, ty = tid / 16;
    float acc[2][8];
    tile_zero(acc);
    tile_fma<2, 8, 32, 16, kPitch, 1, kPitch, 1>(acc, sQ, sS, ty, tx, 0, kHeadDim);
    tile_fma<2, 8, 32, 16, kPitchC, 1, kPitch, 1>(acc, sP, sU, ty, tx, 0, len);
#pragma unroll
    for (int ii = 0; ii < 2; ++ii) {
        const int r = ty + 32 * ii;
        if (r >= len) continue;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
            out[base + (int64_t)r * ld + tx + 16 * jj] = __float2bfloat16_rn(scale * acc[ii][jj]);
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
    cudaError_t setup_err = once_per_device([](int) {
        cudaError_t err;
        if ((err = cudaFuncSetAttribute(intra_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)kIntraSmem)) != cudaSuccess) return err;
        if ((err = cudaFuncSetAttribute(state_prop_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)stc::ALLOC)) != cudaSuccess) return err;
        if ((err = cudaFuncSetAttribute(chunk_out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)kOutSmem)) != cudaSuccess) return err;
        return cudaSuccess;
    });
    if (setup_err != cudaSuccess) return setup_err;
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
                                                                      count, H, w, ut, p, a.t_mat);
    }
    if (a.N > 0) {
        dim3 gs((unsigned)a.N, (unsigned)H);
        state_prop_tc_kernel<<<gs, stc::kThreads, stc::ALLOC, stream>>>(
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
