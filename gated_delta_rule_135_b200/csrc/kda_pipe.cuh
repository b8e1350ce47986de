// kda_pipe.cuh -- the product KDA chunked-prefill kernel (kda_fwd): persistent,
// warp-specialised, sm_100a.
//
// One CTA per SM walks a static longest-first "snake" schedule of (sequence, head) units.
// Its 16 warps have three roles that work on consecutive 64-token chunks at once:
//
//   chain warps 0-3     thread v owns value column v of the state.  The state lives in TMEM
//                       transposed (S^T: lane v, column c) in fp32, lane v scaled by its own
//                       power of two 2^-sigma_v: every column of S evolves on its own and the
//                       recurrence is linear in it, so the scaling is exact and keeps every
//                       fp16 MMA operand derived from the state inside the fp16 range.  Per
//                       chunk (A operands read straight from TMEM, B operands from shared memory):
//                         S^T -> fp16 (TMEM);  S^T <- S^T Diag(gamma_C)  (after the next MMA issues)
//                         [O | Y]^T  = S^T [gamma Q ; -beta gamma K]^T                    K = 128
//                         Y^T       += 2^-sigma (beta V)^T  -> fp16 (TMEM)
//                         U^T        = Y^T T^T                                             K = 64
//                         U^T -> fp16 (TMEM);  [S | O]^T += U^T [Khat | P^T]              N = 192
//                         O^T -> bf16 out (times scale 2^sigma_v)
//   element warps 8-15  chunk n: beta, gate and decay factors (thread: 4 channels x 8 tokens),
//                       every decayed operand tile and the chunk's metadata (scalar gate: V^T)
//   aux warps 4-7       meanwhile chunk n - 1: the A / P read-out (one warp per TMEM lane
//                       quarter) and T = (I + A)^-1; chunk n's V^T and exact P diagonal q_r . k_r
//                       (channel gate), and the TMA load of chunk n + 1's gate input
//   (the chain's thread 0 also issues the A/P MMA and the TMA loads of the next chunk's q, k, v)
//
// Y = beta V - beta gamma K S and U = T Y is the WY/UT form U = T diag(beta)(V - (gamma K) S)
// of the chunk (U~ - W S with the product by T taken last), so that the part of the chain that
// needs the state does not wait for the triangular solve: the element warps build chunk n + 1
// while the aux warps solve chunk n and the chain warps finish it.
//
// Decay factors (16-token blocks; running products of a_t): the A/P MMA (bf16, M = 128 x N = 160)
// multiplies [k R' ; q R'] (R'_r = e^{Gamma_r - Gamma_(block middle)}) by the diagonal-block
// operand k E' (E'_i = e^{Gamma_(block middle) - Gamma_i}) and the block-distance operands
// k E F_d (E = e^{Gamma_(block end) - Gamma_i} <= 1, F_d <= 1 the decay from block J's end to the
// middle of block J + d).  Every factor lies within e^{+-8 |lower_bound|}, so with |q|, |k| < 2^15
// the kernel takes lower_bound >= -9.5 (8 x 9.5 = 76 and 2^15 e^76 < 3.4e38); steeper gates take
// the staged path.  P's main diagonal (no decay, the dominant output term) is taken exactly in fp32.
//
// Operand precision: decay blocks bf16, everything that multiplies T, S, Y, U or P in fp16,
// accumulation and the carried state in fp32.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "umma.cuh"
#include "warp_mma.cuh"

namespace kda {
namespace pipe {

using namespace umma;

constexpr int kThreads = 512;
constexpr int kAuxWarp0 = 4, kElemWarp0 = 8;
// named barriers (0 is __syncthreads)
constexpr uint32_t BAR_CHAIN = 2, BAR_AUX = 3, BAR_ELEM = 4;

// ---- shared memory (bytes from a 1024-aligned base) ----
constexpr uint32_t IN_Q = 0;           // bf16 [64][128] row-major TMA boxes
constexpr uint32_t IN_K = 16384;
constexpr uint32_t IN_V = 32768;
constexpr uint32_t IN_BYTES = 49152;
constexpr uint32_t AP_A = 49152;       // bf16 K-major [128 rows][128]: k R' rows 0-63, q R' rows 64-127
                                       // (between a chunk's A/P MMA and the next chunk's tiles: the
                                       // next chunk's raw gate input, fp32 [64][128])
constexpr uint32_t AP_B = 81920;       // bf16 K-major [160 rows][128]: k E' | C1 | C2 | C3
constexpr uint32_t B1 = 122880;        // fp16 K-major [128 rows][128]: gamma q rows 0-63, -beta gamma k 64-127
constexpr uint32_t B2 = 155648;        // fp16 MN-major, K = 64 tokens: Khat (c 0-63 | c 64-127) | P^T
constexpr uint32_t KH = B2;
constexpr uint32_t PT = B2 + 16384;
constexpr uint32_t VT = 180224;        // bf16 [128 v][64 i]: 128-byte rows, 16-byte chunk j at j ^ (v & 7)
constexpr uint32_t T16 = 196608;       // fp16 K-major [64 r][64 i]
constexpr uint32_t MISC = 204800;
constexpr uint32_t S_BETA = MISC;              // fp32 [2][64] (by chunk parity)
constexpr uint32_t S_GC = MISC + 512;          // fp32 [2][128] gamma_C = e^{Gamma_63}
constexpr uint32_t S_PTOT = MISC + 1536;       // fp32 [4][128] per-block products of a
constexpr uint32_t S_ORDER = MISC + 4096;      // int16 [kSortLimit]
constexpr int kSortLimit = 512;
constexpr uint32_t S_META = S_ORDER + 2 * kSortLimit;   // int32 [2][16] chunk metadata
constexpr uint32_t S_BARS = S_META + 128;               // u64 [16]
constexpr int kNumBars = 11;
constexpr uint32_t S_TMEM = S_BARS + 128;               // u32 tmem base, abort flag, read-out data sequence
constexpr uint32_t S_PH = S_TMEM + 16;                  // u64 [kPhases + 3] (phase-clock builds)
constexpr int kPhases = 24;
// The triangular solve's scratch, apart from the A/P operand tiles (which the element warps
// rewrite for the next chunk while the aux warps solve): A's diagonal 16 x 16 blocks in fp32
// (row pitch 20 floats), its six blocks below the diagonal and the solve's intermediate blocks
// in fp16 (row pitch 24 halves; both pitches keep row accesses free of bank conflicts).
constexpr uint32_t S_PHALF = 210432;                    // fp32 [4][128] product of a over each block's first 8 tokens
constexpr uint32_t SV = S_PHALF + 2048;
constexpr int kAdPitch = 20;
constexpr int kHp = 24;
constexpr uint32_t kHBlk = 16 * kHp * 2;                // bytes of one fp16 block
constexpr uint32_t SV_AD = SV;                          // fp32 [4][16][20]
constexpr uint32_t SV_AL = SV_AD + 4 * 16 * kAdPitch * 4;   // fp16 [6][16][24]: A10 A20 A21 A30 A31 A32
constexpr uint32_t SV_SC = SV_AL + 6 * kHBlk;           // fp16 [8][16][24] intermediates
constexpr uint32_t SC_Y0 = SV_SC, SC_Y2 = SV_SC + kHBlk, SC_T10B = SV_SC + 2 * kHBlk, SC_X20 = SV_SC + 3 * kHBlk,
                   SC_X30 = SV_SC + 4 * kHBlk, SC_X21 = SV_SC + 5 * kHBlk, SC_X31 = SV_SC + 6 * kHBlk,
                   SC_Y32 = SV_SC + 7 * kHBlk;
constexpr uint32_t S_PD2 = SV_SC + 8 * kHBlk;          // fp32 [2][2][64] halves of q_r . k_r, by chunk parity
constexpr uint32_t SMEM_BYTES = S_PD2 + 1024;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;
static_assert(S_PH + 8 * (kPhases + 3) <= S_PHALF, "phase slots below the half-block products");
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");

// ---- TMEM columns ----
constexpr uint32_t TM_S = 0;      // S^T fp32 [128 v][128 c]
constexpr uint32_t TM_O = 128;    // O^T fp32 [v][64 r]
constexpr uint32_t TM_Y = 192;    // Y^T then U^T, fp32 [v][64 i]
constexpr uint32_t TM_H = 256;    // fp16 A operands: S^T (64 columns); then Y^T (+0) and U^T (+32)
constexpr uint32_t TM_AP = 320;   // A/P accumulator [128 rows][160]
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t IDESC_AP = idesc_f16(128, 160, true, false, false);
constexpr uint32_t IDESC_AP_S = idesc_f16(128, 64, true, false, false);   // scalar gate: [K ; Q] K^T
// Scalar-gate variant: q, k, v arrive as 128-byte-swizzled 64-channel blocks of 64 rows (8 KB
// each), laid out k0 | q0 | k1 | q1 | v0 | v1 in the input region, so that [k ; q] is the 128-row
// K-major A operand of the A/P MMA and k its B operand; its per-token gate quantities share the
// block-product array, one set per chunk parity (the aux warps read a chunk's Gamma while the
// element warps form the next chunk's).
__host__ __device__ constexpr uint32_t s_gam(uint32_t sl) { return S_PTOT + sl * 768u; }   // fp32 [64] Gamma (log2)
__host__ __device__ constexpr uint32_t s_ge(uint32_t sl) { return s_gam(sl) + 256u; }      // fp32 [64] 2^Gamma
__host__ __device__ constexpr uint32_t s_kf(uint32_t sl) { return s_gam(sl) + 512u; }      // fp32 [64] 2^(Gamma_63 - Gamma)
constexpr uint32_t IDESC_OY = idesc_f16(128, 128, false, false, false);
constexpr uint32_t IDESC_T = idesc_f16(128, 64, false, false, false);
constexpr uint32_t IDESC_SO = idesc_f16(128, 192, false, false, true);

// fp16 values at or above this magnitude trigger a rescale of the lane (2^15 leaves room below
// the fp16 maximum 65504); a state lane below kSmall with sigma > 0 is scaled back up
constexpr float kRangeHi = 32768.f;
constexpr float kStateHi = 16384.f;
constexpr float kStateLo = 64.f;
constexpr int kSigmaMax = 100;

struct Params {
    const float* g;
    const float* beta;
    const float* A_log;
    const float* dt_bias;
    float lower_bound;
    float scale;
    const float* initial_state;
    const int32_t* cu_seqlens;
    __nv_bfloat16* out;
    float* final_state;
    int64_t seqlen;
    int64_t total_tokens;
    int H;
    int N;
    uint32_t flags;   // kFlagVZero, kFlagInitIdentity (the segment maps of one long sequence)
};

#ifdef KDA_PHASE_CLOCKS
__device__ unsigned long long g_pipe_phase_cycles[kPhases];
constexpr int kMaxCtaRecords = 1024;
// per CTA: global timer at entry and at exit (ns), chunks run, SM id, then its phase cycles
constexpr int kCtaRec = 4 + kPhases;
__device__ unsigned long long g_pipe_cta[kMaxCtaRecords][kCtaRec];
// thread `who` adds the cycles since its role's previous mark to slot i
#define PIPE_MARK(who, slot, i)                                            \
    do {                                                                   \
        if (threadIdx.x == (who)) {                                        \
            const long long now_ = clock64();                              \
            sPh[i] += (unsigned long long)(now_ - sPh[kPhases + (slot)]);  \
            sPh[kPhases + (slot)] = (unsigned long long)now_;              \
        }                                                                  \
    } while (0)
#else
#define PIPE_MARK(who, slot, i) do { } while (0)
#endif

// ---- small helpers ----
// Pulls the line holding `ptr` into L2 (no register result, never waited on).
__device__ __forceinline__ void prefetch_l2(const void* ptr) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}
// fp16 pair, saturating at +-65504 (never inf)
__device__ __forceinline__ uint32_t pack_f16s(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
// running max of |x| over fp16 pairs (sign bits of the result are meaningless)
__device__ __forceinline__ uint32_t hmax_abs(uint32_t m, uint32_t h) {
    uint32_t r;
    asm("max.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(r) : "r"(m), "r"(h));
    return r;
}
__device__ __forceinline__ float hmax_to_float(uint32_t m) {
    const __half2 h = *reinterpret_cast<const __half2*>(&m);
    return fmaxf(fabsf(__low2float(h)), fabsf(__high2float(h)));
}
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
__device__ __forceinline__ float fast_ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float fast_lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float fast_rcp(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// 2^e for an integer e in [-126, 127]
__device__ __forceinline__ float pow2i(int e) { return __int_as_float((127 + e) << 23); }
// floor(log2 |x|) for a normal nonzero x
__device__ __forceinline__ int ilog2f(float x) { return (int)((__float_as_uint(x) >> 23) & 0xFFu) - 127; }

// Byte offset of the 4-channel group starting at channel c0 (a multiple of 4) in row rowbase + i
// of a 128-byte-swizzled 16-bit tile with `rows` rows, where rowbase is a multiple of 8 (so the
// swizzle phase of the row is i): the same value as sw128_off(rowbase + i, c0, rows).
__device__ __forceinline__ uint32_t quad_off(uint32_t rows, uint32_t rowbase, int i, uint32_t c0) {
    return (c0 >> 6) * rows * 128u + (rowbase + (uint32_t)i) * 128u + (((((c0 & 63u) >> 3) ^ (uint32_t)i)) << 4) +
           ((c0 & 7u) << 1);
}

// Shared-memory stores the compiler may move later shared loads above: the operand tiles
// written in one phase are never read back in it (the phase ends with a fence and a barrier,
// which order them before every later use).
__device__ __forceinline__ void st_tile2(const unsigned char* base, uint32_t off, uint32_t a, uint32_t b) {
    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(smem_u32(base) + off), "r"(a), "r"(b));
}
__device__ __forceinline__ void st_tile4(const unsigned char* base, uint32_t off, uint32_t a, uint32_t b,
                                         uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(base) + off), "r"(a), "r"(b), "r"(c),
                 "r"(d));
}
__device__ __forceinline__ void st_tile_h(const unsigned char* base, uint32_t off, uint16_t a) {
    asm volatile("st.shared.b16 [%0], %1;" ::"r"(smem_u32(base) + off), "h"(a));
}
__device__ __forceinline__ void st_v4(unsigned char* base, uint32_t off, uint32_t a, uint32_t b,
                                      uint32_t c, uint32_t d) {
    *reinterpret_cast<uint4*>(base + off) = make_uint4(a, b, c, d);
}

__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Named barrier that also ORs a predicate over the participating threads (uniform result).
__device__ __forceinline__ bool named_bar_or(uint32_t id, uint32_t nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"(pred ? 1u : 0u), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0u;
}

// Every lane of the warp waits (bounded) for the phase, so each has acquired what the phase
// guards; the warp agrees on the outcome.  A timeout is recorded in the device error word.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar, parity));
    if (!ok && (threadIdx.x & 31) == 0) record_error(KDA_DEVERR_TIMEOUT);
    return ok;
}

// A monotonic sequence number in shared memory (a counter cannot skip a phase the way an mbarrier
// parity can): the writer publishes with a release store after a barrier over the producing threads,
// the reader waits for a value with acquire loads, at most limit_ns.
__device__ __forceinline__ void seq_publish(uint32_t* seq, uint32_t v) {
    asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(seq)), "r"(v) : "memory");
}
__device__ __forceinline__ bool seq_wait(const uint32_t* seq, uint32_t target, uint64_t limit_ns = 1000000000ull) {
    uint32_t v;
    asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(seq)) : "memory");
    if (v >= target) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        __nanosleep(100);
        asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(seq)) : "memory");
        if (v >= target) return true;
        if (global_ns() - t0 > limit_ns) return false;
    }
}

// ---- 16 x 16 fp16 block products of the triangular solve (mma.sync m16n8k16, fp32 accumulation) ----
// Operands come from shared memory through ldmatrix: lane l gives the address of row (l & 15),
// columns 8 (l >> 4) .. 8 (l >> 4) + 7 of the block.  Without .trans that yields the A fragment of
// a row-major block; with .trans the B fragment of a row-major [k][n] block.
__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm4t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}
// acc (+)= P Q for 16 x 16 blocks at ldmatrix row addresses pa (P) and qa (Q)
__device__ __forceinline__ void mm16h(float (&acc)[2][4], uint32_t pa, uint32_t qa) {
    uint32_t a[4], b[4];
    ldsm4(pa, a);
    ldsm4t(qa, b);
    const uint32_t b0[2] = {b[0], b[1]}, b1[2] = {b[2], b[3]};
    warpmma::mma_f16_16816(acc[0], a, b0);
    warpmma::mma_f16_16816(acc[1], a, b1);
}
// ldmatrix row address of a fp16 block at byte offset `off` (row pitch kHp halves)
__device__ __forceinline__ uint32_t lm_blk(const unsigned char* sm, uint32_t off) {
    const uint32_t lane = threadIdx.x & 31u;
    return smem_u32(sm) + off + (lane & 15u) * (uint32_t)kHp * 2u + (lane >> 4) * 16u;
}
// ldmatrix row address of block (I, J) of the 128-byte-swizzled fp16 T tile [64 r][64 i]
__device__ __forceinline__ uint32_t lm_t16(const unsigned char* sm, int I, int J) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t row = 16u * (uint32_t)I + (lane & 15u), chunk = 2u * (uint32_t)J + (lane >> 4);
    return smem_u32(sm) + T16 + row * 128u + ((chunk ^ (row & 7u)) << 4);
}
// sign * accumulator -> fp16 block at byte offset `off` (round to nearest, as an operand load would)
__device__ __forceinline__ void store16h(unsigned char* sm, uint32_t off, const float (&acc)[2][4], float sign) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
        const uint32_t col = (uint32_t)(8 * nh + 2 * t);
        *reinterpret_cast<uint32_t*>(sm + off + ((uint32_t)g * kHp + col) * 2u) =
            warpmma::pack_half2(sign * acc[nh][0], sign * acc[nh][1]);
        *reinterpret_cast<uint32_t*>(sm + off + ((uint32_t)(g + 8) * kHp + col) * 2u) =
            warpmma::pack_half2(sign * acc[nh][2], sign * acc[nh][3]);
    }
}
// index of A's block (I, J), J < I, among the six below the diagonal
__device__ __forceinline__ uint32_t al_off(int I, int J) {
    return SV_AL + (uint32_t)(I * (I - 1) / 2 + J) * kHBlk;
}

// ---- schedule ----
// Slot k of CTA b over G CTAs (snake order: even slots forward, odd slots backward).
__device__ __forceinline__ int unit_of(int k, int b, int G) {
    return (k & 1) ? (k + 1) * G - 1 - b : k * G + b;
}

struct Cursor {
    int k, h, n;
    int64_t bos, eos, t0;
    bool valid;
};

__device__ __forceinline__ void decode_unit(const Params& p, const int16_t* order, int u, int* n, int* h,
                                            int64_t* bos, int64_t* eos) {
    const int rank = u / p.H;
    *h = u - rank * p.H;
    *n = (p.N <= kSortLimit) ? order[rank] : rank;
    seq_range(p.cu_seqlens, *n, p.seqlen, p.total_tokens, bos, eos);
}

// The first chunk of the first non-empty unit at slot >= k0 (invalid if none).
__device__ __noinline__ Cursor unit_from(const Params& p, const int16_t* order, int b, int G, int units, int k0) {
    Cursor c;
    c.valid = false;
    for (int k = k0; (int64_t)k * G < units; ++k) {
        const int u = unit_of(k, b, G);
        if (u >= units) continue;
        decode_unit(p, order, u, &c.n, &c.h, &c.bos, &c.eos);
        if (c.eos > c.bos) {
            c.k = k;
            c.t0 = c.bos;
            c.valid = true;
            return c;
        }
    }
    return c;
}

__device__ __forceinline__ Cursor next_chunk(const Params& p, const int16_t* order, int b, int G, int units,
                                             Cursor c) {
    if (c.t0 + kChunk < c.eos) {
        c.t0 += kChunk;
        return c;
    }
    return unit_from(p, order, b, G, units, c.k + 1);
}

__device__ __forceinline__ void issue_chunk_loads(unsigned char* sm, uint64_t* bar, const CUtensorMap* tq,
                                                  const CUtensorMap* tk, const CUtensorMap* tv, int h,
                                                  int64_t t0) {
    mbar_arrive_expect_tx(bar, IN_BYTES);
    const int x = h * kHeadDim, y = (int)t0;
    tma_load_2d(sm + IN_Q, tq, x, y, bar);
    tma_load_2d(sm + IN_K, tk, x, y, bar);
    tma_load_2d(sm + IN_V, tv, x, y, bar);
}

constexpr float kLog2e = 1.4426950408889634f;

// ---- element warps: gate ----
// a[i][e] = a_t for token r0 + i, channel c0 + e: a = max(2^(-e^A_log * log2(1 + 2^x2)), e^lb)
// with x2 = (g + dt_bias) log2 e, i.e. e^(-e^A_log softplus(g + dt_bias)) clamped at e^lb.
// Rows past the chunk's valid length get a = 1.
// gs: the chunk's raw gate input, fp32 [64 tokens][128 channels] in shared memory (a TMA box)
__device__ __forceinline__ void gate_tokens(const Params& p, int h, const float* gs, int L, int c0, int r0,
                                            float (&a)[8][4]) {
    const float nexpA = -expf(p.A_log[h]);
    const float alb = fast_ex2(p.lower_bound * kLog2e);
    const float4 db = *reinterpret_cast<const float4*>(p.dt_bias + h * kHeadDim + c0);
    const float2 db01 = make_float2(db.x * kLog2e, db.y * kLog2e), db23 = make_float2(db.z * kLog2e, db.w * kLog2e);
    const float2 l2e = make_float2(kLog2e, kLog2e);
    float4 gv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) gv[i] = *reinterpret_cast<const float4*>(gs + (r0 + i) * kHeadDim + c0);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float2 x01 = __ffma2_rn(make_float2(gv[i].x, gv[i].y), l2e, db01);
        const float2 x23 = __ffma2_rn(make_float2(gv[i].z, gv[i].w), l2e, db23);
        const float2 s01 = __fadd2_rn(make_float2(1.f, 1.f), make_float2(fast_ex2(x01.x), fast_ex2(x01.y)));
        const float2 s23 = __fadd2_rn(make_float2(1.f, 1.f), make_float2(fast_ex2(x23.x), fast_ex2(x23.y)));
        const float2 l01 = __fmul2_rn(make_float2(nexpA, nexpA), make_float2(fast_lg2(s01.x), fast_lg2(s01.y)));
        const float2 l23 = __fmul2_rn(make_float2(nexpA, nexpA), make_float2(fast_lg2(s23.x), fast_lg2(s23.y)));
        const bool live = r0 + i < L;
        a[i][0] = live ? fmaxf(fast_ex2(l01.x), alb) : 1.f;
        a[i][1] = live ? fmaxf(fast_ex2(l01.y), alb) : 1.f;
        a[i][2] = live ? fmaxf(fast_ex2(l23.x), alb) : 1.f;
        a[i][3] = live ? fmaxf(fast_ex2(l23.y), alb) : 1.f;
    }
}

// Decay factors of an element thread's 8 tokens (4 channels): E[i] = product of a over the
// tokens after i up to the block end, and the initial value of the running product
// R = a-product from the block start (R_i = R0 * a_0 * ... * a_i).  po is the product over the
// other 8-token half of the block (before this half for the second half, after it for the first).
__device__ __forceinline__ void decay_suffix(const float (&a)[8][4], const float (&po)[4], bool second_half,
                                             float2 (&E)[8][2], float2 (&R0)[2]) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        E[7][e] = second_half ? make_float2(1.f, 1.f) : make_float2(po[2 * e], po[2 * e + 1]);
#pragma unroll
        for (int i = 6; i >= 0; --i) E[i][e] = __fmul2_rn(E[i + 1][e], make_float2(a[i + 1][2 * e], a[i + 1][2 * e + 1]));
        R0[e] = second_half ? make_float2(po[2 * e], po[2 * e + 1]) : make_float2(1.f, 1.f);
    }
}
__device__ __forceinline__ uint32_t pack_bf16v(float2 v) { return pack_bf16(v.x, v.y); }
__device__ __forceinline__ uint32_t pack_f16v(float2 v) { return pack_f16s(v.x, v.y); }

// ---- chain warps: rare range repairs (out of line: they cost no instruction-cache space on
// the common path).  lane_base = TMEM address of the warp's lane quarter.

// Every state lane value (TM_S) and O^T (TM_O) times 2^-d.
__device__ __noinline__ void chain_rescale_state(uint32_t lane_base, int d) {
    const float f = pow2i(-d);
#pragma unroll 1
    for (int cb = 0; cb < 6; ++cb) {
        const uint32_t col = cb < 4 ? TM_S + 32u * cb : TM_O + 32u * (cb - 4);
        uint32_t s[32];
        tmem_ld32(lane_base + col, s);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) s[j] = __float_as_uint(f * __uint_as_float(s[j]));
        tmem_st32(lane_base + col, s);
    }
    tmem_wait_st();
}

// The TMEM loads and stores below are warp-collective (.sync.aligned): the whole warp calls these
// repairs when any of its lanes needs one, and lanes that do not need it use a shift of 0.

// A state lane left [kStateLo, kStateHi) (or saturated): choose the shift delta that brings its
// fp32 maximum to [2^12, 2^13) (never below sigma = 0, never above kSigmaMax) and write the fp16
// copy again.  Returns delta (0 where need is false); the caller adds it to sigma.
__device__ __noinline__ int chain_state_reconvert(uint32_t lane_base, int sigma, bool need) {
    float mx = 0.f;
#pragma unroll 1
    for (int cb = 0; cb < 4; ++cb) {
        uint32_t s[32];
        tmem_ld32(lane_base + TM_S + 32u * cb, s);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) mx = fmaxf(mx, fabsf(__uint_as_float(s[j])));
    }
    int delta = mx > 0.f ? ilog2f(mx) - 12 : -sigma;
    if (delta < -sigma) delta = -sigma;
    if (sigma + delta > kSigmaMax) delta = kSigmaMax - sigma;
    if (!need) delta = 0;
    // the fp16 copy and the fp32 state itself, both times 2^-delta
    const float f = pow2i(-delta);
#pragma unroll 1
    for (int cb = 0; cb < 4; ++cb) {
        uint32_t s[32];
        tmem_ld32(lane_base + TM_S + 32u * cb, s);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) s[j] = __float_as_uint(f * __uint_as_float(s[j]));
        uint32_t h16[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) h16[j] = pack_f16s(__uint_as_float(s[2 * j]), __uint_as_float(s[2 * j + 1]));
        tmem_st16(lane_base + TM_H + 16u * cb, h16);
        tmem_st32(lane_base + TM_S + 32u * cb, s);
    }
    tmem_wait_st();
    return delta;
}

// Y (with_beta_v: TM_Y plus 2^-sigma beta v of this lane's value column v) or U (TM_Y as is)
// saturated its fp16 copy in a lane where need is true: shift that lane down so that its fp32
// maximum lands in [2^12, 2^13), convert again into the fp16 columns at TM_H + col, and rescale
// its state and O^T to match.  Returns the shift d (0 where need is false or the lane cannot move
// further); the caller adds it to sigma.
__device__ __noinline__ int chain_vals_reconvert(uint32_t lane_base, uint32_t col, const unsigned char* sm,
                                                 int v, uint32_t slot, bool with_beta_v, int sigma, bool need) {
    const float fs = pow2i(-sigma);
    const float* be = reinterpret_cast<const float*>(sm + S_BETA) + slot * 64u;
    float mx = 0.f;
    int d = 0;
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        const float f = pow2i(-d);
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
            uint32_t t[32];
            tmem_ld32(lane_base + TM_Y + 32u * half, t);
            tmem_wait_ld();
            float x[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) x[j] = __uint_as_float(t[j]);
            if (with_beta_v) {
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    const uint32_t c8 = (uint32_t)(4 * half + ch);
                    const uint4 w = *reinterpret_cast<const uint4*>(sm + VT + (uint32_t)v * 128u +
                                                                    ((c8 ^ ((uint32_t)v & 7u)) << 4));
                    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 vv = bf16x2_to_float2(ww[e]);
                        x[8 * ch + 2 * e] = fmaf(fs * be[8 * c8 + 2 * e], vv.x, x[8 * ch + 2 * e]);
                        x[8 * ch + 2 * e + 1] = fmaf(fs * be[8 * c8 + 2 * e + 1], vv.y, x[8 * ch + 2 * e + 1]);
                    }
                }
            }
            if (pass == 0) {
#pragma unroll
                for (int j = 0; j < 32; ++j) mx = fmaxf(mx, fabsf(x[j]));
            } else {
                uint32_t h16[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) h16[j] = pack_f16s(f * x[2 * j], f * x[2 * j + 1]);
                tmem_st16(lane_base + col + 16u * half, h16);
            }
        }
        if (pass == 0) {
            d = ilog2f(mx) - 12;
            if (sigma + d > kSigmaMax) d = kSigmaMax - sigma;
            if (!need || d < 0) d = 0;
        }
    }
    tmem_wait_st();
    chain_rescale_state(lane_base, d);
    return d;
}

// ---- scalar-gate variant: gate and loads ----
// One warp: lane l handles tokens 2l and 2l + 1 (gv = their raw gate inputs).  s_gam(sl) gets the
// inclusive in-chunk sum Gamma of log2 a (flat past the valid length), s_ge(sl) 2^Gamma and
// s_kf(sl) 2^(Gamma_63 - Gamma).
__device__ __forceinline__ void gate_scan_scalar(unsigned char* sm, const Params& p, int h, int L, float2 gv,
                                                 uint32_t sl) {
    const int lane = threadIdx.x & 31;
    const float nexpA = -expf(p.A_log[h]);
    const float lb2 = p.lower_bound * kLog2e;
    const float db2 = p.dt_bias[h] * kLog2e;
    const int r0 = 2 * lane;
    float2 l;
    {
        const float x0 = fmaf(gv.x, kLog2e, db2), x1 = fmaf(gv.y, kLog2e, db2);
        l.x = fmaxf(nexpA * fast_lg2(1.f + fast_ex2(x0)), lb2);
        l.y = fmaxf(nexpA * fast_lg2(1.f + fast_ex2(x1)), lb2);
    }
    if (r0 >= L) l.x = 0.f;
    if (r0 + 1 >= L) l.y = 0.f;
    const float pair = l.x + l.y;
    float incl = pair;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float t = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += t;
    }
    const float g0 = incl - pair + l.x, g1 = incl;
    const float glast = __shfl_sync(0xffffffffu, incl, 31);
    *reinterpret_cast<float2*>(reinterpret_cast<float*>(sm + s_gam(sl)) + r0) = make_float2(g0, g1);
    *reinterpret_cast<float2*>(reinterpret_cast<float*>(sm + s_ge(sl)) + r0) = make_float2(fast_ex2(g0), fast_ex2(g1));
    *reinterpret_cast<float2*>(reinterpret_cast<float*>(sm + s_kf(sl)) + r0) =
        make_float2(fast_ex2(glast - g0), fast_ex2(glast - g1));
}

__device__ __forceinline__ void issue_chunk_loads_s(unsigned char* sm, uint64_t* bar, const CUtensorMap* tq,
                                                    const CUtensorMap* tk, const CUtensorMap* tv, int h,
                                                    int64_t t0) {
    mbar_arrive_expect_tx(bar, IN_BYTES);
    const int x = h * kHeadDim, y = (int)t0;
#pragma unroll
    for (int cb = 0; cb < 2; ++cb) {
        tma_load_2d(sm + IN_Q + (uint32_t)cb * 16384u, tk, x + 64 * cb, y, bar);
        tma_load_2d(sm + IN_Q + (uint32_t)cb * 16384u + 8192u, tq, x + 64 * cb, y, bar);
        tma_load_2d(sm + IN_V + (uint32_t)cb * 8192u, tv, x + 64 * cb, y, bar);
    }
}

// ---- the kernel ----
template <bool kScalar>
__global__ void __launch_bounds__(kThreads, 1)
kda_pipe_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                const Params p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
#ifdef KDA_PHASE_CLOCKS
    const unsigned long long t_entry = global_ns();
    unsigned long long n_chunks = 0;
#endif
    const int G = gridDim.x, b = blockIdx.x;
    const int H = p.H;
    const int units = p.N * H;

    int16_t* sOrder = reinterpret_cast<int16_t*>(sm + S_ORDER);
    int32_t* sMeta = reinterpret_cast<int32_t*>(sm + S_META);
    uint64_t* bar_in = reinterpret_cast<uint64_t*>(sm + S_BARS);   // inputs landed (TMA)
    uint64_t* bar_ap = bar_in + 1;       // A/P MMA done
    uint64_t* bar_formed = bar_in + 2;   // chunk's B1, Khat, V^T, beta, gamma_C, metadata written
    uint64_t* bar_t = bar_in + 3;        // chunk's P^T and T written
    uint64_t* bar_y = bar_in + 4;        // [O | Y] MMA done
    uint64_t* bar_u = bar_in + 5;        // U MMA done
    uint64_t* bar_s = bar_in + 6;        // [S | O] MMA done (chunk's shared operands free again)
    uint64_t* bar_apready = bar_in + 7;  // chunk's A/P operand tiles written (the chain issues the MMA)
    uint64_t* bar_ro = bar_in + 8;       // chunk's A/P product read out of TMEM (the accumulator is free)
    uint64_t* bar_g = bar_in + 9;        // channel gate: chunk's raw gate input landed (TMA, in the A/P tiles)
    uint64_t* bar_vt = bar_in + 10;      // channel gate: chunk's V^T and P diagonal formed (aux warps)
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + S_TMEM);
    volatile uint32_t* sAbort = sTmem + 1;
    uint32_t* sRdSeq = sTmem + 2;   // chunks whose beta, P diagonal (and scalar Gamma) the element warps published
#ifdef KDA_PHASE_CLOCKS
    volatile unsigned long long* sPh = reinterpret_cast<volatile unsigned long long*>(sm + S_PH);
#endif

    // ---- set-up ----
    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) mbar_init(bar_in + i, 1);
        mbar_init_fence();
        *sAbort = 0u;
        *sRdSeq = 0u;
    }
    if (warp == 0) {
        tmem_alloc(sTmem, TM_COLS);
        tmem_relinquish();
    }
    if (p.N <= kSortLimit) {
        for (int n = tid; n < p.N; n += kThreads) {
            int64_t bn, en;
            seq_range(p.cu_seqlens, n, p.seqlen, p.total_tokens, &bn, &en);
            const int64_t ln = en - bn;
            int rank = 0;
            for (int m = 0; m < p.N; ++m) {
                int64_t bm, em;
                seq_range(p.cu_seqlens, m, p.seqlen, p.total_tokens, &bm, &em);
                const int64_t lm = em - bm;
                rank += (lm > ln) || (lm == ln && m < n);
            }
            sOrder[rank] = (int16_t)n;
        }
    }
    // T16's blocks above the diagonal are never written by the solve: zero them once
    for (int e = tid; e < 8192 / 16; e += kThreads) st_v4(sm, T16 + (uint32_t)e * 16u, 0u, 0u, 0u, 0u);
#ifdef KDA_PHASE_CLOCKS
    if (tid == 0)
        for (int i = 0; i < kPhases + 3; ++i) sPh[i] = (i < kPhases) ? 0ull : (unsigned long long)clock64();
#endif
    __syncthreads();
    // empty units: final state = initial state (the chain never sees them)
    if (p.final_state) {
        for (int k = 0; (int64_t)k * G < units; ++k) {
            const int u = unit_of(k, b, G);
            if (u >= units) continue;
            int n, h;
            int64_t bos, eos;
            decode_unit(p, sOrder, u, &n, &h, &bos, &eos);
            if (eos > bos) continue;
            const int64_t off = ((int64_t)n * H + h) * kHeadDim * kHeadDim;
            const bool ident = (p.flags & kFlagInitIdentity) != 0;
            for (int e = tid; e < kHeadDim * kHeadDim / 4; e += kThreads) {
                const int row = (4 * e) / kHeadDim, col = (4 * e) % kHeadDim;
                float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
                if (p.initial_state) {
                    s = reinterpret_cast<const float4*>(p.initial_state + off)[e];
                } else if (ident) {
                    s = make_float4(row == col ? 1.f : 0.f, row == col + 1 ? 1.f : 0.f, row == col + 2 ? 1.f : 0.f,
                                    row == col + 3 ? 1.f : 0.f);
                }
                reinterpret_cast<float4*>(p.final_state + off)[e] = s;
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *sTmem;

    if (warp < kAuxWarp0) {
        // =============================== chain warps ===============================
        const int v = tid;                       // value column = TMEM lane
        const uint32_t lane_base = tbase + ((uint32_t)(warp * 32) << 16);
        int sigma = 0;                           // this lane's state is stored times 2^-sigma
        uint32_t cc = 0;                         // chunks started
        bool have_prev = false;
        int prev_h = 0, prev_n = 0, prev_L = 0, prev_last = 0;
        int64_t prev_t0 = 0;
        uint32_t issued_y = 0, issued_u = 0, issued_s = 0, done_s = 0, issued_ap = 0;   // thread 0's MMA commits
        bool in_pending = false;   // thread 0: input loads issued (drained on abort)
        uint32_t in_parity = 0;
        bool aborted = false;

        // O^T (TMEM) of the previous chunk -> out, and its final state if it ended a unit.  Lane v
        // holds column v of every output row; lanes v and v + 1 (v even) trade one value per pair of
        // rows, so the even lane writes columns (v, v + 1) of even rows and the odd lane those of odd
        // rows, as 4-byte stores (a warp writes 64 contiguous bytes per row).
        auto retire_prev = [&]() {
            const float sc = p.scale * pow2i(sigma);
            const bool odd = (v & 1) != 0;
            const int64_t row_stride = (int64_t)H * kHeadDim;
            __nv_bfloat16* base = p.out + (prev_t0 * H + prev_h) * kHeadDim + (v & ~1) + (odd ? row_stride : 0);
#pragma unroll 1
            for (int cb = 0; cb < (p.out ? 2 : 0); ++cb) {   // no output: a segment-map pass
                uint32_t o[32];
                tmem_ld32(lane_base + TM_O + 32u * cb, o);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const float e0 = sc * __uint_as_float(o[j]), e1 = sc * __uint_as_float(o[j + 1]);
                    // even lane sends its odd-row value, odd lane its even-row value
                    const float got = __shfl_xor_sync(0xffffffffu, odd ? e0 : e1, 1);
                    const uint32_t w = odd ? pack_bf16(got, e1) : pack_bf16(e0, got);
                    const int r = 32 * cb + j + (odd ? 1 : 0);
                    if (r < prev_L)
                        *reinterpret_cast<uint32_t*>(base + (int64_t)(32 * cb + j) * row_stride) = w;
                }
            }
            if (prev_last && p.final_state) {
                const float f = pow2i(sigma);
                float* fs = p.final_state + ((int64_t)prev_n * H + prev_h) * kHeadDim * kHeadDim + v;
#pragma unroll 1
                for (int cb = 0; cb < 4; ++cb) {
                    uint32_t s[32];
                    tmem_ld32(lane_base + TM_S + 32u * cb, s);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) fs[(32 * cb + j) * kHeadDim] = f * __uint_as_float(s[j]);
                }
            }
        };
        // fp32 values -> fp16 pairs at TMEM column `col` (count/2 columns) times 2^-d; returns max |fp16|
        auto to_f16_tmem = [&](float (&x)[64], uint32_t col, float f) -> float {
            uint32_t m = 0u;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t h16[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    h16[j] = pack_f16s(f * x[32 * half + 2 * j], f * x[32 * half + 2 * j + 1]);
                    m = hmax_abs(m, h16[j]);
                }
                tmem_st16(lane_base + col + 16u * half, h16);
            }
            return hmax_to_float(m);
        };

        // The front end's A/P MMA of chunk cc (thread 0), as soon as its operand tiles are written
        // and the previous chunk's product has been read out of TMEM.  It does not depend on the
        // state, so it goes before the previous chunk's output: the front end waits for it twice
        // (its read-out, and the next chunk's operand tiles, which overwrite its inputs).
        auto issue_ap = [&]() {
            if (!mbar_wait_bounded(bar_apready, cc & 1u) ||
                (cc > 0 && !mbar_wait_bounded(bar_ro, (cc - 1) & 1u))) {
                record_error(KDA_DEVERR_TIMEOUT);
                *sAbort = 1u;
                return;
            }
            fence_after_sync();
            if constexpr (kScalar) {
                // [K ; Q] K^T straight from the swizzled input blocks (the decay is applied at
                // read-out)
                const uint32_t a0 = smem_u32(sm + IN_Q);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_f16(tbase + TM_AP, desc_kmajor(a0, 128, ks), desc_kmajor(a0, 128, ks), IDESC_AP_S,
                            ks > 0 ? 1u : 0u);
            } else {
                const uint32_t a0 = smem_u32(sm + AP_A), b0 = smem_u32(sm + AP_B);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_f16(tbase + TM_AP, desc_kmajor(a0, 128, ks), desc_kmajor(b0, 160, ks), IDESC_AP,
                            ks > 0 ? 1u : 0u);
            }
            mma_commit(bar_ap);
            ++issued_ap;
        };

        // whether another chunk follows (the front end marks a CTA's last chunk in its metadata)
        bool more = unit_from(p, sOrder, b, G, units, 0).valid;
        while (true) {
            bool bad = false;
            if (tid == 0 && more) issue_ap();
            PIPE_MARK(0, 1, 11);
            // the previous chunk's output (and final state), once its [S | O] MMA is done
            if (have_prev) {
                bad |= !warp_wait(bar_s, (cc - 1) & 1u);
                if (tid == 0 && !bad) done_s = issued_s;
                fence_after_sync();
                PIPE_MARK(0, 1, 9);
                if (!bad) retire_prev();
            }
            PIPE_MARK(0, 1, 10);
            if (!more) break;
            PIPE_MARK(0, 1, 12);
            bad |= !warp_wait(bar_formed, cc & 1u);
            const int32_t* meta = sMeta + (cc & 1u) * 16u;
            const int m_h = meta[1], m_n = meta[2], m_t0 = meta[3], m_L = meta[4], m_first = meta[5],
                      m_last = meta[6];
            more = meta[7] != 0;
            // channel gate: the aux warps' V^T (they read this chunk's inputs for it and for P's diagonal)
            if constexpr (!kScalar) bad |= !warp_wait(bar_vt, cc & 1u);
            // the next chunk's q, k, v: the element (and aux) warps are done with this chunk's input
            // tiles (and, for the scalar gate, the A/P MMA that reads them has completed)
            if (tid == 0 && more && !bad) {
                const bool ok = !kScalar || mbar_wait_bounded(bar_ap, cc & 1u);
                if (ok) {
                    if constexpr (kScalar)
                        issue_chunk_loads_s(sm, bar_in, &tm_q, &tm_k, &tm_v, meta[8], meta[9]);
                    else
                        issue_chunk_loads(sm, bar_in, &tm_q, &tm_k, &tm_v, meta[8], meta[9]);
                    in_pending = true;
                    in_parity = (cc + 1u) & 1u;
                } else {
                    record_error(KDA_DEVERR_TIMEOUT);
                    *sAbort = 1u;
                }
            }
            if (named_bar_or(BAR_CHAIN, 128, bad || *sAbort != 0u)) {
                aborted = true;
                break;
            }
            PIPE_MARK(0, 1, 13);
            if (m_first) {
                // the unit's initial state (or zeros) into TMEM
                sigma = 0;
                const float* is = p.initial_state
                    ? p.initial_state + ((int64_t)m_n * H + m_h) * kHeadDim * kHeadDim + v : nullptr;
                const bool ident = (p.flags & kFlagInitIdentity) != 0;
#pragma unroll 1
                for (int cb = 0; cb < 4; ++cb) {
                    uint32_t s[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        s[j] = is ? __float_as_uint(is[(32 * cb + j) * kHeadDim])
                                  : ((ident && 32 * cb + j == v) ? 0x3f800000u : 0u);
                    tmem_st32(lane_base + TM_S + 32u * cb, s);
                }
                tmem_wait_st();
            }
            // ---- S^T -> fp16 A operand (scale kept unless the lane leaves its range) ----
            int delta = 0;
            {
                uint32_t m = 0u;
#pragma unroll 1
                for (int cb = 0; cb < 4; ++cb) {
                    uint32_t s[32];
                    tmem_ld32(lane_base + TM_S + 32u * cb, s);
                    tmem_wait_ld();
                    uint32_t h16[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        h16[j] = pack_f16s(__uint_as_float(s[2 * j]), __uint_as_float(s[2 * j + 1]));
                        m = hmax_abs(m, h16[j]);
                    }
                    tmem_st16(lane_base + TM_H + 16u * cb, h16);
                }
                const float mh = hmax_to_float(m);
                const bool need = mh >= kStateHi || (mh < kStateLo && sigma > 0);
                if (__any_sync(0xffffffffu, need)) {   // rare; the whole warp takes part
                    tmem_wait_st();
                    delta = chain_state_reconvert(lane_base, sigma, need);
                    sigma += delta;
                }
            }
            tmem_wait_st();
            fence_before_sync();
            named_bar_sync(BAR_CHAIN, 128);
            // [O | Y]^T = S^T [gamma Q ; -beta gamma K]^T
            if (tid == 0) {
                fence_after_sync();
                const uint32_t b1 = smem_u32(sm + B1);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_f16_ts(tbase + TM_O, tbase + TM_H + (uint32_t)ks * 8u, desc_kmajor(b1, 128, ks), IDESC_OY,
                               ks > 0 ? 1u : 0u);
                mma_commit(bar_y);
                ++issued_y;
            }
            // S^T <- S^T Diag(gamma_C) (the MMA above reads only the fp16 copy; a rescale of the lane
            // was applied to the fp32 state already)
            {
                const float* gc = reinterpret_cast<const float*>(sm + S_GC) + (cc & 1u) * kHeadDim;
#pragma unroll 1
                for (int cb = 0; cb < 4; ++cb) {
                    uint32_t s[32];
                    tmem_ld32(lane_base + TM_S + 32u * cb, s);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        const float4 g4 = *reinterpret_cast<const float4*>(gc + 32 * cb + j);
                        const float2 a = __fmul2_rn(make_float2(__uint_as_float(s[j]), __uint_as_float(s[j + 1])),
                                                    make_float2(g4.x, g4.y));
                        const float2 c = __fmul2_rn(make_float2(__uint_as_float(s[j + 2]), __uint_as_float(s[j + 3])),
                                                    make_float2(g4.z, g4.w));
                        s[j] = __float_as_uint(a.x);
                        s[j + 1] = __float_as_uint(a.y);
                        s[j + 2] = __float_as_uint(c.x);
                        s[j + 3] = __float_as_uint(c.y);
                    }
                    tmem_st32(lane_base + TM_S + 32u * cb, s);
                }
                tmem_wait_st();
            }
            PIPE_MARK(0, 1, 14);
            // ---- Y^T += 2^-sigma (beta V)^T -> fp16 ----
            bad |= !warp_wait(bar_y, cc & 1u);
            fence_after_sync();
            {
                float y[64];
                {
                    uint32_t t0r[32], t1r[32];
                    tmem_ld32(lane_base + TM_Y, t0r);
                    tmem_ld32(lane_base + TM_Y + 32u, t1r);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        y[j] = __uint_as_float(t0r[j]);
                        y[32 + j] = __uint_as_float(t1r[j]);
                    }
                }
                const float fs = pow2i(-sigma);
                const float2 fs2 = make_float2(fs, fs);
                const float* be = reinterpret_cast<const float*>(sm + S_BETA) + (cc & 1u) * 64u;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const uint4 w = *reinterpret_cast<const uint4*>(sm + VT + (uint32_t)v * 128u +
                                                                    (((uint32_t)ch ^ ((uint32_t)v & 7u)) << 4));
                    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
                    const float4 b0 = *reinterpret_cast<const float4*>(be + 8 * ch);
                    const float4 b1v = *reinterpret_cast<const float4*>(be + 8 * ch + 4);
                    const float2 bb[4] = {make_float2(b0.x, b0.y), make_float2(b0.z, b0.w), make_float2(b1v.x, b1v.y),
                                          make_float2(b1v.z, b1v.w)};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 yy = __ffma2_rn(__fmul2_rn(fs2, bb[e]), bf16x2_to_float2(ww[e]),
                                                     make_float2(y[8 * ch + 2 * e], y[8 * ch + 2 * e + 1]));
                        y[8 * ch + 2 * e] = yy.x;
                        y[8 * ch + 2 * e + 1] = yy.y;
                    }
                }
                const bool need = to_f16_tmem(y, TM_H, 1.f) >= kRangeHi;
                if (__any_sync(0xffffffffu, need)) {   // rare; the whole warp takes part
                    tmem_wait_st();
                    sigma += chain_vals_reconvert(lane_base, TM_H, sm, v, cc & 1u, true, sigma, need);
                }
            }
            tmem_wait_st();
            fence_before_sync();
            if (named_bar_or(BAR_CHAIN, 128, bad || *sAbort != 0u)) {
                aborted = true;
                break;
            }
            PIPE_MARK(0, 1, 15);
            // U^T = Y^T T^T, once the front end has T
            if (tid == 0) {
                if (mbar_wait_bounded(bar_t, cc & 1u)) {
                    fence_after_sync();
                    const uint32_t t16 = smem_u32(sm + T16);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_f16_ts(tbase + TM_Y, tbase + TM_H + (uint32_t)ks * 8u, desc_kmajor(t16, 64, ks), IDESC_T,
                                   ks > 0 ? 1u : 0u);
                    mma_commit(bar_u);
                    ++issued_u;
                } else {
                    record_error(KDA_DEVERR_TIMEOUT);
                    *sAbort = 1u;
                }
            }
            bad |= !warp_wait(bar_u, cc & 1u);
            fence_after_sync();
            PIPE_MARK(0, 1, 16);
            // ---- U^T -> fp16 ----
            {
                float u[64];
                {
                    uint32_t t0r[32], t1r[32];
                    tmem_ld32(lane_base + TM_Y, t0r);
                    tmem_ld32(lane_base + TM_Y + 32u, t1r);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        u[j] = __uint_as_float(t0r[j]);
                        u[32 + j] = __uint_as_float(t1r[j]);
                    }
                }
                const bool need = to_f16_tmem(u, TM_H + 32u, 1.f) >= kRangeHi;
                if (__any_sync(0xffffffffu, need)) {   // rare; the whole warp takes part
                    tmem_wait_st();
                    sigma += chain_vals_reconvert(lane_base, TM_H + 32u, sm, v, cc & 1u, false, sigma, need);
                }
            }
            tmem_wait_st();
            fence_before_sync();
            if (named_bar_or(BAR_CHAIN, 128, bad || *sAbort != 0u)) {
                aborted = true;
                break;
            }
            // [S | O]^T += U^T [Khat | P^T]
            if (tid == 0) {
                fence_after_sync();
                const uint32_t b2 = smem_u32(sm + B2);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_f16_ts(tbase + TM_S, tbase + TM_H + 32u + (uint32_t)ks * 8u, desc_mnmajor(b2, 64, ks),
                               IDESC_SO, 1u);
                mma_commit(bar_s);
                ++issued_s;
            }
            PIPE_MARK(0, 1, 17);
            have_prev = true;
#ifdef KDA_PHASE_CLOCKS
            ++n_chunks;
#endif
            prev_h = m_h;
            prev_n = m_n;
            prev_t0 = m_t0;
            prev_L = m_L;
            prev_last = m_last;
            ++cc;
        }
        // wind-down: no MMA of this thread may still run when TMEM is released
        if (tid == 0 && aborted) {
            if (issued_y > 0) mbar_wait_bounded(bar_y, (issued_y - 1) & 1u);
            if (issued_u > 0) mbar_wait_bounded(bar_u, (issued_u - 1) & 1u);
            if (issued_s > done_s) mbar_wait_bounded(bar_s, (issued_s - 1) & 1u);
            if (issued_ap > 0) mbar_wait_bounded(bar_ap, (issued_ap - 1) & 1u);
            if (in_pending) mbar_wait_bounded(bar_in, in_parity);
        }
        if (aborted && tid == 0) *sAbort = 1u;
    } else {
        // =============================== front end ===============================
        // Element warps 8-15 build chunk n (gate, decay factors, the A/P operand tiles, the chain's
        // operand tiles) while aux warps 4-7 read out the A/P product of chunk n - 1 and solve
        // T = (I + A)^-1 for it (and, for the channel gate, form V^T and P's exact diagonal).  The
        // two groups share no barrier: they meet through mbarriers (A/P operands ready, A/P product
        // done, read-out done, the chain's [S | O] MMA done) and a published sequence number, so the
        // aux warps take a chunk as soon as its product lands.
        const bool is_aux = warp < kElemWarp0;
        const int at = tid - 128;           // aux thread (warps 4-7)
        const int et = tid - 256;           // element thread (warps 8-15)
        const int ew = et >> 5;
        const int eI = ew >> 1, ehf = ew & 1;
        const int c0 = 64 * ehf + 4 * (lane & 15);
        const int r0 = 16 * eI + 8 * (lane >> 4);
        const int quarter = warp & 3;       // TMEM lane quarter of this warp
        const bool loader = tid == 128;     // TMA loads (aux warp 4: it has idle time, the element warps have none)
        const bool elead = tid == 256;      // the element warps' barrier arrivals
        bool tma_pending = false;
        uint32_t tma_parity = 0;
        bool aborted = false;
        uint32_t range_bad = 0u;
        auto chunk_len = [](const Cursor& c) { return (int)(c.eos - c.t0 < kChunk ? c.eos - c.t0 : kChunk); };

        // chunk c's q, k, v into the input tiles
        auto load_inputs = [&](const Cursor& c) {
            if constexpr (kScalar)
                issue_chunk_loads_s(sm, bar_in, &tm_q, &tm_k, &tm_v, c.h, c.t0);
            else
                issue_chunk_loads(sm, bar_in, &tm_q, &tm_k, &tm_v, c.h, c.t0);
        };

        // channel gate: chunk c's raw gate input into the A/P operand region (free between a chunk's
        // A/P MMA and the next chunk's operand tiles); the element warps read it for the gate
        bool g_pending = false;
        uint32_t g_parity = 0;
        auto load_gate_input = [&](const Cursor& c, uint32_t parity) {
            mbar_arrive_expect_tx(bar_g, 32768u);
            tma_load_2d(sm + AP_A, &tm_g, c.h * kHeadDim, (int)c.t0, bar_g);
            g_pending = true;
            g_parity = parity;
        };

        Cursor cur = unit_from(p, sOrder, b, G, units, 0);
        uint32_t ci = 0;
        if (loader && cur.valid) {
            load_inputs(cur);
            tma_pending = true;
            tma_parity = 0;
            if constexpr (!kScalar) load_gate_input(cur, 0);
        }
        if (!is_aux) {
            // ======================= element warps =======================
            float a[8][4];
            float beta_reg = 0.f;   // element threads 0-63: beta of their token of the next chunk
            float2 g_reg = make_float2(0.f, 0.f);   // scalar gate, warp 8: g of tokens 2 lane, 2 lane + 1
            // the scalar gate's inputs of chunk c (rows past its length read as 0)
            auto load_g_scalar = [&](const Cursor& c) {
                const int Lc = chunk_len(c);
                g_reg.x = 2 * lane < Lc ? p.g[(c.t0 + 2 * lane) * H + c.h] : 0.f;
                g_reg.y = 2 * lane + 1 < Lc ? p.g[(c.t0 + 2 * lane + 1) * H + c.h] : 0.f;
            };
            // beta of chunk c: unconditional, row clamped, so that nothing consumes the load before
            // the next chunk's first phase (where rows past the length are masked)
            auto load_beta = [&](const Cursor& c) {
                if (et < kChunk) {
                    const int Lc = chunk_len(c);
                    beta_reg = p.beta[(c.t0 + (et < Lc ? et : Lc - 1)) * H + c.h];
                }
            };
            if (cur.valid) {
                load_beta(cur);
                if constexpr (kScalar) {
                    if (warp == kElemWarp0) load_g_scalar(cur);
                } else {
                    if (!warp_wait(bar_g, 0u)) *sAbort = 1u;
                    gate_tokens(p, cur.h, reinterpret_cast<const float*>(sm + AP_A), chunk_len(cur), c0, r0, a);
                }
            }
            while (cur.valid) {
                const Cursor nxt = next_chunk(p, sOrder, b, G, units, cur);
                const int h = cur.h;
                const int L = chunk_len(cur);
                const uint32_t sl = ci & 1u;
                bool bad = false;
                // scalar gate: the next chunk's gate input into L2 (the channel gate's comes by TMA)
                if constexpr (kScalar) {
                    if (nxt.valid && warp == kElemWarp0) {
                        const int L1 = chunk_len(nxt);
                        if (2 * lane < L1) prefetch_l2(p.g + (nxt.t0 + 2 * lane) * H + nxt.h);
                        if (2 * lane + 1 < L1) prefetch_l2(p.g + (nxt.t0 + 2 * lane + 1) * H + nxt.h);
                    }
                }
                // ================ E0: beta; block products of a / the scalar gate's scan ================
                if (et < kChunk) reinterpret_cast<float*>(sm + S_BETA)[sl * 64u + et] = et < L ? beta_reg : 0.f;
                float po[4];    // channel gate: product of a over the other 8-token half of the block
                float own4[4];  // and over this thread's own 8 tokens
                if constexpr (kScalar) {
                    // the inputs must have landed: rows past the valid length are zeroed in the tiles,
                    // which are MMA operands themselves
                    bad |= !warp_wait(bar_in, ci & 1u);
                    for (int e = L * 8 + et; e < kChunk * 8; e += 256) {
#pragma unroll
                        for (int b6 = 0; b6 < 6; ++b6)
                            st_v4(sm, IN_Q + (uint32_t)b6 * 8192u + (uint32_t)e * 16u, 0u, 0u, 0u, 0u);
                    }
                    if (warp == kElemWarp0) gate_scan_scalar(sm, p, h, L, g_reg, sl);
                    fence_proxy_async();
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float own = a[0][e];
#pragma unroll
                        for (int i = 1; i < 8; ++i) own *= a[i][e];
                        own4[e] = own;
                        po[e] = __shfl_xor_sync(0xffffffffu, own, 16);
                        if ((lane >> 4) == 0) {
                            // block product (both halves agree) and the first half's product
                            reinterpret_cast<float*>(sm + S_PTOT)[eI * kHeadDim + c0 + e] = own * po[e];
                            reinterpret_cast<float*>(sm + S_PHALF)[eI * kHeadDim + c0 + e] = own;
                        }
                    }
                }
                named_bar_sync(BAR_ELEM, 256);
                PIPE_MARK(256, 2, 18);
                // ================ E2: the A/P operand tiles (channel gate) ================
                if constexpr (!kScalar) {
                    bad |= !warp_wait(bar_in, ci & 1u);
                    // the previous chunk's A/P MMA has read the tiles this phase rewrites
                    if (ci > 0) bad |= !warp_wait(bar_ap, (ci - 1) & 1u);
                    PIPE_MARK(256, 2, 19);
                    // Decays are taken relative to the middle of each 16-token block: the A side k R' and
                    // q R' with R'_r = (product of a from the block start to r) / M_I (M_I = product over
                    // the block's first 8 tokens), the diagonal-block B side k E / S2_I (S2_I = product over
                    // its last 8 tokens), so every factor lies within e^{+-8 |lower_bound|}.  The
                    // block-distance operands of block J carry M of the row block J + d.
                    const float* ptot = reinterpret_cast<const float*>(sm + S_PTOT);
                    const float* phalf = reinterpret_cast<const float*>(sm + S_PHALF);
                    const bool second = (lane >> 4) != 0;
                    auto ld4 = [&](const float* base, int J) {
                        const float4 x = *reinterpret_cast<const float4*>(base + (J < 3 ? J : 3) * kHeadDim + c0);
                        return x;
                    };
                    const float4 P1 = ld4(ptot, eI + 1), P2 = ld4(ptot, eI + 2);
                    const float4 M1 = ld4(phalf, eI + 1), M2 = ld4(phalf, eI + 2), M3 = ld4(phalf, eI + 3);
                    const float2 F1a_ = make_float2(M1.x, M1.y), F1b_ = make_float2(M1.z, M1.w);
                    const float2 P1a = make_float2(P1.x, P1.y), P1b = make_float2(P1.z, P1.w);
                    const float2 F2a_ = __fmul2_rn(P1a, make_float2(M2.x, M2.y)), F2b_ = __fmul2_rn(P1b, make_float2(M2.z, M2.w));
                    const float2 F3a_ = __fmul2_rn(__fmul2_rn(P1a, make_float2(P2.x, P2.y)), make_float2(M3.x, M3.y));
                    const float2 F3b_ = __fmul2_rn(__fmul2_rn(P1b, make_float2(P2.z, P2.w)), make_float2(M3.z, M3.w));
                    // Each thread's factors start from its own 8-token half (so that none underflows
                    // when the other half decays steeply): E is the suffix product within the half,
                    // the diagonal-block operand k E (first half) or k E / S2 (second half), the
                    // block-distance operands k E times the rest of the block (first half: S2) and
                    // F_d, and R' = (running product) / M (first half) or the running product.
                    float xs[4], cs[4], r0p[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        xs[e] = second ? fast_rcp(own4[e]) : 1.f;
                        cs[e] = second ? 1.f : po[e];
                        r0p[e] = second ? 1.f : fast_rcp(own4[e]);
                    }
                    const float2 invB01 = make_float2(xs[0], xs[1]), invB23 = make_float2(xs[2], xs[3]);
                    const float2 F1a = __fmul2_rn(make_float2(cs[0], cs[1]), F1a_),
                                 F1b = __fmul2_rn(make_float2(cs[2], cs[3]), F1b_);
                    const float2 F2a = __fmul2_rn(make_float2(cs[0], cs[1]), F2a_),
                                 F2b = __fmul2_rn(make_float2(cs[2], cs[3]), F2b_);
                    const float2 F3a = __fmul2_rn(make_float2(cs[0], cs[1]), F3a_),
                                 F3b = __fmul2_rn(make_float2(cs[2], cs[3]), F3b_);
                    uint32_t mq = 0u, mk = 0u;
                    float2 E[8][2], Rr[2];
                    {
                        const float one4[4] = {1.f, 1.f, 1.f, 1.f};
                        decay_suffix(a, one4, false, E, Rr);
                    }
                    Rr[0] = make_float2(r0p[0], r0p[1]);
                    Rr[1] = make_float2(r0p[2], r0p[3]);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int r = r0 + i;
                        Rr[0] = __fmul2_rn(Rr[0], make_float2(a[i][0], a[i][1]));
                        Rr[1] = __fmul2_rn(Rr[1], make_float2(a[i][2], a[i][3]));
                        uint2 kk = *reinterpret_cast<const uint2*>(sm + IN_K + (uint32_t)r * 256u + (uint32_t)c0 * 2u);
                        uint2 qq = *reinterpret_cast<const uint2*>(sm + IN_Q + (uint32_t)r * 256u + (uint32_t)c0 * 2u);
                        if (r >= L) kk = qq = make_uint2(0u, 0u);
                        asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(mk) : "r"(kk.x));
                        asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(mk) : "r"(kk.y));
                        asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(mq) : "r"(qq.x));
                        asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(mq) : "r"(qq.y));
                        const float2 k01 = bf16x2_to_float2(kk.x), k23 = bf16x2_to_float2(kk.y);
                        const float2 q01 = bf16x2_to_float2(qq.x), q23 = bf16x2_to_float2(qq.y);
                        const float2 kE01 = __fmul2_rn(k01, E[i][0]), kE23 = __fmul2_rn(k23, E[i][1]);
                        st_tile2(sm, AP_A + quad_off(128u, (uint32_t)r0, i, (uint32_t)c0),
                                 pack_bf16v(__fmul2_rn(k01, Rr[0])), pack_bf16v(__fmul2_rn(k23, Rr[1])));
                        st_tile2(sm, AP_A + quad_off(128u, 64u + (uint32_t)r0, i, (uint32_t)c0),
                                 pack_bf16v(__fmul2_rn(q01, Rr[0])), pack_bf16v(__fmul2_rn(q23, Rr[1])));
                        st_tile2(sm, AP_B + quad_off(160u, (uint32_t)r0, i, (uint32_t)c0),
                                 pack_bf16v(__fmul2_rn(kE01, invB01)), pack_bf16v(__fmul2_rn(kE23, invB23)));
                        if (eI <= 2)
                            st_tile2(sm, AP_B + quad_off(160u, 64u + (uint32_t)r0, i, (uint32_t)c0),
                                     pack_bf16v(__fmul2_rn(kE01, F1a)), pack_bf16v(__fmul2_rn(kE23, F1b)));
                        if (eI <= 1)
                            st_tile2(sm, AP_B + quad_off(160u, 112u + (uint32_t)r0, i, (uint32_t)c0),
                                     pack_bf16v(__fmul2_rn(kE01, F2a)), pack_bf16v(__fmul2_rn(kE23, F2b)));
                        if (eI == 0)
                            st_tile2(sm, AP_B + quad_off(160u, 144u + (uint32_t)r0, i, (uint32_t)c0),
                                     pack_bf16v(__fmul2_rn(kE01, F3a)), pack_bf16v(__fmul2_rn(kE23, F3b)));
                    }
                    // |q|, |k| bound every fp16 operand built from them (the decay factors are <= 1)
                    const float2 mkf = bf16x2_to_float2(mk), mqf = bf16x2_to_float2(mq);
                    if (fmaxf(fmaxf(fabsf(mkf.x), fabsf(mkf.y)), fmaxf(fabsf(mqf.x), fabsf(mqf.y))) >= kRangeHi)
                        range_bad = 1u;
                    fence_proxy_async();
                    named_bar_sync(BAR_ELEM, 256);
                }
                PIPE_MARK(256, 2, 20);
                // the A/P operands are ready (the chain issues the MMA), and so are the chunk's beta,
                // P diagonal and scalar Gamma, which the aux warps read (published after the barrier)
                if (elead) {
                    seq_publish(sRdSeq, ci + 1u);
                    mbar_arrive(bar_apready);
                }
                // ================ E4: the chain's operands (once it is done with the last chunk's) ================
                if (ci > 0) bad |= !warp_wait(bar_s, (ci - 1) & 1u);
                PIPE_MARK(256, 2, 21);
                if constexpr (kScalar) {
                    // per-token scalings of the swizzled input blocks; inputs and outputs share the
                    // 128-byte-swizzled geometry, so an item is one 16-byte position of a row
                    const float* sb = reinterpret_cast<const float*>(sm + S_BETA) + sl * 64u;
                    const float* ge = reinterpret_cast<const float*>(sm + s_ge(sl));
                    const float* kf = reinterpret_cast<const float*>(sm + s_kf(sl));
                    uint32_t mq = 0u, mk = 0u;
                    float mbk = 0.f;
#pragma unroll 1
                    for (int e = et; e < kChunk * 16; e += 256) {
                        const int r = e >> 4;
                        const uint32_t cb = (uint32_t)(e >> 3) & 1u, pos = (uint32_t)e & 7u;
                        const uint32_t off = cb * 16384u + (uint32_t)r * 128u + pos * 16u;
                        const uint4 kw = *reinterpret_cast<const uint4*>(sm + IN_Q + off);
                        const uint4 qw = *reinterpret_cast<const uint4*>(sm + IN_Q + off + 8192u);
                        const float g = ge[r], nbg = -sb[r] * g, kfr = kf[r];
                        const float2 g2 = make_float2(g, g), nbg2 = make_float2(nbg, nbg), kf2 = make_float2(kfr, kfr);
                        const uint32_t kk[4] = {kw.x, kw.y, kw.z, kw.w}, qq[4] = {qw.x, qw.y, qw.z, qw.w};
                        uint32_t oq[4], ok[4], oh[4];
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(mk) : "r"(kk[x]));
                            asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(mq) : "r"(qq[x]));
                            const float2 kx = bf16x2_to_float2(kk[x]), qx = bf16x2_to_float2(qq[x]);
                            const float2 gq = __fmul2_rn(g2, qx), bk = __fmul2_rn(nbg2, kx), kh = __fmul2_rn(kf2, kx);
                            oq[x] = pack_f16s(gq.x, gq.y);
                            ok[x] = pack_f16s(bk.x, bk.y);
                            oh[x] = pack_f16s(kh.x, kh.y);
                            mbk = fmaxf(mbk, fmaxf(fabsf(bk.x), fabsf(bk.y)));
                        }
                        st_tile4(sm, B1 + off, oq[0], oq[1], oq[2], oq[3]);
                        st_tile4(sm, B1 + off + 8192u, ok[0], ok[1], ok[2], ok[3]);
                        st_tile4(sm, KH + cb * 8192u + (uint32_t)r * 128u + pos * 16u, oh[0], oh[1], oh[2], oh[3]);
                    }
                    const float2 mkf = bf16x2_to_float2(mk), mqf = bf16x2_to_float2(mq);
                    if (fmaxf(fmaxf(fabsf(mkf.x), fabsf(mkf.y)), fmaxf(fabsf(mqf.x), fabsf(mqf.y))) >= kRangeHi ||
                        mbk >= kRangeHi)
                        range_bad = 1u;
                    if (et < kHeadDim)
                        reinterpret_cast<float*>(sm + S_GC)[sl * kHeadDim + et] = ge[kChunk - 1];
                } else {
                    const float* ptot = reinterpret_cast<const float*>(sm + S_PTOT);
                    float2 before[2] = {make_float2(1.f, 1.f), make_float2(1.f, 1.f)};
                    float2 after[2] = {make_float2(1.f, 1.f), make_float2(1.f, 1.f)};
#pragma unroll
                    for (int J = 0; J < 4; ++J) {
                        const float4 x = *reinterpret_cast<const float4*>(ptot + J * kHeadDim + c0);
                        const float2 x01 = make_float2(x.x, x.y), x23 = make_float2(x.z, x.w);
                        if (J < eI) {
                            before[0] = __fmul2_rn(before[0], x01);
                            before[1] = __fmul2_rn(before[1], x23);
                        }
                        if (J > eI) {
                            after[0] = __fmul2_rn(after[0], x01);
                            after[1] = __fmul2_rn(after[1], x23);
                        }
                    }
                    const float* sb = reinterpret_cast<const float*>(sm + S_BETA) + sl * 64u;
                    float2 E[8][2], Rr[2];
                    decay_suffix(a, po, (lane >> 4) != 0, E, Rr);
                    // E times the products of the later blocks: Khat's factor
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        E[i][0] = __fmul2_rn(E[i][0], after[0]);
                        E[i][1] = __fmul2_rn(E[i][1], after[1]);
                    }
                    Rr[0] = __fmul2_rn(Rr[0], before[0]);
                    Rr[1] = __fmul2_rn(Rr[1], before[1]);
                    float nbk = 0.f;   // max |beta k| over the thread's rows
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int r = r0 + i;
                        const float nb = -sb[r];
                        const float2 nb2 = make_float2(nb, nb);
                        // gamma = R times the products of the earlier blocks
                        Rr[0] = __fmul2_rn(Rr[0], make_float2(a[i][0], a[i][1]));
                        Rr[1] = __fmul2_rn(Rr[1], make_float2(a[i][2], a[i][3]));
                        // k, q again from the input tiles (still resident: the next chunk's loads are
                        // issued after this phase); rows past the valid length are zero
                        uint2 kk = *reinterpret_cast<const uint2*>(sm + IN_K + (uint32_t)r * 256u + (uint32_t)c0 * 2u);
                        uint2 qq = *reinterpret_cast<const uint2*>(sm + IN_Q + (uint32_t)r * 256u + (uint32_t)c0 * 2u);
                        if (r >= L) kk = qq = make_uint2(0u, 0u);
                        const float2 k01 = bf16x2_to_float2(kk.x), k23 = bf16x2_to_float2(kk.y);
                        const float2 q01 = bf16x2_to_float2(qq.x), q23 = bf16x2_to_float2(qq.y);
                        const float2 kg01 = __fmul2_rn(k01, Rr[0]), kg23 = __fmul2_rn(k23, Rr[1]);
                        st_tile2(sm, B1 + quad_off(128u, (uint32_t)r0, i, (uint32_t)c0),
                                 pack_f16v(__fmul2_rn(q01, Rr[0])), pack_f16v(__fmul2_rn(q23, Rr[1])));
                        st_tile2(sm, B1 + quad_off(128u, 64u + (uint32_t)r0, i, (uint32_t)c0),
                                 pack_f16v(__fmul2_rn(nb2, kg01)), pack_f16v(__fmul2_rn(nb2, kg23)));
                        st_tile2(sm, KH + quad_off(64u, (uint32_t)r0, i, (uint32_t)c0),
                                 pack_f16v(__fmul2_rn(k01, E[i][0])), pack_f16v(__fmul2_rn(k23, E[i][1])));
                        nbk = fmaxf(nbk, fabsf(nb) * fmaxf(fmaxf(fabsf(k01.x), fabsf(k01.y)), fmaxf(fabsf(k23.x), fabsf(k23.y))));
                    }
                    // |beta k| bounds the -beta gamma k operand (the decay factors are <= 1)
                    if (nbk >= kRangeHi) range_bad = 1u;
                    if (eI == 0 && (lane >> 4) == 0) {
                        float gc[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
                        for (int J = 0; J < 4; ++J) {
                            const float4 x = *reinterpret_cast<const float4*>(ptot + J * kHeadDim + c0);
                            gc[0] *= x.x; gc[1] *= x.y; gc[2] *= x.z; gc[3] *= x.w;
                        }
                        *reinterpret_cast<float4*>(reinterpret_cast<float*>(sm + S_GC) + sl * kHeadDim + c0) =
                            make_float4(gc[0], gc[1], gc[2], gc[3]);
                    }
                }
                if constexpr (kScalar) {
                    // V^T (bf16 [128 v][64 i], 128-byte rows, 16-byte chunk j at j ^ (v & 7)): thread ->
                    // value columns 2 vp and 2 vp + 1, tokens 16 tq .. 16 tq + 15 (the channel gate's
                    // aux warps form it, with P's diagonal)
                    const int vp = et & 63, tq = et >> 6;
                    const uint32_t v0 = 2u * (uint32_t)vp, v1 = v0 + 1u;
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        uint32_t w[8];
#pragma unroll
                        for (int t = 0; t < 8; ++t) {
                            const int r = 16 * tq + 8 * j + t;
                            uint32_t voff;
                            if constexpr (kScalar)   // 64-channel swizzled blocks: element (r, v0) of block v0 / 64
                                voff = (v0 >> 6) * 8192u + (uint32_t)r * 128u +
                                       ((((v0 & 63u) >> 3) ^ ((uint32_t)r & 7u)) << 4) + (v0 & 7u) * 2u;
                            else
                                voff = (uint32_t)r * 256u + (uint32_t)vp * 4u;
                            w[t] = (r < L && !(p.flags & kFlagVZero)) ? *reinterpret_cast<const uint32_t*>(sm + IN_V + voff)
                                                                      : 0u;
                        }
                        const uint32_t ch = (uint32_t)(2 * tq + j);
                        st_tile4(sm, VT + v0 * 128u + ((ch ^ (v0 & 7u)) << 4), __byte_perm(w[0], w[1], 0x5410),
                                 __byte_perm(w[2], w[3], 0x5410), __byte_perm(w[4], w[5], 0x5410),
                                 __byte_perm(w[6], w[7], 0x5410));
                        st_tile4(sm, VT + v1 * 128u + ((ch ^ (v1 & 7u)) << 4), __byte_perm(w[0], w[1], 0x7632),
                                 __byte_perm(w[2], w[3], 0x7632), __byte_perm(w[4], w[5], 0x7632),
                                 __byte_perm(w[6], w[7], 0x7632));
                    }
                }
                if (elead) {
                    int32_t* meta = sMeta + sl * 16u;
                    meta[0] = 1;
                    meta[1] = cur.h;
                    meta[2] = cur.n;
                    meta[3] = (int32_t)cur.t0;
                    meta[4] = L;
                    meta[5] = cur.t0 == cur.bos ? 1 : 0;
                    meta[6] = cur.t0 + kChunk >= cur.eos ? 1 : 0;
                    meta[7] = nxt.valid ? 1 : 0;   // another chunk follows in this CTA
                    meta[8] = nxt.h;
                    meta[9] = (int32_t)nxt.t0;
                }
                fence_proxy_async();
                if (named_bar_or(BAR_ELEM, 256, bad || *sAbort != 0u)) {
                    aborted = true;
                    break;
                }
                PIPE_MARK(256, 2, 22);
                // hand the chunk to the chain (which then loads the next chunk's inputs over these)
                if (elead) mbar_arrive(bar_formed);
                // ================ E6: the next chunk's beta and gate ================
                if (nxt.valid) {
                    load_beta(nxt);
                    if constexpr (kScalar) {
                        if (warp == kElemWarp0) load_g_scalar(nxt);
                    } else {
                        if (!warp_wait(bar_g, (ci + 1u) & 1u)) *sAbort = 1u;
                        gate_tokens(p, nxt.h, reinterpret_cast<const float*>(sm + AP_A), chunk_len(nxt), c0, r0, a);
                    }
                }
                PIPE_MARK(256, 2, 23);
                cur = nxt;
                ++ci;
            }
            if (aborted) *sAbort = 1u;
        } else {
            // ======================= aux warps =======================
            // For each chunk: once its A/P MMA is done, the next chunk's gate input (channel gate);
            // then the A / P read-out (once the chain is done with the last chunk's P and T) and the
            // solve.
            const int sw = warp - kAuxWarp0;
            float tmax = 0.f;
            // sign * (a 16 x 16 warp-MMA accumulator) into block (I, J) of the fp16 T tile
            auto acc_to_t16 = [&](int I, int J, const float (&acc)[2][4], float sign) {
                const int g = lane >> 2, t = lane & 3;
#pragma unroll
                for (int nh = 0; nh < 2; ++nh) {
                    const uint32_t col = (uint32_t)(16 * J + 8 * nh + 2 * t);
                    tmax = fmaxf(tmax, fmaxf(fmaxf(fabsf(acc[nh][0]), fabsf(acc[nh][1])),
                                             fmaxf(fabsf(acc[nh][2]), fabsf(acc[nh][3]))));
                    *reinterpret_cast<uint32_t*>(sm + T16 + sw128_off((uint32_t)(16 * I + g), col, 64u)) =
                        pack_f16s(sign * acc[nh][0], sign * acc[nh][1]);
                    *reinterpret_cast<uint32_t*>(sm + T16 + sw128_off((uint32_t)(16 * I + g + 8), col, 64u)) =
                        pack_f16s(sign * acc[nh][2], sign * acc[nh][3]);
                }
            };
            while (cur.valid) {
                const Cursor nxt = next_chunk(p, sOrder, b, G, units, cur);
                const uint32_t cj = ci, slp = cj & 1u;
                bool bad = false;
                // the chain is done with the last chunk's V^T, P^T and T (its [S | O] MMA has completed)
                if (cj > 0) bad |= !warp_wait(bar_s, (cj - 1u) & 1u);
                if constexpr (!kScalar) {
                    // ================ A-1: V^T and P's exact diagonal of chunk cj ================
                    const int L = chunk_len(cur);
                    bad |= !warp_wait(bar_in, cj & 1u);
                    {
                        // V^T: thread -> value columns 2 vp and 2 vp + 1, tokens 32 th .. 32 th + 31
                        const int vp = at & 63, th = at >> 6;
                        const uint32_t v0 = 2u * (uint32_t)vp, v1 = v0 + 1u;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            uint32_t w[8];
#pragma unroll
                            for (int t = 0; t < 8; ++t) {
                                const int r = 32 * th + 8 * j + t;
                                w[t] = (r < L && !(p.flags & kFlagVZero))
                                           ? *reinterpret_cast<const uint32_t*>(sm + IN_V + (uint32_t)r * 256u + (uint32_t)vp * 4u)
                                           : 0u;
                            }
                            const uint32_t ch = (uint32_t)(4 * th + j);
                            st_tile4(sm, VT + v0 * 128u + ((ch ^ (v0 & 7u)) << 4), __byte_perm(w[0], w[1], 0x5410),
                                     __byte_perm(w[2], w[3], 0x5410), __byte_perm(w[4], w[5], 0x5410),
                                     __byte_perm(w[6], w[7], 0x5410));
                            st_tile4(sm, VT + v1 * 128u + ((ch ^ (v1 & 7u)) << 4), __byte_perm(w[0], w[1], 0x7632),
                                     __byte_perm(w[2], w[3], 0x7632), __byte_perm(w[4], w[5], 0x7632),
                                     __byte_perm(w[6], w[7], 0x7632));
                        }
                    }
                    {
                        // q_r . k_r in fp32 over one 64-channel half; 16-byte chunks visited in a
                        // row-dependent order (conflict-free)
                        const int r = at & 63, hh = at >> 6;
                        float pd = 0.f;
                        if (r < L) {
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const uint32_t off = (uint32_t)r * 256u + (uint32_t)hh * 128u + (((uint32_t)(j + r) & 7u) << 4);
                                const uint4 qv = *reinterpret_cast<const uint4*>(sm + IN_Q + off);
                                const uint4 kv = *reinterpret_cast<const uint4*>(sm + IN_K + off);
                                const uint32_t qa[4] = {qv.x, qv.y, qv.z, qv.w}, ka[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const float2 a2 = bf16x2_to_float2(qa[e]), b2 = bf16x2_to_float2(ka[e]);
                                    pd = fmaf(a2.x, b2.x, pd);
                                    pd = fmaf(a2.y, b2.y, pd);
                                }
                            }
                        }
                        reinterpret_cast<float*>(sm + S_PD2)[(slp * 2u + (uint32_t)hh) * 64u + r] = pd;
                    }
                    fence_proxy_async();
                    named_bar_sync(BAR_AUX, 128);
                    if (at == 0) mbar_arrive(bar_vt);
                }
                // ================ A0: wait for the chunk's A/P product ================
                bad |= !warp_wait(bar_ap, cj & 1u);
                // channel gate: the next chunk's gate input into the operand tiles the MMA has read
                if constexpr (!kScalar) {
                    if (loader && nxt.valid && !bad) load_gate_input(nxt, (cj + 1u) & 1u);
                }
                // the element warps have published the chunk's beta (and scalar Gamma)
                bad |= !__all_sync(0xffffffffu, seq_wait(sRdSeq, cj + 1u));
                if (bad) *sAbort = 1u;
                fence_after_sync();
                PIPE_MARK(128, 0, 0);
                const bool isA = quarter < 2;
                const int r = (quarter & 1) * 32 + lane;      // token row of A (k rows) or P (q rows)
                const int I = r >> 4;
                const float be = reinterpret_cast<const float*>(sm + S_BETA)[slp * 64u + r];
                float pdg = 0.f;
                if constexpr (!kScalar) {
                    const float* pd = reinterpret_cast<const float*>(sm + S_PD2) + slp * 128u;
                    pdg = pd[r] + pd[64 + r];
                }
                float pmax = 0.f;
#pragma unroll 1
                for (int J = 0; J < 4; ++J) {
                    float row[16];
                    auto pick = [&](uint32_t col_a, uint32_t col_b, int I_a) {
                        uint32_t ta[16], tb[16];
                        tmem_ld16(taddr(tbase, quarter, TM_AP + col_a), ta);
                        tmem_ld16(taddr(tbase, quarter, TM_AP + col_b), tb);
                        tmem_wait_ld();
#pragma unroll
                        for (int x = 0; x < 16; ++x) row[x] = __uint_as_float(I == I_a ? ta[x] : tb[x]);
                    };
                    if constexpr (kScalar) {
                        // raw K K^T / Q K^T times the scalar decay 2^(Gamma_r - Gamma_i) (<= 1 on
                        // and below the diagonal)
                        uint32_t raw[16];
                        tmem_ld16(taddr(tbase, quarter, TM_AP + (uint32_t)J * 16u), raw);
                        tmem_wait_ld();
                        const float* gam = reinterpret_cast<const float*>(sm + s_gam(slp));
                        const float gr = gam[r];
#pragma unroll
                        for (int x = 0; x < 16; ++x) {
                            const int i = J * 16 + x;
                            const bool keep = isA ? (i < r) : (i <= r);
                            row[x] = keep ? __uint_as_float(raw[x]) * fast_ex2(gr - gam[i]) : 0.f;
                        }
                    } else {
                        if ((quarter & 1) == 0) {        // I in {0, 1}
                            if (J == 0) pick(0, 64, 0);            // I=0: diagonal; I=1: C1 of block 0
                            else if (J == 1) pick(16, 16, 1);      // I=1: diagonal (I=0: masked)
                            else {
#pragma unroll
                                for (int x = 0; x < 16; ++x) row[x] = 0.f;
                            }
                        } else {                         // I in {2, 3}
                            if (J == 0) pick(112, 144, 2);         // I=2: C2 of block 0; I=3: C3 of block 0
                            else if (J == 1) pick(80, 128, 2);     // I=2: C1 of block 1; I=3: C2 of block 1
                            else if (J == 2) pick(32, 96, 2);      // I=2: diagonal; I=3: C1 of block 2
                            else pick(48, 48, 3);                  // I=3: diagonal (I=2: masked)
                        }
#pragma unroll
                        for (int x = 0; x < 16; ++x) {
                            const int i = J * 16 + x;
                            row[x] = i < r ? row[x] : ((i == r && !isA) ? pdg : 0.f);
                        }
                    }
                    if (isA) {
                        // beta-scaled A: diagonal blocks in fp32 (the forward substitution), the
                        // blocks below in fp16 (operands of the block products)
                        if (J == I) {
                            float* ad = reinterpret_cast<float*>(sm + SV_AD) + (I * 16 + (r & 15)) * kAdPitch;
#pragma unroll
                            for (int x = 0; x < 16; x += 4)
                                *reinterpret_cast<float4*>(ad + x) =
                                    make_float4(be * row[x], be * row[x + 1], be * row[x + 2], be * row[x + 3]);
                        } else if (J < I) {
                            uint32_t hv[8];
#pragma unroll
                            for (int x = 0; x < 8; ++x) hv[x] = warpmma::pack_half2(be * row[2 * x], be * row[2 * x + 1]);
                            const uint32_t off = al_off(I, J) + (uint32_t)(r & 15) * kHp * 2u;
                            st_v4(sm, off, hv[0], hv[1], hv[2], hv[3]);
                            st_v4(sm, off + 16u, hv[4], hv[5], hv[6], hv[7]);
                        }
                    } else {
                        // P^T (MN-major, K = token i, N = row r): 16-bit stores, a warp writes 64
                        // contiguous bytes per i
#pragma unroll
                        for (int x = 0; x < 16; ++x) {
                            const int i = J * 16 + x;
                            pmax = fmaxf(pmax, fabsf(row[x]));
                            st_tile_h(sm, PT + sw128_off((uint32_t)i, (uint32_t)r, 64u),
                                      __half_as_ushort(__float2half_rn(fminf(fmaxf(row[x], -65504.f), 65504.f))));
                        }
                    }
                }
                if (pmax >= kRangeHi) range_bad = 1u;
                fence_proxy_async();
                tmem_wait_ld();
                fence_before_sync();
                named_bar_sync(BAR_AUX, 128);
                // the accumulator is free for the next chunk's A/P MMA
                if (at == 0) mbar_arrive(bar_ro);
                PIPE_MARK(128, 0, 1);
                // ================ A1: T = (I + A)^-1 of chunk cj ================
                // L0: the four 16 x 16 diagonal blocks by forward substitution in fp32, one column
                // per thread (threads 0-63), right-looking; written to the fp16 T tile
                if (sw < 2) {
                    const int bI = at >> 4, jc = at & 15, o = bI * 16;
                    const float* ad = reinterpret_cast<const float*>(sm + SV_AD) + bI * 16 * kAdPitch;
                    float x[16];
#pragma unroll
                    for (int rr = 0; rr < 16; ++rr) x[rr] = (rr == jc) ? 1.f : 0.f;
#pragma unroll
                    for (int ii = 0; ii < 15; ++ii) {
                        const float xi = x[ii];
#pragma unroll
                        for (int rr = ii + 1; rr < 16; ++rr) x[rr] = fmaf(-ad[rr * kAdPitch + ii], xi, x[rr]);
                    }
#pragma unroll
                    for (int rr = 0; rr < 16; ++rr) {
                        tmax = fmaxf(tmax, fabsf(x[rr]));
                        st_tile_h(sm, T16 + sw128_off((uint32_t)(o + rr), (uint32_t)(o + jc), 64u),
                                  __half_as_ushort(__float2half_rn(fminf(fmaxf(x[rr], -65504.f), 65504.f))));
                    }
                }
                named_bar_sync(BAR_AUX, 128);
                PIPE_MARK(128, 0, 2);
                // L1 (16 x 16 warp-MMA products, fp16 operands, fp32 accumulation):
                //   T10 = -T11 (A10 T00), T32 = -T33 (A32 T22),
                //   X20 = A20 T00 + A21 T10, X30 = A30 T00 + A31 T10, X21 = A21 T11, X31 = A31 T11.
                // Aux warps 0 and 2 both form T10 (warp 2 in its own scratch) so that neither waits
                // for the other.
                {
                    float acc[2][4] = {};
                    if (sw == 0 || sw == 2) {
                        const uint32_t ysc = sw == 0 ? SC_Y0 : SC_Y2;
                        mm16h(acc, lm_blk(sm, al_off(1, 0)), lm_t16(sm, 0, 0));       // A10 T00
                        store16h(sm, ysc, acc, 1.f);
                        __syncwarp();
                        float a2[2][4] = {};
                        mm16h(a2, lm_t16(sm, 1, 1), lm_blk(sm, ysc));                 // T10
                        if (sw == 0) acc_to_t16(1, 0, a2, -1.f);
                        else store16h(sm, SC_T10B, a2, -1.f);
                        __syncwarp();
                        const int I = sw == 0 ? 2 : 3;
                        float a3[2][4] = {};
                        mm16h(a3, lm_blk(sm, al_off(I, 0)), lm_t16(sm, 0, 0));
                        mm16h(a3, lm_blk(sm, al_off(I, 1)), sw == 0 ? lm_t16(sm, 1, 0) : lm_blk(sm, SC_T10B));
                        store16h(sm, sw == 0 ? SC_X20 : SC_X30, a3, 1.f);             // X20 / X30
                    } else if (sw == 1) {
                        mm16h(acc, lm_blk(sm, al_off(3, 2)), lm_t16(sm, 2, 2));       // A32 T22
                        store16h(sm, SC_Y32, acc, 1.f);
                        __syncwarp();
                        float a2[2][4] = {};
                        mm16h(a2, lm_t16(sm, 3, 3), lm_blk(sm, SC_Y32));
                        acc_to_t16(3, 2, a2, -1.f);                                   // T32
                        float a3[2][4] = {};
                        mm16h(a3, lm_blk(sm, al_off(2, 1)), lm_t16(sm, 1, 1));
                        store16h(sm, SC_X21, a3, 1.f);                                // X21
                    } else {
                        mm16h(acc, lm_blk(sm, al_off(3, 1)), lm_t16(sm, 1, 1));
                        store16h(sm, SC_X31, acc, 1.f);                               // X31
                    }
                }
                named_bar_sync(BAR_AUX, 128);
                // L2: T_LL = -T_LR X, written straight to the fp16 tile:
                //   T20 = -T22 X20, T21 = -T22 X21, T30 = -(T32 X20 + T33 X30), T31 = -(T32 X21 + T33 X31)
                {
                    float acc[2][4] = {};
                    const int J = sw & 1;
                    if (sw < 2) {
                        mm16h(acc, lm_t16(sm, 2, 2), lm_blk(sm, J == 0 ? SC_X20 : SC_X21));
                        acc_to_t16(2, J, acc, -1.f);
                    } else {
                        mm16h(acc, lm_t16(sm, 3, 2), lm_blk(sm, J == 0 ? SC_X20 : SC_X21));
                        mm16h(acc, lm_t16(sm, 3, 3), lm_blk(sm, J == 0 ? SC_X30 : SC_X31));
                        acc_to_t16(3, J, acc, -1.f);
                    }
                }
                if (tmax >= kRangeHi) range_bad = 1u;
                fence_proxy_async();
                named_bar_sync(BAR_AUX, 128);
                if (at == 0) mbar_arrive(bar_t);
                PIPE_MARK(128, 0, 3);
                PIPE_MARK(128, 0, 4);
                if (named_bar_or(BAR_AUX, 128, *sAbort != 0u)) {
                    aborted = true;
                    break;
                }
                PIPE_MARK(128, 0, 5);
                cur = nxt;
                ++ci;
            }
            if (aborted) {
                *sAbort = 1u;
                if (loader && tma_pending) mbar_wait_bounded(bar_in, tma_parity);
                if (loader && g_pending) mbar_wait_bounded(bar_g, g_parity);
            }
        }
        if (range_bad) record_error(KDA_DEVERR_RANGE);
    }

    // wind-down: every role has drained its own asynchronous operations
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == 0) tmem_dealloc(tbase, TM_COLS);
#ifdef KDA_PHASE_CLOCKS
    if (tid == 0) {
        for (int i = 0; i < kPhases; ++i) atomicAdd(&g_pipe_phase_cycles[i], (unsigned long long)sPh[i]);
        if (blockIdx.x < kMaxCtaRecords) {
            unsigned int smid;
            asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
            g_pipe_cta[blockIdx.x][0] = t_entry;
            g_pipe_cta[blockIdx.x][1] = global_ns();
            g_pipe_cta[blockIdx.x][2] = n_chunks;
            g_pipe_cta[blockIdx.x][3] = smid;
            for (int i = 0; i < kPhases; ++i) g_pipe_cta[blockIdx.x][4 + i] = sPh[i];
        }
    }
#endif
}

// ---- host side ----

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link-time libcuda symbol).
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 2-D map over [rows][cols] with a box of box_cols x 64 rows; swizzled maps put each box in the
// 128-byte-swizzled K-major layout of the MMA operands.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint32_t elem, int64_t rows, int64_t cols,
              uint32_t box_cols = kHeadDim, bool swizzle128 = false) {
    auto fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * elem};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)kChunk};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kScalar>
cudaError_t launch(const StagedArgs& a, cudaStream_t stream) {
    cudaError_t err = once_per_device([](int) {
        return cudaFuncSetAttribute(kda_pipe_kernel<kScalar>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)SMEM_ALLOC);
    });
    if (err != cudaSuccess) return err;
    int dev = 0, sm_count = 0;
    if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
    if ((err = cudaDeviceGetAttribute(&sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return err;
    if (sm_count <= 0) return cudaErrorInvalidDevice;
    CUtensorMap tq, tk, tv, tg;
    const int64_t rows = a.total_tokens, cols = (int64_t)a.H * kHeadDim;
    // channel-wise gate: 128-channel unswizzled boxes (CUDA cores read them); scalar gate:
    // 64-channel 128-byte-swizzled boxes (the MMA reads them)
    const uint32_t box = kScalar ? 64u : (uint32_t)kHeadDim;
    if (!make_map(&tq, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, cols, box, kScalar) ||
        !make_map(&tk, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, cols, box, kScalar) ||
        !make_map(&tv, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, cols, box, kScalar))
        return cudaErrorInvalidValue;
    if (kScalar) {
        tg = tq;   // unused: the scalar gate input is read with plain loads
    } else if (!make_map(&tg, a.g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, rows, cols)) {
        return cudaErrorInvalidValue;
    }
    Params p;
    p.g = a.g;
    p.beta = a.beta;
    p.A_log = a.A_log;
    p.dt_bias = a.dt_bias;
    p.lower_bound = a.lower_bound;
    p.scale = a.scale;
    p.initial_state = a.initial_state;
    p.cu_seqlens = a.cu_seqlens;
    p.out = static_cast<__nv_bfloat16*>(a.out);
    p.final_state = a.final_state;
    p.seqlen = a.seqlen;
    p.total_tokens = a.total_tokens;
    p.H = a.H;
    p.N = a.N;
    p.flags = a.flags;
    const int64_t units = (int64_t)a.N * a.H;
    const int grid = (int)(units < sm_count ? units : sm_count);
    if (grid <= 0) return cudaSuccess;
    kda_pipe_kernel<kScalar><<<grid, kThreads, SMEM_ALLOC, stream>>>(tq, tk, tv, tg, p);
    return cudaGetLastError();
}

}  // namespace pipe

#ifdef KDA_PHASE_CLOCKS
// Debug builds only: copies and clears the per-phase cycle totals of the pipelined kernel
// (slots 0-6: aux warps, thread 128; slots 9-17: chain, thread 0; slots 18-23: element warps,
// thread 256).
extern "C" int kda_debug_pipe_phase_cycles(unsigned long long* out) {
    if (cudaMemcpyFromSymbol(out, pipe::g_pipe_phase_cycles, sizeof(unsigned long long) * pipe::kPhases) !=
        cudaSuccess)
        return -1;
    unsigned long long zero[pipe::kPhases] = {};
    return cudaMemcpyToSymbol(pipe::g_pipe_phase_cycles, zero, sizeof zero) == cudaSuccess ? pipe::kPhases : -1;
}
// Debug builds only: per-CTA records of the last launch (entry and exit global time in ns, chunks
// run, SM id, then the CTA's cycles per phase slot), up to max_ctas of them; returns how many
// were copied.
extern "C" int kda_debug_pipe_cta(unsigned long long* out, int max_ctas) {
    const int n = max_ctas < pipe::kMaxCtaRecords ? max_ctas : pipe::kMaxCtaRecords;
    if (n <= 0) return 0;
    return cudaMemcpyFromSymbol(out, pipe::g_pipe_cta, sizeof(unsigned long long) * pipe::kCtaRec * (size_t)n) ==
                   cudaSuccess
               ? n
               : -1;
}
#endif

bool fused_supported(float lower_bound) { return lower_bound >= KDA_FUSED_MIN_LOWER_BOUND; }
cudaError_t launch_pipe(const StagedArgs& a, cudaStream_t stream) { return pipe::launch<false>(a, stream); }
cudaError_t launch_pipe_gdn(const StagedArgs& a, cudaStream_t stream) { return pipe::launch<true>(a, stream); }

}  // namespace kda
