/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention chunked-prefill forward.
 *
 * The operation (FlashKDA posts: donniechu.com, section "Số liệu kỹ thuật" --
 * flash_kda.fwd() with batch, variable length via cu_seqlens, initial/final
 * recurrent state, fine-grained channel-wise gate with learned A_log, dt_bias,
 * lower_bound, bf16 + fp32 precision, K = V = 128; toolarium.ru post, section
 * "Где ограничения прямо сейчас" -- K = V = 128 is a hard constraint and the
 * released kernels target the prefill forward).  The pages print no formula;
 * this library computes, per sequence and head, with S a K x V fp32 state:
 *
 *   log a_t = max(-exp(A_log[h]) * softplus(g_t + dt_bias[h]), lower_bound)  (per channel)
 *   S_t     = (I - beta_t k_t k_t^T) Diag(a_t) S_{t-1} + beta_t k_t v_t^T
 *   o_t     = scale * S_t^T q_t
 *
 * S_0 = initial_state (or 0); final_state = S after the sequence's last token.
 *
 * Layouts (all row-major, all pointers are DEVICE memory owned by the caller):
 *   q, k        bf16  [Ttot, H, 128]     Ttot = batch * seqlen (fixed) or the packed total
 *   v           bf16  [Ttot, H, 128]
 *   g           fp32  [Ttot, H, 128]     raw gate input
 *   beta        fp32  [Ttot, H]
 *   A_log       fp32  [H]
 *   dt_bias     fp32  [H, 128]
 *   initial_state fp32 [N, H, 128, 128]  ([seq][head][k][v]); NULL means zeros
 *   cu_seqlens  int32 [N + 1]            NULL means N = batch sequences of length seqlen
 *   out         bf16  [Ttot, H, 128]     written, rounded to nearest even from fp32
 *   final_state fp32  [N, H, 128, 128]   NULL means "do not write"
 * With cu_seqlens, batch must be 1, seqlen is the packed total Ttot, N = num_seqs,
 * cu_seqlens[0] = 0, cu_seqlens[N] = Ttot and the offsets are non-decreasing
 * (empty sequences are allowed: their final state is their initial state).
 * cu_seqlens is read only on the device: no call synchronises with the host.
 *
 * Alignment: every tensor base address must be 16-byte aligned, except beta (and the
 * scalar-gate g of kda_gdn_fwd), which need 4 bytes: slices at any token offset.
 * Aliasing: final_state may alias initial_state (in-place state update); out
 * must not overlap any input.
 * Streams: every compute call is asynchronous on `stream` (a cudaStream_t;
 * NULL = the legacy default stream).  Argument errors are reported
 * synchronously, before any launch.
 * A kernel that detects a violated precondition on the device (offsets out of
 * range, a wait that ran out) records it in a device error word instead of
 * faulting; kda_check_device_error() reads and clears it.
 * Contexts: the library sets its kernels' shared-memory attributes once per device and
 * process.  Do not call it again after cudaDeviceReset in the same process: the attributes
 * belong to the destroyed context, and the launches of the new one are refused (KDA_ERR_CUDA).
 * Nothing else is cached across calls (kda_fwd_staged_noalloc looks its scratch up each time).
 */
#ifndef KDA_H
#define KDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* kda_stream_t;   /* same type as cudaStream_t */

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,   /* NULL required pointer, bad dims, bad scalar */
    KDA_ERR_UNSUPPORTED = 2,   /* head dims other than 128, or no sm_100 device */
    KDA_ERR_ALIGNMENT = 3,     /* a base address not 16-byte aligned */
    KDA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
    KDA_ERR_DEVICE = 5,        /* a kernel recorded a device-side error (see kda_check_device_error) */
    KDA_ERR_WORKSPACE = 6,     /* workspace missing or smaller than required */
    KDA_ERR_SCRATCH_LIMIT = 7  /* kda_fwd_staged_noalloc: problem exceeds its fixed scratch */
} kda_status;

typedef struct {
    int32_t batch;       /* B: sequences of the fixed-length layout (1 with cu_seqlens) */
    int64_t seqlen;      /* tokens per sequence (fixed) or packed total Ttot (varlen) */
    int32_t num_heads;   /* H >= 1 */
    int32_t num_seqs;    /* N with cu_seqlens; ignored (taken as batch) without */
    int32_t head_dim_k;  /* must be 128 */
    int32_t head_dim_v;  /* must be 128 */
} kda_dims;

/* Device error bits recorded by kernels (returned by kda_check_device_error via
 * kda_last_device_error_bits). */
#define KDA_DEVERR_BAD_OFFSETS 0x1u   /* cu_seqlens not monotone / out of [0, Ttot] */
#define KDA_DEVERR_TIMEOUT     0x2u   /* a bounded wait ran out of iterations */
#define KDA_DEVERR_BOUNDS      0x4u   /* an index outside its buffer was skipped */
#define KDA_DEVERR_RANGE       0x8u   /* kda_fwd: an input outside the fused path's operating range
                                         (see kda_fwd); the affected values were saturated */

/*
 * kda_fwd -- the chunked prefill forward (the product path).
 *
 * Runs the fused persistent sm_100a kernel when lower_bound >= KDA_FUSED_MIN_LOWER_BOUND, and
 * the staged exact-decay kernels otherwise (their intra-chunk decays are formed pair by pair and
 * cannot overflow for any gate).  The staged fallback allocates its workspace stream-ordered
 * (cudaMallocAsync).
 *
 * The fused kernel: one CTA per SM carries each (sequence, head) state in tensor memory and
 * runs the 64-token chunks through tcgen05 MMAs with fp16/bf16 operands and fp32 accumulation;
 * warps 0-3 advance the state while the others build the next chunk.
 * Operating range of the fused kernel:
 *   - the initial state and v: any finite values.  The state is stored with a power-of-two
 *     scale per value column (each column of S evolves independently and linearly), so no
 *     fp16 operand derived from it can overflow;
 *   - q, k and beta: |q|, |k|, |beta * k| elementwise and |q_r . k_i| below 2^15, which
 *     L2-normalised q and k with beta <= 1 satisfy with a wide margin.
 * An input outside that range is not an error before the launch: the kernel saturates the
 * affected fp16 operands (never inf or NaN), records KDA_DEVERR_RANGE in the device error word
 * and the output is then not guaranteed; kda_fwd_staged computes such inputs in fp32.
 *
 * One long sequence with few heads (fixed layout, batch 1, when kda_fwd_segments() > 1): the fused
 * kernel runs one CTA per (sequence, head), so such a call would leave most SMs idle.  kda_fwd then
 * splits the sequence into R chunk-aligned segments and runs them together: every segment's affine
 * state map (from S = I with v = 0, and from S = 0), their fold into each segment's starting state
 * (S_r = A_{r-1} S_{r-1} + B_{r-1}, kda_state_affine), and every segment from its state.  The result
 * is the same recurrence (up to rounding); the call allocates 3 R H 64 KiB of workspace
 * stream-ordered and launches R + 3 kernels.
 *
 * lower_bound: <= 0 (may be -INFINITY: no clamp); NaN or > 0 is rejected.
 * scale: finite.  Returns KDA_OK or an error code; never aborts.
 */
kda_status kda_fwd(const void* q, const void* k, const void* v,
                   const float* g, const float* beta,
                   const float* A_log, const float* dt_bias,
                   float lower_bound, float scale,
                   const float* initial_state, const int32_t* cu_seqlens,
                   void* out, float* final_state,
                   kda_dims dims, kda_stream_t stream);

/* The number of segments kda_fwd and kda_gdn_fwd split a call with these dims into on the current
 * device (1: none).  Only one sequence in the fixed layout (varlen == 0, batch == 1) of at least
 * 8192 tokens is split; the count minimises an estimate of three passes over R H units against
 * one pass over H units. */
int32_t kda_fwd_segments(kda_dims dims, int32_t varlen);

/* Gates at or above this clamp keep every factored intra-chunk decay of the fused kernel inside
 * the fp32/bf16 exponent range: its factors span at most 8 tokens of decay around the middle of a
 * 16-token block, e^{8 x 9.5} = e^76, and |k| e^76 < 3.4e38 for |k| < 2^15. */
#define KDA_FUSED_MIN_LOWER_BOUND (-9.5f)

/*
 * kda_fwd_staged -- the same forward as four separate kernels with intermediates in a
 * caller-provided workspace:
 *   (a) gate pre-pass: Gamma = in-chunk inclusive cumsum of log a;
 *   (b) intra-chunk WY: A, T = (I + A)^-1, W = T diag(beta)(gamma*K), U~ = T diag(beta) V, P;
 *   (c) state propagation: U = U~ - W S_c, S_{c+1} = Diag(gamma_C) S_c + Khat^T U;
 *   (d) output: O = scale ((gamma*Q) S_c + P U).
 * (a), (b) and (d) are fp32 CUDA-core kernels, every intra-chunk decay formed pair by pair (exact
 * for any gate).  (c) runs on the tensor cores with the state in fp32 and bf16 high + low operand
 * parts (about 16 mantissa bits per product).
 * Chunks are 64 tokens, restarting at every sequence start.
 * workspace: device buffer of at least kda_staged_workspace_size(dims) bytes,
 * 256-byte aligned.  Its layout (offsets from kda_staged_workspace_layout) is
 * part of the ABI so that tests can read each stage's output.
 */
size_t kda_staged_workspace_size(kda_dims dims, int varlen);

typedef struct {
    size_t chunk_table;   /* int32 [max_chunks][4]: seq, t0, len, chunk index in seq; then int32 count */
    size_t gamma;         /* fp32 [Ttot, H, 128]  Gamma (in-chunk inclusive cumsum of log a) */
    size_t w;             /* fp32 [Ttot, H, 128]  W */
    size_t u_tilde;       /* fp32 [Ttot, H, 128]  U~ */
    size_t p;             /* fp32 [Ttot, H, 64]   row r of the token's chunk P (columns past r are 0) */
    size_t u;             /* fp32 [Ttot, H, 128]  U */
    size_t chunk_states;  /* fp32 [max_chunks, H, 128, 128]  state at each chunk's start */
    size_t total;         /* bytes */
    int64_t max_chunks;   /* ceil(Ttot / 64) + N */
} kda_staged_layout;

/* Bytes of workspace kda_fwd_staged needs for `dims`, whichever layout the call uses: the
 * larger of the varlen reading (N = num_seqs, Ttot = seqlen) and the fixed one (N = batch,
 * Ttot = batch * seqlen).  kda_fwd itself takes no workspace (its staged fallback and its
 * split of one long sequence allocate stream-ordered).  0 for invalid dims. */
size_t kda_fwd_workspace_size(kda_dims dims);

/* varlen != 0: the call passes cu_seqlens (N = num_seqs, Ttot = seqlen);
 * varlen == 0: fixed layout (N = batch, Ttot = batch * seqlen). */
kda_status kda_staged_workspace_layout(kda_dims dims, int varlen, kda_staged_layout* layout);

kda_status kda_fwd_staged(const void* q, const void* k, const void* v,
                          const float* g, const float* beta,
                          const float* A_log, const float* dt_bias,
                          float lower_bound, float scale,
                          const float* initial_state, const int32_t* cu_seqlens,
                          void* out, float* final_state,
                          kda_dims dims, void* workspace, size_t workspace_bytes,
                          kda_stream_t stream);

/*
 * kda_fwd_staged_noalloc -- the staged forward (same kernels and results as
 * kda_fwd_staged) without any device allocation.  No page describes this entry
 * point; it exists for callers that cannot allocate device memory: callers
 * whose device memory is entirely owned by another allocator (a framework's
 * caching allocator, a pre-reserved arena), where cudaMalloc would fail or
 * fragment that pool, and latency-critical callers that must not enter the
 * driver's allocator.
 *
 * Scratch: a fixed 16 MiB array in device global memory (see
 * kda_noalloc_scratch_bytes), present on every GPU that loads the library
 * until the process exits.  The call neither allocates nor frees anything.
 * Limit: problems whose staged workspace (kda_staged_workspace_size) exceeds
 * the scratch are rejected with KDA_ERR_SCRATCH_LIMIT before any launch
 * (roughly T * H <= 4500 tokens x heads at N = 1).
 * Set-up: the first call on each device resolves the scratch's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before capturing a stream.
 * Sharing: all calls share the one scratch, which keeps the last call's
 * contents (nothing in it needs to start at zero).  Calls that overlap on the
 * GPU -- on different streams or from different host threads -- race on it;
 * serialise them.
 * Arguments, layouts and other errors are those of kda_fwd.
 */
kda_status kda_fwd_staged_noalloc(const void* q, const void* k, const void* v,
                                  const float* g, const float* beta,
                                  const float* A_log, const float* dt_bias,
                                  float lower_bound, float scale,
                                  const float* initial_state, const int32_t* cu_seqlens,
                                  void* out, float* final_state,
                                  kda_dims dims, kda_stream_t stream);

/* Size in bytes of the scratch kda_fwd_staged_noalloc uses (16 MiB). */
size_t kda_noalloc_scratch_bytes(void);

/*
 * kda_decode -- one recurrent step (decode) per sequence, in place on the state.
 * The token-by-token form of the same KDA recurrence; the FlashKDA post
 * (donniechu.com, sections "Hạn chế & điều kiện" and "What's next") lists
 * decode as not yet tuned and a decode kernel as future work of that release.
 *   q, k, v  bf16 [batch, H, 128]     g fp32 [batch, H, 128]     beta fp32 [batch, H]
 *   A_log fp32 [H], dt_bias fp32 [H, 128]
 *   state    fp32 [batch, H, 128, 128] ([k][v]); read and overwritten with the new state
 *   out      bf16 [batch, H, 128] = scale * S_new^T q
 * Errors as for kda_fwd (checked before the launch); out must not overlap any
 * input or the state.  Asynchronous on `stream`.
 */
kda_status kda_decode(const void* q, const void* k, const void* v,
                      const float* g, const float* beta,
                      const float* A_log, const float* dt_bias,
                      float lower_bound, float scale,
                      float* state, void* out,
                      int32_t batch, int32_t num_heads, kda_stream_t stream);

/*
 * kda_gdn_decode -- one decode step of the scalar-gate variant: as kda_decode, with
 * g fp32 [batch, H] and dt_bias fp32 [H] (one decay per sequence and head).
 */
kda_status kda_gdn_decode(const void* q, const void* k, const void* v,
                          const float* g, const float* beta,
                          const float* A_log, const float* dt_bias,
                          float lower_bound, float scale,
                          float* state, void* out,
                          int32_t batch, int32_t num_heads, kda_stream_t stream);

/*
 * kda_gdn_fwd -- the scalar-gate variant (Gated DeltaNet): the same recurrence with
 * one decay per (token, head) instead of one per key channel,
 *   log a_t = max(-exp(A_log_h) * softplus(g_t,h + dt_bias_h), lower_bound),
 * applied to every channel of the state.  The FlashKDA H20 benchmark table
 * (toolarium.ru, section "Что показывают H20-бенчмарки") compares against such a
 * "gdn" kernel in its second column.
 *   q, k, v, out, initial_state, final_state, cu_seqlens, dims: as for kda_fwd
 *   g        fp32 [B*T, H]   (one gate input per token and head)
 *   beta     fp32 [B*T, H]
 *   A_log    fp32 [H],  dt_bias fp32 [H]
 * Any lower_bound <= 0 is accepted (the intra-chunk decays are formed pairwise).
 * Errors, alignment, aliasing and asynchrony as for kda_fwd.
 */
kda_status kda_gdn_fwd(const void* q, const void* k, const void* v,
                       const float* g, const float* beta,
                       const float* A_log, const float* dt_bias,
                       float lower_bound, float scale,
                       const float* initial_state, const int32_t* cu_seqlens,
                       void* out, float* final_state,
                       kda_dims dims, kda_stream_t stream);

/*
 * kda_state_affine -- one step of the context-parallel state fold:
 *   out[h] = A[h] S[h] + B[h]   for h < num_heads, all fp32 [num_heads][128][128] ([k][v]).
 * The forward is affine in the state a segment starts from.  For a segment, A is its final
 * state from initial state I with v = 0, and B its final state from initial state 0.  So
 * when one long sequence is split into segments (one per rank, for the 128k-1M contexts the
 * FlashKDA posts target: donniechu.com, "Số liệu kỹ thuật"), segment r starts from
 * S_r = A_{r-1} S_{r-1} + B_{r-1}.  out may alias B but not A or S.  Errors as for kda_fwd.
 */
kda_status kda_state_affine(const float* A, const float* S, const float* B, float* out,
                            int32_t num_heads, kda_stream_t stream);

/*
 * kda_bwd -- the backward of kda_fwd: gradients of the scalar
 *   L = <d_out, out> + <d_final_state, final_state>
 * with respect to every input of the forward.  The pages describe the forward only (the
 * FlashKDA posts: donniechu.com, "Hạn chế & điều kiện" -- the release targets prefill); the
 * backward is the chain rule taken through the same chunked form (WY / UT representation
 * of each 64-token chunk and the chunk-to-chunk state recurrence), stage by stage:
 *   (1) the staged forward into the workspace (Gamma, W, P, U, the state at every chunk start);
 *   (2) dS backwards over each sequence's chunks, storing dS' per chunk and dU;
 *   (3) per chunk: dKhat, d(gamma q), dW and d gamma_C from U, dU, dO, S, dS';
 *   (4) per chunk: T = (I + A)^-1 recomputed; dT, dA, dv and the T-side dk, dGamma, dbeta;
 *   (5) per chunk: dP and the pairwise decay terms (products of a, never exponentials of
 *       differences), dq, dk, dbeta, then d log a (dGamma summed from the chunk's end) and
 *       the gate's chain rule (zero where the lower_bound clamp is active);
 *   (6) dA_log and ddt_bias summed over chunks in a fixed order (deterministic).
 * Stages (2), (3) and the state propagation of (1) run on the tensor cores with fp32
 * accumulation and bf16 high + low operand parts (about 16 mantissa bits per product); the
 * rest is fp32 CUDA-core arithmetic.  No atomics, so results are bitwise reproducible.
 *
 * Inputs q ... cu_seqlens, lower_bound, scale, dims: exactly those of the kda_fwd call.
 *   d_out          bf16 [Ttot, H, 128]       gradient of out
 *   d_final_state  fp32 [N, H, 128, 128]     gradient of final_state; NULL means zero
 * Outputs (device, caller-owned, written in full; none may overlap an input or another):
 *   dq, dk, dv, dg fp32 [Ttot, H, 128]       dbeta fp32 [Ttot, H]
 *   dA_log         fp32 [H]                  ddt_bias fp32 [H, 128]
 *   d_initial_state fp32 [N, H, 128, 128]    NULL means "do not write"; may alias
 *                                            d_final_state exactly (in place)
 * workspace: at least kda_bwd_workspace_size(dims, varlen) bytes, 256-byte aligned; or
 * NULL with workspace_bytes = 0, and the call allocates it stream-ordered
 * (cudaMallocAsync / cudaFreeAsync).  Alignment as for kda_fwd: 16 bytes, except beta and
 * dbeta (4 bytes).  Errors are reported before any launch.  Asynchronous on `stream`.
 */
typedef struct {
    float* dq;
    float* dk;
    float* dv;
    float* dg;
    float* dbeta;
    float* dA_log;
    float* ddt_bias;
    float* d_initial_state;
} kda_grads;

size_t kda_bwd_workspace_size(kda_dims dims, int varlen);

kda_status kda_bwd(const void* q, const void* k, const void* v,
                   const float* g, const float* beta,
                   const float* A_log, const float* dt_bias,
                   float lower_bound, float scale,
                   const float* initial_state, const int32_t* cu_seqlens,
                   const void* d_out, const float* d_final_state,
                   const kda_grads* grads,
                   kda_dims dims, void* workspace, size_t workspace_bytes,
                   kda_stream_t stream);

/*
 * kda_selftest_wait_timeout -- diagnostics: exercises the recovery path of the library's bounded
 * waits without any fault.  No page has a counterpart; every kernel here waits on mbarriers with a
 * wall-clock limit, and this entry point makes one such wait run out on purpose.  It launches one
 * CTA that allocates tensor memory, starts one tensor-core MMA, then waits (at most limit_ns
 * nanoseconds) on an mbarrier that nothing arrives at.  As in the product kernels, the expired
 * wait records KDA_DEVERR_TIMEOUT, the CTA waits (bounded) for its own MMA, frees its tensor
 * memory and returns; the device stays usable.
 *   limit_ns   in [1, 1e9]
 *   observed   NULL, or device uint32 [2]: [0] = 1 if the wait ran out, [1] = 1 if the MMA had
 *              completed before the tensor memory was freed
 * Asynchronous on `stream`; read the result with kda_check_device_error.
 */
kda_status kda_selftest_wait_timeout(uint64_t limit_ns, uint32_t* observed, kda_stream_t stream);

/* Human-readable name of a status code (static storage; never NULL). */
const char* kda_strerror(kda_status status);

/* Synchronises `stream`, then reads and clears the device error word.
 * Returns KDA_OK, KDA_ERR_DEVICE (bits available from kda_last_device_error_bits)
 * or KDA_ERR_CUDA.  Not capturable (it synchronises). */
kda_status kda_check_device_error(kda_stream_t stream);
uint32_t kda_last_device_error_bits(void);

/* Library version, "major.minor.patch". */
const char* kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H */
