// kda_api.cu -- the C ABI (include/kda.h): argument validation, dispatch and
// the device error word.  This is the library's single translation unit: the
// kernels are included below so that they share the error word without
// relocatable device code.

#include <math.h>
#include <string.h>


#include "kda_common.cuh"
#include "kda_internal.h"

#include "kda_staged.cuh"
#include "kda_pipe.cuh"
#include "kda_decode.cuh"
#include "kda_cp.cuh"
#include "kda_backward.cuh"
#include "kda_selftest.cuh"

namespace {

using kda::StagedArgs;

thread_local uint32_t t_last_device_bits = 0;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

bool overlaps(const void* a, size_t an, const void* b, size_t bn) {
    if (!a || !b || an == 0 || bn == 0) return false;
    uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + bn && b0 < a0 + an;
}

kda_status device_ok() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return KDA_ERR_CUDA;
    return major == 10 ? KDA_OK : KDA_ERR_UNSUPPORTED;
}

// Validates arguments and fills the kernel argument block.  g_per_head is the number of
// gate values per (token, head): 128 (one per key channel) or 1 (the scalar-gate variant).
kda_status prepare(const void* q, const void* k, const void* v, const float* g, const float* beta,
                   const float* A_log, const float* dt_bias, float lower_bound, float scale,
                   const float* initial_state, const int32_t* cu_seqlens, void* out,
                   float* final_state, const kda_dims& d, StagedArgs* a, size_t g_per_head = kda::kHeadDim,
                   bool check_device = true) {
    if (d.head_dim_k != kda::kHeadDim || d.head_dim_v != kda::kHeadDim) return KDA_ERR_UNSUPPORTED;
    if (d.num_heads < 1 || d.seqlen < 0) return KDA_ERR_INVALID_ARG;
    if (isnan(lower_bound) || lower_bound > 0.f) return KDA_ERR_INVALID_ARG;
    if (!isfinite(scale)) return KDA_ERR_INVALID_ARG;
    int64_t N, total;
    if (cu_seqlens) {
        if (d.batch != 1 || d.num_seqs < 0) return KDA_ERR_INVALID_ARG;
        N = d.num_seqs;
        total = d.seqlen;
    } else {
        if (d.batch < 0) return KDA_ERR_INVALID_ARG;
        N = d.batch;
        total = (int64_t)d.batch * d.seqlen;
    }
    if (total >= ((int64_t)1 << 31) || N >= ((int64_t)1 << 30)) return KDA_ERR_INVALID_ARG;
    const int64_t H = d.num_heads;
    if (total > 0 && (!q || !k || !v || !g || !beta || !out)) return KDA_ERR_INVALID_ARG;
    if (!A_log || !dt_bias) return KDA_ERR_INVALID_ARG;
    // TMA-loaded and vector-accessed arrays need 16-byte bases; beta (and the scalar-gate
    // g) are read one element at a time, so 4 bytes suffice and token-offset slices work
    const void* ptrs[] = {q, k, v, g_per_head > 1 ? (const void*)g : nullptr, A_log, dt_bias, initial_state,
                          cu_seqlens, out, final_state};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_ALIGNMENT;
    if ((beta && !aligned4(beta)) || (g_per_head == 1 && g && !aligned4(g))) return KDA_ERR_ALIGNMENT;
    const size_t tok = (size_t)total * (size_t)H;
    const size_t out_bytes = tok * kda::kHeadDim * 2;
    const size_t st_bytes = (size_t)N * H * kda::kHeadDim * kda::kHeadDim * 4;
    if (overlaps(out, out_bytes, q, out_bytes) || overlaps(out, out_bytes, k, out_bytes) ||
        overlaps(out, out_bytes, v, out_bytes) || overlaps(out, out_bytes, g, tok * g_per_head * 4) ||
        overlaps(out, out_bytes, beta, tok * 4) || overlaps(out, out_bytes, initial_state, st_bytes) ||
        overlaps(out, out_bytes, final_state, st_bytes))
        return KDA_ERR_INVALID_ARG;
    if (final_state && initial_state && final_state != initial_state &&
        overlaps(final_state, st_bytes, initial_state, st_bytes))
        return KDA_ERR_INVALID_ARG;
    a->q = q; a->k = k; a->v = v; a->g = g; a->beta = beta; a->A_log = A_log; a->dt_bias = dt_bias;
    a->lower_bound = lower_bound; a->scale = scale;
    a->initial_state = initial_state; a->cu_seqlens = cu_seqlens;
    a->out = out; a->final_state = final_state;
    a->seqlen = d.seqlen; a->total_tokens = total; a->H = (int)H; a->N = (int)N;
    return check_device ? device_ok() : KDA_OK;
}

// Carries the initial state to the final state when no token is processed.
kda_status copy_states_only(const StagedArgs& a, cudaStream_t s) {
    if (!a.final_state || a.N == 0) return KDA_OK;
    const size_t bytes = (size_t)a.N * a.H * kda::kHeadDim * kda::kHeadDim * 4;
    cudaError_t err = a.initial_state
        ? (a.initial_state == a.final_state ? cudaSuccess
           : cudaMemcpyAsync(a.final_state, a.initial_state, bytes, cudaMemcpyDeviceToDevice, s))
        : cudaMemsetAsync(a.final_state, 0, bytes, s);
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // namespace

// ---------------------------------------------------------------------------
// kda_fwd_staged_noalloc: the staged forward on a library-owned scratch buffer.
//
// For callers that cannot allocate device memory: code whose device memory is
// entirely owned by another allocator (a framework's caching allocator or a
// pre-reserved arena, so that cudaMalloc fails or would fragment it) and code
// on latency-critical paths that must not enter the driver's allocator.  The
// scratch is a fixed array in device global memory that exists on every GPU
// that loads this library, from load until process exit.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch in the current context, looked up on every call (host code
// may not use the array's name as a device address).  Nothing is cached, so a context created
// after cudaDeviceReset gets its own array's address.
cudaError_t noalloc_scratch(void** out) {
    void* ptr = nullptr;
    const cudaError_t err = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (err != cudaSuccess) return err;
    *out = ptr;
    return cudaSuccess;
}

}  // namespace

extern "C" {

size_t kda_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

kda_status kda_fwd_staged_noalloc(const void* q, const void* k, const void* v, const float* g,
                                  const float* beta, const float* A_log, const float* dt_bias,
                                  float lower_bound, float scale, const float* initial_state,
                                  const int32_t* cu_seqlens, void* out, float* final_state,
                                  kda_dims dims, kda_stream_t stream) {
    StagedArgs a{};
    kda_status st = prepare(q, k, v, g, beta, A_log, dt_bias, lower_bound, scale, initial_state,
                            cu_seqlens, out, final_state, dims, &a);
    if (st != KDA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (a.total_tokens == 0) return copy_states_only(a, s);
    const kda::StagedLayout L = kda::staged_layout(a.total_tokens, a.H, a.N);
    if (L.total > kNoAllocScratchBytes) return KDA_ERR_SCRATCH_LIMIT;
    void* ws = nullptr;
    if (noalloc_scratch(&ws) != cudaSuccess) return KDA_ERR_CUDA;
    // Every byte the staged kernels read is written earlier in the same call
    // (chunk table, Gamma, W, U~, P, U, chunk states), so nothing is cleared.
    return kda::launch_staged(a, static_cast<char*>(ws), L, s) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}


kda_status kda_staged_workspace_layout(kda_dims dims, int varlen, kda_staged_layout* layout) {
    if (!layout) return KDA_ERR_INVALID_ARG;
    if (dims.num_heads < 1 || dims.seqlen < 0 || dims.batch < 0 || dims.num_seqs < 0)
        return KDA_ERR_INVALID_ARG;
    int64_t N = dims.num_seqs, total = dims.seqlen;
    if (!varlen) {
        N = dims.batch;
        total = (int64_t)dims.batch * dims.seqlen;
    }
    kda::StagedLayout L = kda::staged_layout(total, dims.num_heads, (int)N);
    layout->chunk_table = L.chunk_table;
    layout->gamma = L.gamma;
    layout->w = L.w;
    layout->u_tilde = L.u_tilde;
    layout->p = L.p;
    layout->u = L.u;
    layout->chunk_states = L.chunk_states;
    layout->total = L.total;
    layout->max_chunks = L.max_chunks;
    return KDA_OK;
}

size_t kda_staged_workspace_size(kda_dims dims, int varlen) {
    kda_staged_layout L;
    return kda_staged_workspace_layout(dims, varlen, &L) == KDA_OK ? L.total : 0;
}

size_t kda_fwd_workspace_size(kda_dims dims) {
    const size_t a = kda_staged_workspace_size(dims, 1), b = kda_staged_workspace_size(dims, 0);
    return a > b ? a : b;
}

kda_status kda_fwd_staged(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, const float* A_log, const float* dt_bias,
                          float lower_bound, float scale, const float* initial_state,
                          const int32_t* cu_seqlens, void* out, float* final_state, kda_dims dims,
                          void* workspace, size_t workspace_bytes, kda_stream_t stream) {
    StagedArgs a{};
    kda_status st = prepare(q, k, v, g, beta, A_log, dt_bias, lower_bound, scale, initial_state,
                            cu_seqlens, out, final_state, dims, &a);
    if (st != KDA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (a.total_tokens == 0) return copy_states_only(a, s);
    kda::StagedLayout L = kda::staged_layout(a.total_tokens, a.H, a.N);
    if (!workspace || workspace_bytes < L.total) return KDA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KDA_ERR_ALIGNMENT;
    return kda::launch_staged(a, static_cast<char*>(workspace), L, s) == cudaSuccess ? KDA_OK
                                                                                     : KDA_ERR_CUDA;
}

namespace {

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

// Segments for a fused-forward call: one sequence in the fixed layout (its boundaries are known
// on the host) whose heads leave SMs idle.
int segments_for(const StagedArgs& a, bool varlen) {
    if (varlen || a.N != 1) return 1;
    return kda::choose_segments(a.total_tokens, a.H, sm_count());
}

// One long sequence as R segments run together (the context-parallel decomposition on one GPU):
// (1) every segment from S = I with v = 0 gives its A map, (2) from S = 0 its B map, (3) the
// maps fold into each segment's starting state, S_r = A_{r-1} S_{r-1} + B_{r-1}, and (4) every
// segment runs from its state and writes the output.  Workspace (stream-ordered): the segment
// offsets and three [R][H][128][128] fp32 state arrays.
cudaError_t launch_segmented(const StagedArgs& a, int R, bool gdn, cudaStream_t s) {
    auto fused = [&](const StagedArgs& x) { return gdn ? kda::launch_pipe_gdn(x, s) : kda::launch_pipe(x, s); };
    const int64_t T = a.total_tokens;
    const size_t per_seg = (size_t)a.H * kda::kHeadDim * kda::kHeadDim;   // floats
    const size_t map_bytes = (size_t)R * per_seg * sizeof(float);
    char* ws = nullptr;
    cudaError_t err = cudaMallocAsync(reinterpret_cast<void**>(&ws), 256 + 3 * map_bytes, s);
    if (err != cudaSuccess) return err;
    int32_t* cu = reinterpret_cast<int32_t*>(ws);
    float* A = reinterpret_cast<float*>(ws + 256);
    float* B = A + (size_t)R * per_seg;
    float* S = B + (size_t)R * per_seg;
    kda::cp::segment_offsets_kernel<<<1, 64, 0, s>>>(cu, R, kda::cp::segment_step(T, R), T);
    err = cudaGetLastError();
    StagedArgs m = a;
    m.cu_seqlens = cu;
    m.N = R;
    m.seqlen = T;
    m.out = nullptr;
    m.initial_state = nullptr;
    if (err == cudaSuccess) {   // A maps
        m.flags = kda::kFlagVZero | kda::kFlagInitIdentity;
        m.final_state = A;
        err = fused(m);
    }
    if (err == cudaSuccess) {   // B maps
        m.flags = 0;
        m.final_state = B;
        err = fused(m);
    }
    const size_t st_bytes = per_seg * sizeof(float);
    if (err == cudaSuccess)
        err = a.initial_state ? cudaMemcpyAsync(S, a.initial_state, st_bytes, cudaMemcpyDeviceToDevice, s)
                              : cudaMemsetAsync(S, 0, st_bytes, s);
    for (int r = 1; r < R && err == cudaSuccess; ++r)
        err = kda::launch_state_affine(A + (size_t)(r - 1) * per_seg, S + (size_t)(r - 1) * per_seg,
                                       B + (size_t)(r - 1) * per_seg, S + (size_t)r * per_seg, a.H, s);
    if (err == cudaSuccess) {   // every segment from its state; its final states over the B maps
        StagedArgs f = a;
        f.cu_seqlens = cu;
        f.N = R;
        f.seqlen = T;
        f.initial_state = S;
        f.final_state = B;
        err = fused(f);
    }
    if (err == cudaSuccess && a.final_state)
        err = cudaMemcpyAsync(a.final_state, B + (size_t)(R - 1) * per_seg, st_bytes, cudaMemcpyDeviceToDevice, s);
    const cudaError_t err2 = cudaFreeAsync(ws, s);
    return err != cudaSuccess ? err : err2;
}

}  // namespace

int32_t kda_fwd_segments(kda_dims dims, int32_t varlen) {
    if (dims.num_heads < 1 || dims.seqlen < 0) return 1;
    if (varlen || dims.batch != 1) return 1;
    return kda::choose_segments(dims.seqlen, dims.num_heads, sm_count());
}

kda_status kda_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                   const float* A_log, const float* dt_bias, float lower_bound, float scale,
                   const float* initial_state, const int32_t* cu_seqlens, void* out,
                   float* final_state, kda_dims dims, kda_stream_t stream) {
    StagedArgs a{};
    kda_status st = prepare(q, k, v, g, beta, A_log, dt_bias, lower_bound, scale, initial_state,
                            cu_seqlens, out, final_state, dims, &a);
    if (st != KDA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (a.total_tokens == 0) return copy_states_only(a, s);
    if (kda::fused_supported(lower_bound)) {
        const int R = segments_for(a, cu_seqlens != nullptr);
        const cudaError_t err = R > 1 ? launch_segmented(a, R, false, s) : kda::launch_pipe(a, s);
        return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }
    kda::StagedLayout L = kda::staged_layout(a.total_tokens, a.H, a.N);
    void* ws = nullptr;
    if (cudaMallocAsync(&ws, L.total, s) != cudaSuccess) return KDA_ERR_CUDA;
    cudaError_t err = kda::launch_staged(a, static_cast<char*>(ws), L, s);
    cudaError_t err2 = cudaFreeAsync(ws, s);
    return (err == cudaSuccess && err2 == cudaSuccess) ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_gdn_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                       const float* A_log, const float* dt_bias, float lower_bound, float scale,
                       const float* initial_state, const int32_t* cu_seqlens, void* out,
                       float* final_state, kda_dims dims, kda_stream_t stream) {
    StagedArgs a{};
    kda_status st = prepare(q, k, v, g, beta, A_log, dt_bias, lower_bound, scale, initial_state,
                            cu_seqlens, out, final_state, dims, &a, 1);
    if (st != KDA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (a.total_tokens == 0) return copy_states_only(a, s);
    const int R = segments_for(a, cu_seqlens != nullptr);
    const cudaError_t err = R > 1 ? launch_segmented(a, R, true, s) : kda::launch_pipe_gdn(a, s);
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

namespace {

struct Span {
    const void* p;
    size_t n;
};

// Validates the backward's arguments: the forward's (with d_out in the place of out) and the
// gradient outputs, which must be aligned and overlap neither an input nor one another.
kda_status prepare_bwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                       const float* A_log, const float* dt_bias, float lower_bound, float scale,
                       const float* initial_state, const int32_t* cu_seqlens, const void* d_out,
                       const float* d_final, const kda_grads* gr, const kda_dims& d, StagedArgs* a,
                       kda::BwdArgs* b) {
    if (!gr) return KDA_ERR_INVALID_ARG;
    kda_status st = prepare(q, k, v, g, beta, A_log, dt_bias, lower_bound, scale, initial_state, cu_seqlens,
                            const_cast<void*>(d_out), nullptr, d, a, kda::kHeadDim, false);
    if (st != KDA_OK) return st;
    const size_t tok = (size_t)a->total_tokens * a->H, D = kda::kHeadDim;
    const size_t st_bytes = (size_t)a->N * a->H * D * D * 4;
    if (tok > 0 && (!gr->dq || !gr->dk || !gr->dv || !gr->dg || !gr->dbeta)) return KDA_ERR_INVALID_ARG;
    if (!gr->dA_log || !gr->ddt_bias) return KDA_ERR_INVALID_ARG;
    const void* a16[] = {gr->dq, gr->dk, gr->dv, gr->dg, gr->dA_log, gr->ddt_bias, gr->d_initial_state, d_final};
    for (const void* p : a16)
        if (p && !aligned16(p)) return KDA_ERR_ALIGNMENT;
    if (gr->dbeta && !aligned4(gr->dbeta)) return KDA_ERR_ALIGNMENT;
    const Span outs[] = {{gr->dq, tok * D * 4}, {gr->dk, tok * D * 4}, {gr->dv, tok * D * 4},
                         {gr->dg, tok * D * 4}, {gr->dbeta, tok * 4}, {gr->dA_log, (size_t)a->H * 4},
                         {gr->ddt_bias, (size_t)a->H * D * 4}, {gr->d_initial_state, st_bytes}};
    const Span ins[] = {{q, tok * D * 2}, {k, tok * D * 2}, {v, tok * D * 2}, {g, tok * D * 4},
                        {beta, tok * 4}, {A_log, (size_t)a->H * 4}, {dt_bias, (size_t)a->H * D * 4},
                        {initial_state, st_bytes}, {cu_seqlens, cu_seqlens ? ((size_t)a->N + 1) * 4 : 0},
                        {d_out, tok * D * 2}};
    const int n_out = sizeof(outs) / sizeof(outs[0]);
    for (int i = 0; i < n_out; ++i) {
        for (const Span& in : ins)
            if (overlaps(outs[i].p, outs[i].n, in.p, in.n)) return KDA_ERR_INVALID_ARG;
        for (int j = i + 1; j < n_out; ++j)
            if (overlaps(outs[i].p, outs[i].n, outs[j].p, outs[j].n)) return KDA_ERR_INVALID_ARG;
    }
    // d_initial_state may alias d_final_state exactly, not partially
    if (gr->d_initial_state && d_final && (const void*)gr->d_initial_state != (const void*)d_final &&
        overlaps(gr->d_initial_state, st_bytes, d_final, st_bytes))
        return KDA_ERR_INVALID_ARG;
    for (int i = 0; i < n_out - 1; ++i)
        if (overlaps(outs[i].p, outs[i].n, d_final, st_bytes)) return KDA_ERR_INVALID_ARG;
    a->out = nullptr;
    b->d_out = d_out;
    b->d_final = d_final;
    b->dq = gr->dq; b->dk = gr->dk; b->dv = gr->dv; b->dg = gr->dg; b->dbeta = gr->dbeta;
    b->dA_log = gr->dA_log; b->ddt_bias = gr->ddt_bias; b->d_initial = gr->d_initial_state;
    return device_ok();
}

// With no token to process: the parameter gradients are zero and d_initial = d_final.
kda_status bwd_no_tokens(const StagedArgs& a, const kda::BwdArgs& b, cudaStream_t s) {
    const size_t D = kda::kHeadDim;
    if (cudaMemsetAsync(b.dA_log, 0, (size_t)a.H * 4, s) != cudaSuccess) return KDA_ERR_CUDA;
    if (cudaMemsetAsync(b.ddt_bias, 0, (size_t)a.H * D * 4, s) != cudaSuccess) return KDA_ERR_CUDA;
    if (!b.d_initial || a.N == 0) return KDA_OK;
    const size_t bytes = (size_t)a.N * a.H * D * D * 4;
    cudaError_t err = b.d_final
        ? ((const void*)b.d_final == (const void*)b.d_initial ? cudaSuccess
           : cudaMemcpyAsync(b.d_initial, b.d_final, bytes, cudaMemcpyDeviceToDevice, s))
        : cudaMemsetAsync(b.d_initial, 0, bytes, s);
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status decode_common(const void* q, const void* k, const void* v, const float* g, const float* beta,
                         const float* A_log, const float* dt_bias, float lower_bound, float scale,
                         float* state, void* out, int32_t batch, int32_t num_heads, kda_stream_t stream,
                         bool scalar_gate) {
    if (batch < 0 || num_heads < 1) return KDA_ERR_INVALID_ARG;
    if (isnan(lower_bound) || lower_bound > 0.f || !isfinite(scale)) return KDA_ERR_INVALID_ARG;
    if (batch == 0) return KDA_OK;
    if (!q || !k || !v || !g || !beta || !A_log || !dt_bias || !state || !out) return KDA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, g, beta, A_log, dt_bias, state, out};
    for (const void* p : ptrs)
        if (!aligned16(p)) return KDA_ERR_ALIGNMENT;
    const size_t bh = (size_t)batch * num_heads;
    const size_t ob = bh * kda::kHeadDim * 2;
    if (overlaps(out, ob, q, ob) || overlaps(out, ob, k, ob) || overlaps(out, ob, v, ob) ||
        overlaps(out, ob, g, bh * (scalar_gate ? 1 : kda::kHeadDim) * 4) || overlaps(out, ob, beta, bh * 4) ||
        overlaps(out, ob, state, bh * kda::kHeadDim * kda::kHeadDim * 4))
        return KDA_ERR_INVALID_ARG;
    kda_status st = device_ok();
    if (st != KDA_OK) return st;
    return kda::launch_decode(q, k, v, g, beta, A_log, dt_bias, lower_bound, scale, state, out, batch,
                              num_heads, reinterpret_cast<cudaStream_t>(stream), scalar_gate) == cudaSuccess
               ? KDA_OK : KDA_ERR_CUDA;
}

}  // namespace

kda_status kda_decode(const void* q, const void* k, const void* v, const float* g, const float* beta,
                      const float* A_log, const float* dt_bias, float lower_bound, float scale,
                      float* state, void* out, int32_t batch, int32_t num_heads, kda_stream_t stream) {
    return decode_common(q, k, v, g, beta, A_log, dt_bias, lower_bound, scale, state, out, batch, num_heads,
                         stream, false);
}

kda_status kda_state_affine(const float* A, const float* S, const float* B, float* out, int32_t num_heads,
                            kda_stream_t stream) {
    if (num_heads < 0) return KDA_ERR_INVALID_ARG;
    if (num_heads == 0) return KDA_OK;
    if (!A || !S || !B || !out) return KDA_ERR_INVALID_ARG;
    const void* ptrs[] = {A, S, B, out};
    for (const void* p : ptrs)
        if (!aligned16(p)) return KDA_ERR_ALIGNMENT;
    const size_t bytes = (size_t)num_heads * kda::kHeadDim * kda::kHeadDim * 4;
    if (overlaps(out, bytes, A, bytes) || overlaps(out, bytes, S, bytes)) return KDA_ERR_INVALID_ARG;
    kda_status st = device_ok();
    if (st != KDA_OK) return st;
    return kda::launch_state_affine(A, S, B, out, num_heads, reinterpret_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? KDA_OK
               : KDA_ERR_CUDA;
}

kda_status kda_gdn_decode(const void* q, const void* k, const void* v, const float* g, const float* beta,
                          const float* A_log, const float* dt_bias, float lower_bound, float scale,
                          float* state, void* out, int32_t batch, int32_t num_heads, kda_stream_t stream) {
    return decode_common(q, k, v, g, beta, A_log, dt_bias, lower_bound, scale, state, out, batch, num_heads,
                         stream, true);
}

size_t kda_bwd_workspace_size(kda_dims dims, int varlen) {
    if (dims.num_heads < 1 || dims.seqlen < 0 || dims.batch < 0 || dims.num_seqs < 0) return 0;
    int64_t N = dims.num_seqs, total = dims.seqlen;
    if (!varlen) {
        N = dims.batch;
        total = (int64_t)dims.batch * dims.seqlen;
    }
    return kda::bwd_layout(total, dims.num_heads, (int)N).total;
}

kda_status kda_bwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                   const float* A_log, const float* dt_bias, float lower_bound, float scale,
                   const float* initial_state, const int32_t* cu_seqlens, const void* d_out,
                   const float* d_final_state, const kda_grads* grads, kda_dims dims, void* workspace,
                   size_t workspace_bytes, kda_stream_t stream) {
    StagedArgs a{};
    kda::BwdArgs b{};
    kda_status st = prepare_bwd(q, k, v, g, beta, A_log, dt_bias, lower_bound, scale, initial_state,
                                cu_seqlens, d_out, d_final_state, grads, dims, &a, &b);
    if (st != KDA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (a.total_tokens == 0) return bwd_no_tokens(a, b, s);
    const kda::BwdLayout B = kda::bwd_layout(a.total_tokens, a.H, a.N);
    if (workspace) {
        if (workspace_bytes < B.total) return KDA_ERR_WORKSPACE;
        if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KDA_ERR_ALIGNMENT;
        return kda::launch_bwd(a, b, static_cast<char*>(workspace), B, s) == cudaSuccess ? KDA_OK
                                                                                       : KDA_ERR_CUDA;
    }
    if (workspace_bytes != 0) return KDA_ERR_WORKSPACE;
    void* ws = nullptr;
    if (cudaMallocAsync(&ws, B.total, s) != cudaSuccess) return KDA_ERR_CUDA;
    cudaError_t err = kda::launch_bwd(a, b, static_cast<char*>(ws), B, s);
    cudaError_t err2 = cudaFreeAsync(ws, s);
    return (err == cudaSuccess && err2 == cudaSuccess) ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_selftest_wait_timeout(uint64_t limit_ns, uint32_t* observed, kda_stream_t stream) {
    if (limit_ns < 1 || limit_ns > 1000000000ull) return KDA_ERR_INVALID_ARG;
    if (observed && !aligned4(observed)) return KDA_ERR_ALIGNMENT;
    kda_status st = device_ok();
    if (st != KDA_OK) return st;
    return kda::launch_wait_timeout_selftest(limit_ns, observed, reinterpret_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? KDA_OK
               : KDA_ERR_CUDA;
}

const char* kda_strerror(kda_status status) {
    switch (status) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG: invalid pointer, dimension or scalar";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: head dims must be 128 on an sm_100 device";
        case KDA_ERR_ALIGNMENT: return "KDA_ERR_ALIGNMENT: a base address is not 16-byte aligned";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA: a CUDA call or kernel launch failed";
        case KDA_ERR_DEVICE: return "KDA_ERR_DEVICE: a kernel recorded a device-side error";
        case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE: workspace missing or too small";
        case KDA_ERR_SCRATCH_LIMIT:
            return "KDA_ERR_SCRATCH_LIMIT: the problem needs more than the 16 MiB scratch of "
                   "kda_fwd_staged_noalloc (use kda_fwd_staged with a workspace)";
    }
    return "KDA_ERR_UNKNOWN";
}

kda_status kda_check_device_error(kda_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return KDA_ERR_CUDA;
    unsigned int bits = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&bits, kda::g_device_error, sizeof bits) != cudaSuccess) return KDA_ERR_CUDA;
    if (bits && cudaMemcpyToSymbol(kda::g_device_error, &zero, sizeof zero) != cudaSuccess)
        return KDA_ERR_CUDA;
    t_last_device_bits = bits;
    return bits ? KDA_ERR_DEVICE : KDA_OK;
}

uint32_t kda_last_device_error_bits(void) { return t_last_device_bits; }

const char* kda_version(void) { return "0.1.0"; }

}  // extern "C"
