// kda_internal.h -- host-side interfaces between the C ABI and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>

namespace kda {

// Runs `setup` (cudaFuncSetAttribute calls and the like) once for the current device: kernel
// attributes belong to a device, so a process that drives several GPUs needs them on each.
template <typename F>
cudaError_t once_per_device(F setup) {
    static std::mutex m;
    static uint64_t done = 0;   // bit d: device d is set up (devices past 63 always run setup)
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    std::lock_guard<std::mutex> lock(m);
    if (dev < 64 && (done >> dev) & 1u) return cudaSuccess;
    err = setup(dev);
    if (err == cudaSuccess && dev < 64) done |= uint64_t(1) << dev;
    return err;
}

// StagedArgs::flags of the fused forward (the segment maps of one long sequence)
constexpr uint32_t kFlagVZero = 1u;          // treat v as zero
constexpr uint32_t kFlagInitIdentity = 2u;   // start every sequence from S = I (initial_state NULL)

struct StagedArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* g;
    const float* beta;
    const float* A_log;
    const float* dt_bias;
    float lower_bound;
    float scale;
    const float* initial_state;
    const int32_t* cu_seqlens;
    void* out;
    float* final_state;
    int64_t seqlen;        // per-sequence length (fixed layout) or packed total
    int64_t total_tokens;  // Ttot
    int H;
    int N;                 // number of sequences
    float* t_mat;          // optional: T = (I + A)^-1 of every chunk, [max_chunks][H][64][64]
    uint32_t flags;        // fused forward only: kFlagVZero | kFlagInitIdentity; out may then be NULL
};

struct StagedLayout {
    size_t chunk_table, gamma, w, u_tilde, p, u, chunk_states, total;
    int64_t max_chunks;
};

StagedLayout staged_layout(int64_t total_tokens, int H, int N);
cudaError_t launch_staged(const StagedArgs& a, char* workspace, const StagedLayout& L,
                          cudaStream_t stream);

// The backward: gradients of <dO, out> + <dS_final, final_state>.
struct BwdArgs {
    const void* d_out;       // bf16 [Ttot, H, 128]
    const float* d_final;    // fp32 [N, H, 128, 128] or null (zero)
    float* dq;               // fp32 [Ttot, H, 128]
    float* dk;
    float* dv;
    float* dg;
    float* dbeta;            // fp32 [Ttot, H]
    float* dA_log;           // fp32 [H]
    float* ddt_bias;         // fp32 [H, 128]
    float* d_initial;        // fp32 [N, H, 128, 128] or null (not written)
};

// The staged forward's workspace followed by the backward's own buffers.
struct BwdLayout {
    StagedLayout fwd;
    size_t t_mat, dsn, du, dkhat, dqg, dw, dG, da, dgc, dalog_part, ddt_part, total;
};

BwdLayout bwd_layout(int64_t total_tokens, int H, int N);
cudaError_t launch_bwd(const StagedArgs& a, const BwdArgs& d, char* workspace, const BwdLayout& B,
                       cudaStream_t stream);

cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* g, const float* beta,
                          const float* A_log, const float* dt_bias, float lower_bound, float scale,
                          float* state, void* out, int batch, int H, cudaStream_t stream,
                          bool scalar_gate = false);

// out_h = A_h S_h + B_h for h < H (all [128][128] fp32); out must not overlap A or S.
cudaError_t launch_state_affine(const float* A, const float* S, const float* B, float* out, int H,
                                cudaStream_t stream);

// The fused persistent tcgen05 kernel of kda_fwd (same arguments; no workspace); it needs
// lower_bound >= KDA_FUSED_MIN_LOWER_BOUND (fused_supported).
cudaError_t launch_pipe(const StagedArgs& a, cudaStream_t stream);
bool fused_supported(float lower_bound);
// Scalar-gate (Gated DeltaNet) variant: a.g is [Ttot][H], a.dt_bias [H]; any lower bound.
cudaError_t launch_pipe_gdn(const StagedArgs& a, cudaStream_t stream);

}  // namespace kda
