/*
 * kda_ref.c -- fp64 CPU oracle for the Kimi Delta Attention (KDA) forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: only the tests, __graft_entry__.smoke() and the CPU-baseline
 * leg of bench.py use it.  It shares no code with the CUDA library.
 *
 * What it computes (the plain definition, token by token, no chunking):
 *
 *   KDA is the gated delta rule with channel-wise decay ("FlashKDA ... Kimi
 *   Delta Attention", donniechu.com, section "Số liệu kỹ thuật": fine-grained
 *   channel-wise gating with learned A_log, dt_bias, lower_bound; batch,
 *   cu_seqlens varlen, initial/final recurrent state; K = V = 128).  The pages
 *   print no formula; this library fixes it as
 *
 *     x_t        = g_t + dt_bias_h                        (per channel)
 *     softplus   = log(1 + exp(x))                        (exact, no cutoff)
 *     log a_t    = max(-exp(A_log_h) * softplus(x_t), lower_bound)
 *     S_t        = (I - beta_t k_t k_t^T) Diag(a_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t        = scale * S_t^T q_t
 *
 *   S is K x V (rows = key channels).  The decay acts on the key rows and
 *   precedes the erase; o_t reads the state after token t's update.  The
 *   transition (I - beta k k^T) Diag(a) = Diag(a) - beta k (a*k)^T is the
 *   diagonal-plus-low-rank form the asksurf.ai English post's comparison
 *   table attributes to KDA.
 *
 * Every (sequence, head) pair is independent; they are spread over OpenMP
 * threads.  All arithmetic is IEEE double.  q/k/v arrive as raw bf16 bit
 * patterns and g/beta as float32; both widen to double exactly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 bit pattern -> double, exactly: a bf16 value is the top half of a
 * float32 with the low 16 mantissa bits zero. */
static double bf16_to_double(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

void kda_oracle_bf16_to_f64(const uint16_t* src, double* dst, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) dst[i] = bf16_to_double(src[i]);
}

/* softplus(x) = log(1 + e^x), written without overflow: max(x,0) + log1p(e^-|x|). */
static double softplus(double x)
{
    return (x > 0.0 ? x : 0.0) + log1p(exp(-fabs(x)));
}

/* Gate: log a = max(-exp(A_log) * softplus(g + dt_bias), lower_bound).
 * A lower_bound of -inf leaves the value unclamped. */
static double log_decay(double g, double dt_bias, double A_log, double lower_bound)
{
    double la = -exp(A_log) * softplus(g + dt_bias);
    return la > lower_bound ? la : lower_bound;
}

/* Public gate evaluation for tests: la[t,h,c] over a [T,H,K] float32 g. */
void kda_oracle_gate(const float* g, const float* A_log, const float* dt_bias,
                     double lower_bound, int64_t T, int64_t H, int64_t K, double* la)
{
    for (int64_t t = 0; t < T; ++t)
        for (int64_t h = 0; h < H; ++h)
            for (int64_t c = 0; c < K; ++c) {
                int64_t i = (t * H + h) * K + c;
                la[i] = log_decay((double)g[i], (double)dt_bias[h * K + c],
                                  (double)A_log[h], lower_bound);
            }
}

/*
 * kda_oracle_recurrent
 *   q, k      : [T, H, K] bf16 bits        v : [T, H, V] bf16 bits
 *   g         : [T, H, K] float32 (gate_mode 0: raw gate input;
 *               gate_mode 1: the log-decay log a itself, gate bypassed)
 *   beta      : [T, H] float32
 *   A_log     : [H] float32, dt_bias : [H, K] float32 (unused in gate_mode 1)
 *   initial_state : [N, H, K, V] double, or NULL for zeros
 *   cu_seqlens: [N + 1] int64 offsets into T (monotone, cu[0] = 0, cu[N] = T)
 *   additive  : 0 = delta rule; 1 = plain additive update S += beta k v^T
 *               (linear attention; used only by the tests' invariants)
 *   out       : [T, H, V] double
 *   final_state : [N, H, K, V] double, or NULL to skip
 * Returns 0, or -1 on an allocation failure.
 */
int kda_oracle_recurrent(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                         const float* g, const float* beta,
                         const float* A_log, const float* dt_bias,
                         double lower_bound, double scale,
                         const double* initial_state, const int64_t* cu_seqlens,
                         int64_t N, int64_t T, int64_t H, int64_t K, int64_t V,
                         int gate_mode, int additive,
                         double* out, double* final_state, int nthreads)
{
    (void)T;
    int failed = 0;
    int64_t units = N * H;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
#endif
    for (int64_t u = 0; u < units; ++u) {
        int64_t n = u / H, h = u % H;
        double* S = (double*)malloc(sizeof(double) * (size_t)(K * V));
        double* kk = (double*)malloc(sizeof(double) * (size_t)K);
        double* qq = (double*)malloc(sizeof(double) * (size_t)K);
        double* a = (double*)malloc(sizeof(double) * (size_t)K);
        double* vv = (double*)malloc(sizeof(double) * (size_t)V);
        double* w = (double*)malloc(sizeof(double) * (size_t)V);
        if (!S || !kk || !qq || !a || !vv || !w) {
            failed = 1;
            free(S); free(kk); free(qq); free(a); free(vv); free(w);
            continue;
        }
        if (initial_state)
            memcpy(S, initial_state + (n * H + h) * K * V, sizeof(double) * (size_t)(K * V));
        else
            memset(S, 0, sizeof(double) * (size_t)(K * V));

        for (int64_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
            const int64_t base_k = (t * H + h) * K;
            const int64_t base_v = (t * H + h) * V;
            const double b = (double)beta[t * H + h];
            for (int64_t c = 0; c < K; ++c) {
                kk[c] = bf16_to_double(k[base_k + c]);
                qq[c] = bf16_to_double(q[base_k + c]);
                double la = gate_mode == 0
                    ? log_decay((double)g[base_k + c], (double)dt_bias[h * K + c],
                                (double)A_log[h], lower_bound)
                    : (double)g[base_k + c];
                a[c] = exp(la);
            }
            for (int64_t j = 0; j < V; ++j) vv[j] = bf16_to_double(v[base_v + j]);

            /* S <- Diag(a) S : the decay scales each key row. */
            for (int64_t c = 0; c < K; ++c) {
                double* row = S + c * V;
                for (int64_t j = 0; j < V; ++j) row[j] *= a[c];
            }
            if (additive) {
                /* S <- S + beta k v^T */
                for (int64_t c = 0; c < K; ++c) {
                    double* row = S + c * V;
                    double f = b * kk[c];
                    for (int64_t j = 0; j < V; ++j) row[j] += f * vv[j];
                }
            } else {
                /* w = S^T k (the value the state currently predicts for k) */
                for (int64_t j = 0; j < V; ++j) w[j] = 0.0;
                for (int64_t c = 0; c < K; ++c) {
                    const double* row = S + c * V;
                    for (int64_t j = 0; j < V; ++j) w[j] += kk[c] * row[j];
                }
                /* S <- S - beta k (S^T k)^T + beta k v^T = S + beta k (v - w)^T */
                for (int64_t j = 0; j < V; ++j) w[j] = vv[j] - w[j];
                for (int64_t c = 0; c < K; ++c) {
                    double* row = S + c * V;
                    double f = b * kk[c];
                    for (int64_t j = 0; j < V; ++j) row[j] += f * w[j];
                }
            }
            /* o_t = scale * S_t^T q_t */
            double* o = out + base_v;
            for (int64_t j = 0; j < V; ++j) o[j] = 0.0;
            for (int64_t c = 0; c < K; ++c) {
                const double* row = S + c * V;
                for (int64_t j = 0; j < V; ++j) o[j] += qq[c] * row[j];
            }
            for (int64_t j = 0; j < V; ++j) o[j] *= scale;
        }
        if (final_state)
            memcpy(final_state + (n * H + h) * K * V, S, sizeof(double) * (size_t)(K * V));
        free(S); free(kk); free(qq); free(a); free(vv); free(w);
    }
    return failed ? -1 : 0;
}

/* Number of OpenMP threads a parallel region would use (1 without OpenMP). */
int kda_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
