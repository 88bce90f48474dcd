/*
 * Oracle for the Kimi Delta Attention (KDA) forward pass — TEST INFRASTRUCTURE ONLY.
 *
 * This file is the plain, slow, obviously-correct CPU statement of what the GPU path
 * computes.  Only the tests, the smoke check and the bench's CPU-baseline leg may load it;
 * the product path never does.  It shares no code, header or table with the CUDA library.
 *
 * What it computes (fp64 throughout, token by token, one (sequence, head) unit at a time):
 *
 *   Inputs are the arguments of FlashKDA's `fwd` / fla's `chunk_kda` as the pages print
 *   them ("What CUDA Version Is Required to Use FlashKDA?", section Usage Examples; vLLM
 *   PR #54859 report, section 关键源码片段, test_flashkda_near_collinear_keys_remain_finite):
 *   bf16 q, k, v, g (raw gate), beta (raw), fp32 A_log[H], dt_bias[H,K], lower_bound,
 *   scale, fp32 initial/final state [N,H,K,V], int32 cu_seqlens [N+1].
 *
 *   In-kernel transforms (the flags use_qk_l2norm_in_kernel, use_beta_sigmoid_in_kernel,
 *   use_gate_in_kernel and safe_gate that the chunk_kda example turns on):
 *     qhat = q / sqrt(sum q^2 + eps),  khat likewise,  eps = 1e-6
 *     beta = sigmoid(raw_beta)
 *     log_alpha_c = lower_bound * sigmoid(exp(A_log[h]) * (g_c + dt_bias[h,c]))
 *
 *   The KDA recurrence (gated delta rule with a per-channel diagonal decay):
 *     S_t = (I - beta_t khat_t khat_t^T) Diag(alpha_t) S_{t-1} + beta_t khat_t v_t^T
 *     o_t = scale * S_t^T qhat_t
 *   evaluated as: decay the rows of S by alpha, predict S^T khat, add the rank-1 delta
 *   correction beta * khat (v - pred)^T, read the output from the updated state.
 *   S is K x V and stored S[k][v].
 *
 * Readings taken where the pages are silent:
 *   - eps of the L2 norm is 1e-6 and sits inside the square root; a zero vector maps to 0.
 *   - `scale` multiplies the output only; it never enters the state.
 *   - the output reads the state after the token's update.
 *   - a NULL initial state means zeros; a NULL final state is not written.
 *   - state_transposed = 1 stores the state as [N,H,V,K] (S^T) instead of [N,H,K,V].
 *
 * Inputs in bf16 are passed as their raw 16-bit patterns and widened exactly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define KDA_ORACLE_L2_EPS 1e-6

static double bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* qhat (or khat) of one token: x / sqrt(sum x^2 + eps). */
static void l2_normalize(const uint16_t* x, int d, double* out) {
    double ss = 0.0;
    for (int c = 0; c < d; ++c) {
        double xc = bf16_to_double(x[c]);
        out[c] = xc;
        ss += xc * xc;
    }
    double inv = 1.0 / sqrt(ss + KDA_ORACLE_L2_EPS);
    for (int c = 0; c < d; ++c) out[c] *= inv;
}

/* log alpha of one token: lower_bound * sigmoid(exp(A_log) * (g + dt_bias)). */
static void safe_gate(const uint16_t* g, const float* dt_bias_h, double a_log, double lower_bound,
                      int d, double* log_alpha) {
    double a = exp(a_log);
    for (int c = 0; c < d; ++c) {
        double x = bf16_to_double(g[c]) + (double)dt_bias_h[c];
        log_alpha[c] = lower_bound * sigmoid(a * x);
    }
}

/* One token of the recurrence on S[K][V] given the transformed inputs. */
static void recurrence_step(double* S, const double* qhat, const double* khat, const double* v,
                            const double* log_alpha, double beta, double scale, int dk, int dv,
                            double* pred, double* o) {
    for (int c = 0; c < dk; ++c) {
        double alpha = exp(log_alpha[c]);
        double* row = S + (size_t)c * dv;
        for (int j = 0; j < dv; ++j) row[j] *= alpha;
    }
    for (int j = 0; j < dv; ++j) pred[j] = 0.0;
    for (int c = 0; c < dk; ++c) {
        const double* row = S + (size_t)c * dv;
        for (int j = 0; j < dv; ++j) pred[j] += row[j] * khat[c];
    }
    for (int j = 0; j < dv; ++j) pred[j] = beta * (v[j] - pred[j]); /* delta */
    for (int c = 0; c < dk; ++c) {
        double* row = S + (size_t)c * dv;
        for (int j = 0; j < dv; ++j) row[j] += khat[c] * pred[j];
    }
    for (int j = 0; j < dv; ++j) o[j] = 0.0;
    for (int c = 0; c < dk; ++c) {
        const double* row = S + (size_t)c * dv;
        for (int j = 0; j < dv; ++j) o[j] += row[j] * qhat[c];
    }
    for (int j = 0; j < dv; ++j) o[j] *= scale;
}

static void load_state(double* S, const double* src, int transposed, int dk, int dv) {
    if (!src) {
        memset(S, 0, sizeof(double) * (size_t)dk * dv);
        return;
    }
    for (int c = 0; c < dk; ++c)
        for (int j = 0; j < dv; ++j)
            S[(size_t)c * dv + j] = transposed ? src[(size_t)j * dk + c] : src[(size_t)c * dv + j];
}

static void store_state(const double* S, double* dst, int transposed, int dk, int dv) {
    if (!dst) return;
    for (int c = 0; c < dk; ++c)
        for (int j = 0; j < dv; ++j) {
            if (transposed) dst[(size_t)j * dk + c] = S[(size_t)c * dv + j];
            else dst[(size_t)c * dv + j] = S[(size_t)c * dv + j];
        }
}

static int check_cu(const int32_t* cu, int32_t n, int64_t total) {
    if (!cu || n < 0) return 1;
    if (cu[0] != 0 || (int64_t)cu[n] != total) return 1;
    for (int32_t i = 0; i < n; ++i)
        if (cu[i + 1] < cu[i]) return 1;
    return 0;
}

/*
 * Full forward from the raw inputs.
 *   q, k, g   : bf16 bits [total_tokens, H, dk]   (a [B,T,H,dk] batch is B*T tokens)
 *   v         : bf16 bits [total_tokens, H, dv]
 *   beta      : bf16 bits [total_tokens, H] (raw, before the sigmoid)
 *   A_log     : fp32 [H];  dt_bias: fp32 [H, dk]
 *   initial_state / final_state : fp64 [N, H, dk, dv] (or [N,H,dv,dk] when transposed); NULL allowed
 *   out       : fp64 [total_tokens, H, dv]
 *   cu_seqlens: host int32 [N+1], cu[0] = 0, cu[N] = total_tokens, non-decreasing
 * Returns 0 on success, 1 on a malformed cu_seqlens or size.
 */
int kda_oracle_fwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* g,
                   const uint16_t* beta, double scale, const float* A_log, const float* dt_bias,
                   double lower_bound, const double* initial_state, double* final_state, double* out,
                   const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens, int32_t num_heads,
                   int32_t dk, int32_t dv, int32_t state_transposed, int32_t num_threads) {
    if (dk <= 0 || dv <= 0 || num_heads <= 0 || total_tokens < 0) return 1;
    if (check_cu(cu_seqlens, num_seqs, total_tokens)) return 1;
    const int64_t units = (int64_t)num_seqs * num_heads;
    const size_t state_elems = (size_t)dk * dv;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif
#pragma omp parallel
    {
        double* S = (double*)malloc(sizeof(double) * state_elems);
        double* qh = (double*)malloc(sizeof(double) * dk);
        double* kh = (double*)malloc(sizeof(double) * dk);
        double* la = (double*)malloc(sizeof(double) * dk);
        double* vv = (double*)malloc(sizeof(double) * dv);
        double* pred = (double*)malloc(sizeof(double) * dv);
#pragma omp for schedule(dynamic, 1)
        for (int64_t u = 0; u < units; ++u) {
            const int32_t n = (int32_t)(u / num_heads);
            const int32_t h = (int32_t)(u % num_heads);
            const size_t soff = ((size_t)n * num_heads + h) * state_elems;
            load_state(S, initial_state ? initial_state + soff : NULL, state_transposed, dk, dv);
            const double a_log = (double)A_log[h];
            const float* dtb = dt_bias + (size_t)h * dk;
            for (int64_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
                const size_t row = (size_t)t * num_heads + h;
                l2_normalize(q + row * dk, dk, qh);
                l2_normalize(k + row * dk, dk, kh);
                safe_gate(g + row * dk, dtb, a_log, lower_bound, dk, la);
                const double b = sigmoid(bf16_to_double(beta[row]));
                for (int j = 0; j < dv; ++j) vv[j] = bf16_to_double(v[row * dv + j]);
                recurrence_step(S, qh, kh, vv, la, b, scale, dk, dv, pred, out + row * dv);
            }
            store_state(S, final_state ? final_state + soff : NULL, state_transposed, dk, dv);
        }
        free(S); free(qh); free(kh); free(la); free(vv); free(pred);
    }
    return 0;
}

/*
 * The in-kernel transforms alone, for every token and head:
 *   qhat, khat, log_alpha : fp64 [total_tokens, H, dk];  beta_out : fp64 [total_tokens, H]
 */
void kda_oracle_prologue(const uint16_t* q, const uint16_t* k, const uint16_t* g, const uint16_t* beta,
                         const float* A_log, const float* dt_bias, double lower_bound,
                         int64_t total_tokens, int32_t num_heads, int32_t dk, double* qhat,
                         double* khat, double* log_alpha, double* beta_out) {
    for (int64_t t = 0; t < total_tokens; ++t)
        for (int32_t h = 0; h < num_heads; ++h) {
            const size_t row = (size_t)t * num_heads + h;
            if (qhat) l2_normalize(q + row * dk, dk, qhat + row * dk);
            if (khat) l2_normalize(k + row * dk, dk, khat + row * dk);
            if (log_alpha)
                safe_gate(g + row * dk, dt_bias + (size_t)h * dk, (double)A_log[h], lower_bound, dk,
                          log_alpha + row * dk);
            if (beta_out) beta_out[row] = sigmoid(bf16_to_double(beta[row]));
        }
}

/*
 * The recurrence alone, from already-transformed fp64 inputs (for the invariant tests,
 * which need beta and alpha exactly 0 or 1):
 *   qhat, khat, log_alpha : [total_tokens, H, dk];  v : [total_tokens, H, dv];  beta : [total_tokens, H]
 *   S0 / S_final : [N, H, dk, dv] (S[k][v]); out : [total_tokens, H, dv]
 */
int kda_oracle_core(const double* qhat, const double* khat, const double* v, const double* log_alpha,
                    const double* beta, double scale, const double* S0, double* S_final, double* out,
                    const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                    int32_t num_heads, int32_t dk, int32_t dv) {
    if (dk <= 0 || dv <= 0 || num_heads <= 0 || total_tokens < 0) return 1;
    if (check_cu(cu_seqlens, num_seqs, total_tokens)) return 1;
    const size_t state_elems = (size_t)dk * dv;
    double* S = (double*)malloc(sizeof(double) * state_elems);
    double* pred = (double*)malloc(sizeof(double) * dv);
    for (int32_t n = 0; n < num_seqs; ++n)
        for (int32_t h = 0; h < num_heads; ++h) {
            const size_t soff = ((size_t)n * num_heads + h) * state_elems;
            load_state(S, S0 ? S0 + soff : NULL, 0, dk, dv);
            for (int64_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
                const size_t row = (size_t)t * num_heads + h;
                recurrence_step(S, qhat + row * dk, khat + row * dk, v + row * dv,
                                log_alpha + row * dk, beta[row], scale, dk, dv, pred, out + row * dv);
            }
            store_state(S, S_final ? S_final + soff : NULL, 0, dk, dv);
        }
    free(S);
    free(pred);
    return 0;
}
