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

/* ------------------------------------------------------------------------------------------
 * Backward pass (gradients) — TEST INFRASTRUCTURE ONLY, like everything in this file.
 *
 * torchtitan trains through chunk_kda, and its varlen test checks the gradient as well as the
 * forward (torchtitan PR #4374, Results: test_varlen_matches_independent_documents, "forward and
 * gradient").  The adjoint below is the reverse-mode derivative of the token recurrence above,
 * taken step by step in reverse token order.  For one token (with Stil = Diag(alpha) S_{t-1},
 * p = Stil^T khat, delta = beta (v - p), S_t = Stil + khat delta^T, o_t = scale S_t^T qhat), given
 * dS (the gradient of the loss w.r.t. S_t, from later tokens and the final state) and do_t:
 *   dS     += scale qhat do^T                   dqhat  = scale S_t do
 *   dkhat   = dS delta                          ddelta = dS^T khat
 *   dbeta   = ddelta . (v - p)                  dv     = beta ddelta,   dp = -beta ddelta
 *   dStil   = dS + khat dp^T                    dkhat += Stil dp
 *   dalpha_c = sum_j dStil[c][j] S_{t-1}[c][j]  dS_{t-1} = Diag(alpha) dStil
 * then back through the in-kernel transforms:
 *   qhat = q / n (n = sqrt(sum q^2 + eps)):  dq = (dqhat - qhat (qhat . dqhat)) / n   (k alike)
 *   beta = sigmoid(b):                       db = dbeta beta (1 - beta)
 *   log alpha = lb sigmoid(x), x = e^A (g + dt):
 *       dx = dalpha alpha lb sigmoid(x) (1 - sigmoid(x));  dg = dx e^A;  ddt += dx e^A;  dA += dx x
 * The loss is sum(do * o) + sum(dfinal * S_final); d_initial is the gradient w.r.t. S_0.
 * Inputs here are fp64 (raw values before the transforms), so that finite differences of
 * kda_oracle_fwd_f64 can pin the adjoint.
 * ------------------------------------------------------------------------------------------ */

static void l2_normalize_d(const double* x, int d, double* out, double* norm) {
    double ss = 0.0;
    for (int c = 0; c < d; ++c) ss += x[c] * x[c];
    double n = sqrt(ss + KDA_ORACLE_L2_EPS);
    for (int c = 0; c < d; ++c) out[c] = x[c] / n;
    if (norm) *norm = n;
}

/* Forward pass from fp64 raw inputs (same steps as kda_oracle_fwd; no bf16 widening).  States
 * are [N,H,dk,dv] (S[k][v]). */
int kda_oracle_fwd_f64(const double* q, const double* k, const double* v, const double* g,
                       const double* beta, double scale, const double* A_log, const double* dt_bias,
                       double lower_bound, const double* initial_state, double* final_state,
                       double* out, const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                       int32_t num_heads, int32_t dk, int32_t dv) {
    if (dk <= 0 || dv <= 0 || num_heads <= 0 || total_tokens < 0) return 1;
    if (check_cu(cu_seqlens, num_seqs, total_tokens)) return 1;
    const size_t state_elems = (size_t)dk * dv;
    double* S = (double*)malloc(sizeof(double) * state_elems);
    double* qh = (double*)malloc(sizeof(double) * dk);
    double* kh = (double*)malloc(sizeof(double) * dk);
    double* la = (double*)malloc(sizeof(double) * dk);
    double* pred = (double*)malloc(sizeof(double) * dv);
    for (int32_t n = 0; n < num_seqs; ++n)
        for (int32_t h = 0; h < num_heads; ++h) {
            const size_t soff = ((size_t)n * num_heads + h) * state_elems;
            load_state(S, initial_state ? initial_state + soff : NULL, 0, dk, dv);
            const double a = exp(A_log[h]);
            for (int64_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
                const size_t row = (size_t)t * num_heads + h;
                l2_normalize_d(q + row * dk, dk, qh, NULL);
                l2_normalize_d(k + row * dk, dk, kh, NULL);
                for (int c = 0; c < dk; ++c)
                    la[c] = lower_bound * sigmoid(a * (g[row * dk + c] + dt_bias[(size_t)h * dk + c]));
                recurrence_step(S, qh, kh, v + row * dv, la, sigmoid(beta[row]), scale, dk, dv, pred,
                                out + row * dv);
            }
            store_state(S, final_state ? final_state + soff : NULL, 0, dk, dv);
        }
    free(S); free(qh); free(kh); free(la); free(pred);
    return 0;
}

/* Gradients of sum(d_out * o) + sum(d_final * S_final) w.r.t. every input, fp64.  Shapes as
 * kda_oracle_fwd_f64; d_final may be NULL (zero); dA_log [H] and ddt_bias [H,dk] are summed over
 * sequences; d_initial [N,H,dk,dv] may be NULL. */
int kda_oracle_bwd(const double* q, const double* k, const double* v, const double* g,
                   const double* beta, double scale, const double* A_log, const double* dt_bias,
                   double lower_bound, const double* initial_state, const double* d_out,
                   const double* d_final, const int32_t* cu_seqlens, int32_t num_seqs,
                   int64_t total_tokens, int32_t num_heads, int32_t dk, int32_t dv, double* dq,
                   double* dkey, double* dval, double* dg, double* dbeta, double* dA_log,
                   double* ddt_bias, double* d_initial, int32_t num_threads) {
    if (dk <= 0 || dv <= 0 || num_heads <= 0 || total_tokens < 0) return 1;
    if (check_cu(cu_seqlens, num_seqs, total_tokens)) return 1;
    const int64_t units = (int64_t)num_seqs * num_heads;
    const size_t se = (size_t)dk * dv;
    /* per-unit partial sums of the per-head parameter gradients, added up after the loop */
    double* part = (double*)calloc((size_t)(units > 0 ? units : 1) * (1 + dk), sizeof(double));
    int failed = 0;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif
#pragma omp parallel for schedule(dynamic, 1) reduction(|:failed)
    for (int64_t u = 0; u < units; ++u) {
        const int32_t n = (int32_t)(u / num_heads), h = (int32_t)(u % num_heads);
        const int64_t t0 = cu_seqlens[n], L = cu_seqlens[n + 1] - cu_seqlens[n];
        const size_t soff = ((size_t)n * num_heads + h) * se;
        const double ea = exp(A_log[h]);
        /* the forward, keeping every state and every transformed input */
        double* hist = (double*)malloc(sizeof(double) * se * (size_t)(L + 1));
        double* qh = (double*)malloc(sizeof(double) * dk * (size_t)(L > 0 ? L : 1));
        double* kh = (double*)malloc(sizeof(double) * dk * (size_t)(L > 0 ? L : 1));
        double* nq = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
        double* nk = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
        double* xg = (double*)malloc(sizeof(double) * dk * (size_t)(L > 0 ? L : 1));
        double* la = (double*)malloc(sizeof(double) * dk * (size_t)(L > 0 ? L : 1));
        double* bt = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
        double* pred = (double*)malloc(sizeof(double) * dv);
        double* otmp = (double*)malloc(sizeof(double) * dv);
        double* dS = (double*)malloc(sizeof(double) * se);
        double* dSt = (double*)malloc(sizeof(double) * se);
        double* St = (double*)malloc(sizeof(double) * se);
        double* vec = (double*)malloc(sizeof(double) * (4 * (size_t)dk + 4 * (size_t)dv));
        if (!hist || !qh || !kh || !nq || !nk || !xg || !la || !bt || !pred || !otmp || !dS || !dSt ||
            !St || !vec) {
            failed = 1;
        } else {
            load_state(hist, initial_state ? initial_state + soff : NULL, 0, dk, dv);
            for (int64_t i = 0; i < L; ++i) {
                const size_t row = (size_t)(t0 + i) * num_heads + h;
                l2_normalize_d(q + row * dk, dk, qh + i * dk, nq + i);
                l2_normalize_d(k + row * dk, dk, kh + i * dk, nk + i);
                for (int c = 0; c < dk; ++c) {
                    xg[i * dk + c] = ea * (g[row * dk + c] + dt_bias[(size_t)h * dk + c]);
                    la[i * dk + c] = lower_bound * sigmoid(xg[i * dk + c]);
                }
                bt[i] = sigmoid(beta[row]);
                memcpy(hist + (size_t)(i + 1) * se, hist + (size_t)i * se, sizeof(double) * se);
                recurrence_step(hist + (size_t)(i + 1) * se, qh + i * dk, kh + i * dk, v + row * dv,
                                la + i * dk, bt[i], scale, dk, dv, pred, otmp);
            }
            /* the reverse sweep */
            double* dqh = vec;
            double* dkh = vec + dk;
            double* dal = vec + 2 * (size_t)dk;
            double* alpha = vec + 3 * (size_t)dk;
            double* p = vec + 4 * (size_t)dk;
            double* delta = p + dv;
            double* ddelta = delta + dv;
            double* dp = ddelta + dv;
            for (size_t e = 0; e < se; ++e) dS[e] = d_final ? d_final[soff + e] : 0.0;
            double* ppart = part + (size_t)u * (1 + dk);
            for (int64_t i = L - 1; i >= 0; --i) {
                const size_t row = (size_t)(t0 + i) * num_heads + h;
                const double* Sp = hist + (size_t)i * se;
                const double* Sn = hist + (size_t)(i + 1) * se;
                const double* qi = qh + i * dk;
                const double* ki = kh + i * dk;
                const double* doi = d_out + row * dv;
                const double* vi = v + row * dv;
                const double b = bt[i];
                for (int c = 0; c < dk; ++c) alpha[c] = exp(la[i * dk + c]);
                /* o_t = scale S_t^T qhat */
                for (int c = 0; c < dk; ++c) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) {
                        dS[(size_t)c * dv + j] += scale * qi[c] * doi[j];
                        acc += Sn[(size_t)c * dv + j] * doi[j];
                    }
                    dqh[c] = scale * acc;
                }
                /* Stil, p, delta */
                for (int c = 0; c < dk; ++c)
                    for (int j = 0; j < dv; ++j) St[(size_t)c * dv + j] = alpha[c] * Sp[(size_t)c * dv + j];
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int c = 0; c < dk; ++c) acc += St[(size_t)c * dv + j] * ki[c];
                    p[j] = acc;
                    delta[j] = b * (vi[j] - acc);
                }
                /* S_t = Stil + khat delta^T */
                for (int c = 0; c < dk; ++c) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += dS[(size_t)c * dv + j] * delta[j];
                    dkh[c] = acc;
                }
                double dbt = 0.0;
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int c = 0; c < dk; ++c) acc += dS[(size_t)c * dv + j] * ki[c];
                    ddelta[j] = acc;
                    dbt += acc * (vi[j] - p[j]);
                    dval[row * dv + j] = b * acc;
                    dp[j] = -b * acc;
                }
                /* dStil = dS + khat dp^T;  dkhat += Stil dp;  dalpha;  dS_{t-1} = Diag(alpha) dStil */
                for (int c = 0; c < dk; ++c) {
                    double acc = 0.0, da = 0.0;
                    for (int j = 0; j < dv; ++j) {
                        const double d = dS[(size_t)c * dv + j] + ki[c] * dp[j];
                        dSt[(size_t)c * dv + j] = d;
                        acc += St[(size_t)c * dv + j] * dp[j];
                        da += d * Sp[(size_t)c * dv + j];
                    }
                    dkh[c] += acc;
                    dal[c] = da;
                }
                for (int c = 0; c < dk; ++c)
                    for (int j = 0; j < dv; ++j) dS[(size_t)c * dv + j] = alpha[c] * dSt[(size_t)c * dv + j];
                /* back through the transforms */
                double sq = 0.0, sk = 0.0;
                for (int c = 0; c < dk; ++c) {
                    sq += qi[c] * dqh[c];
                    sk += ki[c] * dkh[c];
                }
                for (int c = 0; c < dk; ++c) {
                    dq[row * dk + c] = (dqh[c] - qi[c] * sq) / nq[i];
                    dkey[row * dk + c] = (dkh[c] - ki[c] * sk) / nk[i];
                    const double sig = sigmoid(xg[i * dk + c]);
                    const double dx = dal[c] * alpha[c] * lower_bound * sig * (1.0 - sig);
                    dg[row * dk + c] = dx * ea;
                    ppart[1 + c] += dx * ea;
                    ppart[0] += dx * xg[i * dk + c];
                }
                dbeta[row] = dbt * b * (1.0 - b);
            }
            if (d_initial)
                for (size_t e = 0; e < se; ++e) d_initial[soff + e] = dS[e];
        }
        free(hist); free(qh); free(kh); free(nq); free(nk); free(xg); free(la); free(bt); free(pred);
        free(otmp); free(dS); free(dSt); free(St); free(vec);
    }
    if (!failed) {
        for (int32_t h = 0; h < num_heads; ++h) {
            dA_log[h] = 0.0;
            for (int c = 0; c < dk; ++c) ddt_bias[(size_t)h * dk + c] = 0.0;
        }
        for (int64_t u = 0; u < units; ++u) {
            const int32_t h = (int32_t)(u % num_heads);
            dA_log[h] += part[(size_t)u * (1 + dk)];
            for (int c = 0; c < dk; ++c) ddt_bias[(size_t)h * dk + c] += part[(size_t)u * (1 + dk) + 1 + c];
        }
    }
    free(part);
    return failed ? 2 : 0;
}
