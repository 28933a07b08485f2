/*
 * kda_oracle.c -- float64 CPU oracle for the Kimi Delta Attention (KDA) forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link or
 * call this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or helper with the
 * CUDA library; the two agree only because both follow the same pages.
 *
 * Sources restated here (page title, then section / equation / table):
 *   [R] KDA notes, "KDA 递归核心" (recurrence core), §逐步公式, steps 1-4 (decay,
 *       residual, rank-1 write, read-out); same steps in the KDA ledger,
 *       derivation DER1, and in the DeltaNet-family digest, section
 *       "Kimi Delta Attention: channel-wise decay", steps 1-5.
 *   [W] KDA notes, "KDA 递归核心", warning box on exp(g_t).unsqueeze(-1): the
 *       decay is per KEY channel and shared by all value columns.
 *   [G] KDA notes, "Gate 激活", table "两种 Gate" and the itemised definitions
 *       input = g_raw + dt_bias[HV,K], rate = exp(A_log[HV]).
 *   [C] DeltaNet-family digest, section "Chunkwise KDA": cumulative decay
 *       D_{0:i}, provisional errors, coupling rho_ij, causal solve, chunk-end
 *       state and chunk outputs.
 *
 * All arithmetic is IEEE double with no reordering beyond what the
 * definitions state.  Layouts (row-major, contiguous):
 *   q, k   [B, T, H, K]     v [B, T, HV, V]     g, g_raw [B, T, HV, K]
 *   beta   [B, T, HV]       S0, S_out [B, HV, K, V] (key-major state)
 *   o      [B, T, HV, V]    A_log [HV]          dt_bias [HV, K]
 * GVA: value head hv reads q/k head hv / (HV/H) (repeat_interleave).
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#define KDA_ORACLE_GATE_SAFE 1
#define KDA_ORACLE_GATE_STANDARD 2

/* [G] Gate activation, element by element.
 *   safe:     g = L * sigmoid(rate * input)      -- rate is INSIDE the sigmoid
 *   standard: g = -rate * softplus(input)        -- rate is OUTSIDE the softplus
 * softplus(x) = max(x,0) + log1p(exp(-|x|)) is the exact softplus written so
 * that it cannot overflow.  `rows` = B*T.  Returns 0, or -1 on a bad mode. */
int kda_oracle_gate(const double* g_raw, const double* A_log, const double* dt_bias,
                    long rows, int HV, int K, int mode, double lower_bound, double* g_out)
{
    if (mode != KDA_ORACLE_GATE_SAFE && mode != KDA_ORACLE_GATE_STANDARD) return -1;
    for (long r = 0; r < rows; ++r) {
        for (int h = 0; h < HV; ++h) {
            const double rate = exp(A_log[h]);
            for (int d = 0; d < K; ++d) {
                const long idx = ((long)r * HV + h) * K + d;
                const double x = g_raw[idx] + (dt_bias ? dt_bias[(long)h * K + d] : 0.0);
                double g;
                if (mode == KDA_ORACLE_GATE_SAFE) {
                    g = lower_bound / (1.0 + exp(-rate * x));
                } else {
                    const double sp = (x > 0.0 ? x : 0.0) + log1p(exp(-fabs(x)));
                    g = -rate * sp;
                }
                g_out[idx] = g;
            }
        }
    }
    return 0;
}

/* [R] The naive per-token recurrence.  For each (b, hv) independently,
 * starting from S = S0 (or 0):
 *   S_dec[d,:] = exp(g_t[d]) * S[d,:]            step 1, decay per key channel [W]
 *   p          = sum_d k_t[d] * S_dec[d,:]       step 2, prediction
 *   r          = v_t - p                         step 2, residual
 *   S          = S_dec + (beta_t k_t) (x) r      step 3, rank-1 write
 *   o_t        = scale * sum_d q_t[d] * S[d,:]   step 4, read-out (scale = 1/sqrt(K))
 * `g` is the log-space decay (already gated). */
void kda_oracle_recurrent(const double* q, const double* k, const double* v, const double* g,
                          const double* beta, const double* S0, int B, int T, int H, int HV,
                          int K, int V, double scale, double* o, double* S_out)
{
    const int G = HV / H;
    const long npairs = (long)B * HV;
#pragma omp parallel for schedule(dynamic, 1)
    for (long pair = 0; pair < npairs; ++pair) {
        const int b = (int)(pair / HV);
        const int hv = (int)(pair % HV);
        const int h = hv / G;
        double* S = (double*)malloc(sizeof(double) * (size_t)K * V);
        double* p = (double*)malloc(sizeof(double) * (size_t)V);
        if (S0) memcpy(S, S0 + pair * (long)K * V, sizeof(double) * (size_t)K * V);
        else memset(S, 0, sizeof(double) * (size_t)K * V);
        for (int t = 0; t < T; ++t) {
            const long tok = (long)b * T + t;
            const double* qt = q + (tok * H + h) * K;
            const double* kt = k + (tok * H + h) * K;
            const double* vt = v + (tok * HV + hv) * V;
            const double* gt = g + (tok * HV + hv) * K;
            const double bt = beta[tok * HV + hv];
            /* step 1 */
            for (int d = 0; d < K; ++d) {
                const double a = exp(gt[d]);
                for (int j = 0; j < V; ++j) S[(long)d * V + j] *= a;
            }
            /* step 2 */
            for (int j = 0; j < V; ++j) p[j] = 0.0;
            for (int d = 0; d < K; ++d)
                for (int j = 0; j < V; ++j) p[j] += kt[d] * S[(long)d * V + j];
            for (int j = 0; j < V; ++j) p[j] = vt[j] - p[j]; /* p now holds r */
            /* step 3 */
            for (int d = 0; d < K; ++d) {
                const double a = bt * kt[d];
                for (int j = 0; j < V; ++j) S[(long)d * V + j] += a * p[j];
            }
            /* step 4 */
            double* ot = o + (tok * HV + hv) * V;
            for (int j = 0; j < V; ++j) ot[j] = 0.0;
            for (int d = 0; d < K; ++d)
                for (int j = 0; j < V; ++j) ot[j] += qt[d] * S[(long)d * V + j];
            for (int j = 0; j < V; ++j) ot[j] *= scale;
        }
        if (S_out) memcpy(S_out + pair * (long)K * V, S, sizeof(double) * (size_t)K * V);
        free(p);
        free(S);
    }
}

/* [C] A second, separately written form: the chunkwise equations, used to pin
 * the recurrence (the pages state that the chunked schedule reproduces the
 * recurrent one exactly).  Per chunk of n <= C tokens starting from state S:
 *   Gam_i      = sum_{m<=i} g_m                         (inclusive, per key channel)
 *   ebar_i     = beta_i (v_i - sum_d k_id e^{Gam_id} S[d,:])          provisional error
 *   rho_ij     = beta_i sum_d k_id k_jd e^{Gam_id - Gam_jd},  j < i    coupling
 *   e_i        = ebar_i - sum_{j<i} rho_ij e_j                        causal solve
 *   o_i        = scale sum_d q_id e^{Gam_id} S[d,:]
 *              + sum_{j<=i} (scale sum_d q_id k_jd e^{Gam_id - Gam_jd}) e_j
 *   S[d,:]    <- e^{Gam_{n-1,d}} S[d,:] + sum_j k_jd e^{Gam_{n-1,d} - Gam_jd} e_j
 * Every decay factor is an explicit exp of a difference of prefix sums; no
 * factorisation, no inverse matrix. */
void kda_oracle_chunkwise(const double* q, const double* k, const double* v, const double* g,
                          const double* beta, const double* S0, int B, int T, int H, int HV,
                          int K, int V, int C, double scale, double* o, double* S_out)
{
    const int G = HV / H;
    const long npairs = (long)B * HV;
#pragma omp parallel for schedule(dynamic, 1)
    for (long pair = 0; pair < npairs; ++pair) {
        const int b = (int)(pair / HV);
        const int hv = (int)(pair % HV);
        const int h = hv / G;
        double* S = (double*)malloc(sizeof(double) * (size_t)K * V);
        double* Gam = (double*)malloc(sizeof(double) * (size_t)C * K);
        double* E = (double*)malloc(sizeof(double) * (size_t)C * V);
        double* rho = (double*)malloc(sizeof(double) * (size_t)C * C);
        double* Snew = (double*)malloc(sizeof(double) * (size_t)K * V);
        if (S0) memcpy(S, S0 + pair * (long)K * V, sizeof(double) * (size_t)K * V);
        else memset(S, 0, sizeof(double) * (size_t)K * V);
        for (int c0 = 0; c0 < T; c0 += C) {
            const int n = (T - c0 < C) ? (T - c0) : C;
#define TOK(i) ((long)b * T + c0 + (i))
#define QI(i) (q + (TOK(i) * H + h) * K)
#define KI(i) (k + (TOK(i) * H + h) * K)
#define VI(i) (v + (TOK(i) * HV + hv) * V)
#define GI(i) (g + (TOK(i) * HV + hv) * K)
#define BI(i) (beta[TOK(i) * HV + hv])
            for (int d = 0; d < K; ++d) {
                double acc = 0.0;
                for (int i = 0; i < n; ++i) {
                    acc += GI(i)[d];
                    Gam[(long)i * K + d] = acc;
                }
            }
            /* provisional errors */
            for (int i = 0; i < n; ++i) {
                for (int j = 0; j < V; ++j) {
                    double acc = 0.0;
                    for (int d = 0; d < K; ++d)
                        acc += KI(i)[d] * exp(Gam[(long)i * K + d]) * S[(long)d * V + j];
                    E[(long)i * V + j] = BI(i) * (VI(i)[j] - acc);
                }
            }
            /* coupling */
            for (int i = 0; i < n; ++i)
                for (int j = 0; j < i; ++j) {
                    double acc = 0.0;
                    for (int d = 0; d < K; ++d)
                        acc += KI(i)[d] * KI(j)[d] * exp(Gam[(long)i * K + d] - Gam[(long)j * K + d]);
                    rho[(long)i * C + j] = BI(i) * acc;
                }
            /* causal solve, one value channel at a time, rows in order */
            for (int i = 0; i < n; ++i)
                for (int j = 0; j < i; ++j)
                    for (int x = 0; x < V; ++x)
                        E[(long)i * V + x] -= rho[(long)i * C + j] * E[(long)j * V + x];
            /* outputs */
            for (int i = 0; i < n; ++i) {
                double* oi = o + (TOK(i) * HV + hv) * V;
                for (int x = 0; x < V; ++x) {
                    double acc = 0.0;
                    for (int d = 0; d < K; ++d)
                        acc += QI(i)[d] * exp(Gam[(long)i * K + d]) * S[(long)d * V + x];
                    oi[x] = scale * acc;
                }
                for (int j = 0; j <= i; ++j) {
                    double a = 0.0;
                    for (int d = 0; d < K; ++d)
                        a += QI(i)[d] * KI(j)[d] * exp(Gam[(long)i * K + d] - Gam[(long)j * K + d]);
                    a *= scale;
                    for (int x = 0; x < V; ++x) oi[x] += a * E[(long)j * V + x];
                }
            }
            /* chunk-end state */
            for (int d = 0; d < K; ++d) {
                const double gend = Gam[(long)(n - 1) * K + d];
                for (int x = 0; x < V; ++x) {
                    double acc = exp(gend) * S[(long)d * V + x];
                    for (int j = 0; j < n; ++j)
                        acc += KI(j)[d] * exp(gend - Gam[(long)j * K + d]) * E[(long)j * V + x];
                    Snew[(long)d * V + x] = acc;
                }
            }
            memcpy(S, Snew, sizeof(double) * (size_t)K * V);
#undef TOK
#undef QI
#undef KI
#undef VI
#undef GI
#undef BI
        }
        if (S_out) memcpy(S_out + pair * (long)K * V, S, sizeof(double) * (size_t)K * V);
        free(Snew);
        free(rho);
        free(E);
        free(Gam);
        free(S);
    }
}

/* Number of OpenMP threads a parallel region of this library would use
 * (1 when built without OpenMP).  Reported beside CPU timings. */
int kda_oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
