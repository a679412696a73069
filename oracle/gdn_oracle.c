/*
 * gdn_oracle.c -- float64 CPU oracle for the Gated DeltaNet recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code with the CUDA library.
 *
 * It is written to be read against the pages, not to be fast: one
 * (request, value head) or (batch row, head) unit at a time, one token at a
 * time, every sum in float64, no blocking and no reordering.  OpenMP only
 * spreads independent units over host threads.
 *
 * Sources (pages, by title and section):
 *  - "com.microsoft.GatedDeltaNet" (ONNX Runtime contrib op), Description:
 *      S_t = exp(g_t) S_{t-1} + k_t (beta_t (v_t - exp(g_t) S_{t-1}^T k_t))^T,
 *      o_t = scale * S_t^T q_t, per value head; value head h reads query/key
 *      head h*Hq/Hv; Inputs table: cu_seqlens clamping, V-major float32
 *      initial/final state, empty requests copy their state through;
 *      Attributes table: qk_l2_norm with epsilon 1e-12, scale; update_rule
 *      (linear drops the decay and the delta retrieval, gated keeps only the
 *      decay, delta only the retrieval, gated_delta both; decay is an input
 *      exactly for gated / gated_delta, beta exactly for delta / gated_delta);
 *      gate_activation qwen: g = -exp(a_log) * softplus(decay + dt_bias);
 *      beta_activation sigmoid.
 *  - "Gated DeltaNet State Update" (tensortonic), statement: the same
 *      recurrence in the gamma form S_t = gamma_t (I - beta_t k_t k_t^T)
 *      S_{t-1} + beta_t k_t v_t^T with y_t = q_t^T S_t (gamma_t = exp(g_t)).
 *  - "flashinfer.cake_gdp.cake_gated_delta_product_mtp", description and
 *      Parameters: the decode/MTP pool update with the fused gate
 *      alpha = exp(-exp(A_log) softplus(a + dt_bias)) (softplus threshold 20),
 *      beta = sigmoid(b) per Householder sub-step, L2 norm x*rsqrt(sum x^2 +
 *      1e-6), padding rows, write-slot override and per-token scatter.
 *  - "max.nn.legacy.state_space.gated_delta_conv1d_fwd", description,
 *      Parameters and example: causal depthwise conv1d over ragged requests
 *      with a slot-indexed window pool updated in place (oracle_conv1d).
 *
 * Readings where the pages are silent (each one listed in the design notes):
 *  - the prefill L2 norm is x * (sum x^2 + 1e-12)^(-1/2);
 *  - h*Hq/Hv is integer floor division;
 *  - decode reads every row's slot from the pool as it was before the call
 *    (pool_in) and writes into a separate copy (pool_out); under the
 *    precondition that no row writes a slot another row reads, this is the
 *    in-place result;
 *  - a slot index >= pool_size is treated like a negative one (skipped);
 *  - an update rule without beta writes k_t v_t^T (beta = 1); one without
 *    the retrieval drops the -exp(g_t) S_{t-1}^T k_t term; one without decay
 *    uses g_t = 0;
 *  - the prefill qwen gate uses the decode page's softplus threshold 20.
 *
 * Parity pins: tests/test_oracle_pins.py checks this file against the worked
 * examples of "Gated DeltaNet State Update", a brute-force product of the
 * gamma form, closed forms and invariants; tests/test_oracle_conv1d_pins.py
 * checks the conv1d against its page's worked example, numpy's convolution,
 * delta-weight closed forms and continuation over calls.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static int64_t clamp_i64(int64_t x, int64_t lo, int64_t hi)
{
    return x < lo ? lo : (x > hi ? hi : x);
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static double softplus20(double x) { return x > 20.0 ? x : log1p(exp(x)); }

/* ------------------------------------------------------------------------
 * Prefill.
 *   q, k          [N, Hq, Dk]
 *   v, out        [N, Hv, Dv]
 *   g, beta       [N, Hv]            (log-space decay, update rate); g is NULL
 *                                    for rules without decay, beta for rules
 *                                    without retrieval
 *   g_per_key     non-zero: g is [N, Hv, Dk], one log-space decay per key
 *                                    dimension (the op's per-key-dimension
 *                                    spelling of `decay`)
 *   rule          0 gated_delta, 1 gated, 2 delta, 3 linear
 *   a_log, dt_bias [Hv] or NULL      (non-NULL: qwen gate on g)
 *   beta_sigmoid  non-zero: beta <- sigmoid(beta)
 *   cu_seqlens    [B+1] or NULL      (NULL: uniform packing, N = B*S)
 *   initial_state [B, Hv, Dv, Dk] or NULL (NULL: zero)
 *   final_state   [B, Hv, Dv, Dk]
 * The state is held here K-major, S[i][j] with i over Dk and j over Dv, as in
 * the gamma-form statement; the V-major inputs/outputs are transposed on the
 * way in and out.
 * ---------------------------------------------------------------------- */
void oracle_prefill(const double *q, const double *k, const double *v,
                    const double *g, const double *beta,
                    const int32_t *cu_seqlens,
                    const double *initial_state, double *final_state,
                    double *out,
                    int B, int64_t N, int Hq, int Hv, int Dk, int Dv,
                    double scale, int qk_l2norm, int rule,
                    const double *a_log, const double *dt_bias, int beta_sigmoid,
                    int g_per_key, int nthreads)
{
    int nunits = B * Hv;
    const int has_decay = rule == 0 || rule == 1;
    const int has_retrieval = rule == 0 || rule == 2;
    if (nthreads <= 0) nthreads = 1;

#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (int unit = 0; unit < nunits; ++unit) {
        int b = unit / Hv;
        int h = unit % Hv;
        int qh = (int)(((int64_t)h * Hq) / Hv);   /* floor(h * Hq / Hv) */

        int64_t start, end;
        if (cu_seqlens) {
            start = clamp_i64(cu_seqlens[b], 0, N);
            end = clamp_i64(cu_seqlens[b + 1], 0, N);
        } else {
            int64_t S = N / B;
            start = (int64_t)b * S;
            end = start + S;
        }

        double *S = (double *)calloc((size_t)Dk * Dv, sizeof(double));
        double *xq = (double *)malloc(sizeof(double) * Dk);
        double *xk = (double *)malloc(sizeof(double) * Dk);
        double *p = (double *)malloc(sizeof(double) * Dv);

        /* S_0 = initial_state[b, h]^T, or zero. */
        if (initial_state) {
            const double *s0 = initial_state + ((int64_t)b * Hv + h) * Dv * Dk;
            for (int i = 0; i < Dk; ++i)
                for (int j = 0; j < Dv; ++j)
                    S[(int64_t)i * Dv + j] = s0[(int64_t)j * Dk + i];
        }

        for (int64_t t = start; t < end; ++t) {
            const double *qt = q + (t * Hq + qh) * Dk;
            const double *kt = k + (t * Hq + qh) * Dk;
            const double *vt = v + (t * Hv + h) * Dv;
            for (int i = 0; i < Dk; ++i) {
                xq[i] = qt[i];
                xk[i] = kt[i];
            }
            if (qk_l2norm) {
                double sq = 0.0, sk = 0.0;
                for (int i = 0; i < Dk; ++i) {
                    sq += xq[i] * xq[i];
                    sk += xk[i] * xk[i];
                }
                double rq = 1.0 / sqrt(sq + 1e-12);
                double rk = 1.0 / sqrt(sk + 1e-12);
                for (int i = 0; i < Dk; ++i) {
                    xq[i] *= rq;
                    xk[i] *= rk;
                }
            }
            if (g_per_key) {
                /* Per-key-dimension decay: the scalar exp(g_t) of the recurrence becomes
                 * D_t = diag(exp(g_t[0..Dk))) acting on the key axis of S, in both of its
                 * places: S_t = D_t S_{t-1} + k_t (beta_t (v_t - (D_t S_{t-1})^T k_t))^T. */
                double bt = 1.0;
                if (has_retrieval) {
                    bt = beta[t * Hv + h];
                    if (beta_sigmoid) bt = 1.0 / (1.0 + exp(-bt));
                }
                const double *gt = g + (t * Hv + h) * Dk;
                /* S <- D_t S_{t-1} */
                for (int i = 0; i < Dk; ++i) {
                    double li = gt[i];
                    if (a_log) li = -exp(a_log[h]) * softplus20(li + dt_bias[h]);
                    const double gi = exp(li);
                    for (int j = 0; j < Dv; ++j) S[(int64_t)i * Dv + j] *= gi;
                }
                /* p = (D_t S_{t-1})^T k_t */
                for (int j = 0; j < Dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < Dk; ++i) acc += S[(int64_t)i * Dv + j] * xk[i];
                    p[j] = acc;
                }
                /* S_t = D_t S_{t-1} + k_t (beta (v_t - p))^T; without the retrieval the
                 * written value is beta v_t */
                for (int i = 0; i < Dk; ++i)
                    for (int j = 0; j < Dv; ++j) {
                        double u = bt * (vt[j] - (has_retrieval ? p[j] : 0.0));
                        S[(int64_t)i * Dv + j] += xk[i] * u;
                    }
                double *ot = out + (t * Hv + h) * Dv;
                for (int j = 0; j < Dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < Dk; ++i) acc += S[(int64_t)i * Dv + j] * xq[i];
                    ot[j] = scale * acc;
                }
                continue;
            }
            /* gate: log-space decay (qwen form if requested), update rate */
            double lg = 0.0;
            if (has_decay) {
                lg = g[t * Hv + h];
                if (a_log) lg = -exp(a_log[h]) * softplus20(lg + dt_bias[h]);
            }
            double gamma = exp(lg);
            double bt = 1.0;
            if (has_retrieval) {
                bt = beta[t * Hv + h];
                if (beta_sigmoid) bt = 1.0 / (1.0 + exp(-bt));
            }

            /* p = S_{t-1}^T k_t */
            for (int j = 0; j < Dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < Dk; ++i) acc += S[(int64_t)i * Dv + j] * xk[i];
                p[j] = acc;
            }
            /* S_t = gamma S_{t-1} + k_t (beta (v_t - gamma p))^T; without the
             * retrieval the written value is beta v_t */
            for (int i = 0; i < Dk; ++i)
                for (int j = 0; j < Dv; ++j) {
                    double u = bt * (vt[j] - (has_retrieval ? gamma * p[j] : 0.0));
                    S[(int64_t)i * Dv + j] = gamma * S[(int64_t)i * Dv + j] + xk[i] * u;
                }
            /* o_t = scale * S_t^T q_t */
            double *ot = out + (t * Hv + h) * Dv;
            for (int j = 0; j < Dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < Dk; ++i) acc += S[(int64_t)i * Dv + j] * xq[i];
                ot[j] = scale * acc;
            }
        }

        /* final_state[b, h] = S^T (V-major). */
        double *sf = final_state + ((int64_t)b * Hv + h) * Dv * Dk;
        for (int j = 0; j < Dv; ++j)
            for (int i = 0; i < Dk; ++i)
                sf[(int64_t)j * Dk + i] = S[(int64_t)i * Dv + j];

        free(S);
        free(xq);
        free(xk);
        free(p);
    }
}

/* ------------------------------------------------------------------------
 * Decode / MTP (Gated DeltaProduct with num_householder = nh sub-steps).
 *   q        [B, T, H, Dk]
 *   k        [B, T, nh, H, Dk]
 *   v        [B, T, nh, HV, Dv]
 *   pool_in  [P, HV, Dv, Dk]   slots as they were before the call
 *   pool_out [P, HV, Dv, Dk]   receives write-backs / scatters (the caller
 *                              starts it as a copy of pool_in)
 *   read_idx [B]; write_idx [B] or NULL (= read_idx); scatter_idx [B, T] or NULL
 *   A_log, dt_bias [HV]; a [B, T, HV]; bgate [B, T, nh, HV]
 *   out      [B, T, HV, Dv]    rows whose read slot is skipped are not written
 * H must equal HV (no grouping on this path); head h reads q/k head h.
 * ---------------------------------------------------------------------- */
static double softplus_thr20(double x)
{
    return x > 20.0 ? x : log1p(exp(x));
}

void oracle_decode(const double *q, const double *k, const double *v,
                   const double *pool_in, double *pool_out, int pool_size,
                   const int32_t *read_idx, const int32_t *write_idx,
                   const int32_t *scatter_idx,
                   const double *A_log, const double *a, const double *dt_bias,
                   const double *bgate, double scale, double *out,
                   int B, int T, int nh, int H, int HV, int Dk, int Dv,
                   int use_qk_l2norm, int disable_state_update, int nthreads)
{
    int nunits = B * HV;
    int64_t slot_elems = (int64_t)HV * Dv * Dk;
    (void)H;
    if (nthreads <= 0) nthreads = 1;

#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (int unit = 0; unit < nunits; ++unit) {
        int b = unit / HV;
        int h = unit % HV;
        int r = read_idx[b];
        if (r < 0 || r >= pool_size) continue;   /* padding row: nothing at all */

        double *S = (double *)malloc(sizeof(double) * Dk * Dv);
        double *xq = (double *)malloc(sizeof(double) * Dk);
        double *xk = (double *)malloc(sizeof(double) * Dk);
        double *p = (double *)malloc(sizeof(double) * Dv);

        const double *s0 = pool_in + r * slot_elems + (int64_t)h * Dv * Dk;
        for (int i = 0; i < Dk; ++i)
            for (int j = 0; j < Dv; ++j)
                S[(int64_t)i * Dv + j] = s0[(int64_t)j * Dk + i];

        for (int t = 0; t < T; ++t) {
            int64_t bt = (int64_t)b * T + t;
            /* alpha_t = exp(-exp(A_log) * softplus(a_t + dt_bias)) */
            double alpha = exp(-exp(A_log[h]) * softplus_thr20(a[bt * HV + h] + dt_bias[h]));
            for (int64_t e = 0; e < (int64_t)Dk * Dv; ++e) S[e] *= alpha;

            for (int j = 0; j < nh; ++j) {
                const double *kt = k + ((bt * nh + j) * H + h) * Dk;
                const double *vt = v + ((bt * nh + j) * HV + h) * Dv;
                double bta = 1.0 / (1.0 + exp(-bgate[(bt * nh + j) * HV + h]));
                for (int i = 0; i < Dk; ++i) xk[i] = kt[i];
                if (use_qk_l2norm) {
                    double s = 0.0;
                    for (int i = 0; i < Dk; ++i) s += xk[i] * xk[i];
                    double rn = 1.0 / sqrt(s + 1e-6);
                    for (int i = 0; i < Dk; ++i) xk[i] *= rn;
                }
                /* one Householder-style delta sub-step: S += k (beta (v - S^T k))^T */
                for (int jv = 0; jv < Dv; ++jv) {
                    double acc = 0.0;
                    for (int i = 0; i < Dk; ++i) acc += S[(int64_t)i * Dv + jv] * xk[i];
                    p[jv] = acc;
                }
                for (int i = 0; i < Dk; ++i)
                    for (int jv = 0; jv < Dv; ++jv)
                        S[(int64_t)i * Dv + jv] += xk[i] * (bta * (vt[jv] - p[jv]));
            }

            const double *qt = q + (bt * H + h) * Dk;
            for (int i = 0; i < Dk; ++i) xq[i] = qt[i];
            if (use_qk_l2norm) {
                double s = 0.0;
                for (int i = 0; i < Dk; ++i) s += xq[i] * xq[i];
                double rn = 1.0 / sqrt(s + 1e-6);
                for (int i = 0; i < Dk; ++i) xq[i] *= rn;
            }
            double *ot = out + (bt * HV + h) * Dv;
            for (int jv = 0; jv < Dv; ++jv) {
                double acc = 0.0;
                for (int i = 0; i < Dk; ++i) acc += S[(int64_t)i * Dv + jv] * xq[i];
                ot[jv] = scale * acc;
            }

            if (scatter_idx && !disable_state_update) {
                int s = scatter_idx[bt];
                if (s >= 0 && s < pool_size) {
                    double *dst = pool_out + s * slot_elems + (int64_t)h * Dv * Dk;
                    for (int jv = 0; jv < Dv; ++jv)
                        for (int i = 0; i < Dk; ++i)
                            dst[(int64_t)jv * Dk + i] = S[(int64_t)i * Dv + jv];
                }
            }
        }

        if (!scatter_idx && !disable_state_update) {
            int w = write_idx ? write_idx[b] : r;
            if (w >= 0 && w < pool_size) {
                double *dst = pool_out + w * slot_elems + (int64_t)h * Dv * Dk;
                for (int jv = 0; jv < Dv; ++jv)
                    for (int i = 0; i < Dk; ++i)
                        dst[(int64_t)jv * Dk + i] = S[(int64_t)i * Dv + jv];
            }
        }

        free(S);
        free(xq);
        free(xk);
        free(p);
    }
}

/*
 * Causal depthwise conv1d over a ragged token stream with a slot-indexed
 * window pool.
 *
 * Source: "max.nn.legacy.state_space.gated_delta_conv1d_fwd" (description,
 * Parameters and the worked example): input x [N, conv_dim], depthwise
 * weights w [conv_dim, K], pool [max_slots, conv_dim, K-1] addressed by
 * slot_idx[b], ragged offsets [B+1]; the pool is updated in place unless
 * write_state is 0, and the untouched slots keep their values.
 *
 * For request b with tokens [s, e) and slot r, channel c sees the extended
 * sequence
 *     xe = (pool[r, c, 0], ..., pool[r, c, K-2], x[s, c], ..., x[e-1, c])
 * and
 *     y[s + i, c] = sum_{j=0}^{K-1} w[c, j] * xe[i + j]     (0 <= i < e - s)
 * (w[c, K-1] weighs the current token, w[c, 0] the oldest); with write_state
 * slot r receives the last K-1 entries of xe.
 *
 * Readings where the page is silent (listed in the design notes):
 *  - the window is stored oldest first, and weight index K-1 meets the
 *    current token (the causal-convolution convention the example's "last
 *    three inputs" fits);
 *  - a request shorter than K-1 keeps the newest old entries in front of its
 *    inputs (the window slides; it is not zero-filled);
 *  - no activation follows the convolution (the page names none);
 *  - offsets are clamped to [0, N] and a request with e <= s is empty (its
 *    slot is left as it was);
 *  - a slot >= max_slots is skipped: no output row and no pool access;
 *  - every request reads the pool as it was before the call (pool_in) and
 *    writes pool_out; with distinct slots this is the in-place result.
 */
void oracle_conv1d(const double *x, const double *w, const double *pool_in,
                   double *pool_out, const uint32_t *slot_idx,
                   const uint32_t *offsets, double *y, int B, int64_t N,
                   int conv_dim, int K, int max_slots, int write_state)
{
    const int W = K - 1;
    for (int b = 0; b < B; ++b) {
        const int64_t s = clamp_i64((int64_t)offsets[b], 0, N);
        const int64_t e = clamp_i64((int64_t)offsets[b + 1], 0, N);
        const uint32_t r = slot_idx[b];
        if (r >= (uint32_t)max_slots) continue;
        if (e <= s) continue;
        const int64_t len = e - s;
        double *xe = (double *)malloc(sizeof(double) * (size_t)(W + len));
        for (int c = 0; c < conv_dim; ++c) {
            const double *win = pool_in + ((int64_t)r * conv_dim + c) * W;
            for (int j = 0; j < W; ++j) xe[j] = win[j];
            for (int64_t i = 0; i < len; ++i) xe[W + i] = x[(s + i) * conv_dim + c];
            for (int64_t i = 0; i < len; ++i) {
                double acc = 0.0;
                for (int j = 0; j < K; ++j) acc += w[(int64_t)c * K + j] * xe[i + j];
                y[(s + i) * conv_dim + c] = acc;
            }
            if (write_state) {
                double *wout = pool_out + ((int64_t)r * conv_dim + c) * W;
                for (int j = 0; j < W; ++j) wout[j] = xe[len + j];
            }
        }
        free(xe);
    }
}
