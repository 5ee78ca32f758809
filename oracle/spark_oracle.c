/*
 * spark_oracle.c -- plain, slow, fp64 CPU restatement of the Spark FFN and of
 * statistical top-k.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes or
 * calls this file; only the test suite, the smoke check and the CPU-baseline leg
 * of the benchmark load it.  It shares no code, header, table or helper with the
 * CUDA path.
 *
 * Source of every step: the paper notes page "Spark Transformer: Reactivating
 * Sparsity in FFN and Attention" (NeurIPS 2025, arXiv 2506.06644), section
 * 方法详解 / 关键设计:
 *   - "Spark FFN": split q into q[:r] and q[r:]; the predictor K1^T q[:r];
 *     top-k selects k neurons; only the selected columns of K2 and rows of V are
 *     used; Spark-FFN(q) = V . (sigma(Top_k(K1^T q[:r])) (.) (K2^T q[r:])).
 *   - "Statistical Top-k": theta(x,k) = mean(x) + std(x) . Q(1 - k/d) with Q the
 *     standard-normal quantile, followed by Soft-Threshold(x, theta) =
 *     max{x - theta, 0}; cost about 2d FLOPs, "like LayerNorm".
 *
 * Readings taken where the page is silent (each is repeated at its use):
 *   - std is the population standard deviation (divide by d), as LayerNorm does.
 *   - sigma(.) is GELU in its tanh form; the exact-erf GELU is a switch.
 *   - Top_k(x) is read as SoftThreshold(x, theta(x,k)) element by element: a
 *     neuron is active iff x_i > theta (strict); no top-up or truncation to k.
 *   - a row with zero spread has theta = mean, so no neuron is active.
 *
 * Arithmetic: every value is widened to double (bf16 and fp32 inputs widen
 * exactly); sums run in plain index order; no blocking, fusion or reordering.
 * Build with -ffp-contract=off so that a*b+c is never fused.
 *
 * Spark Attention (one decoding position) follows the same page, item "Spark
 * Attention"; its readings are at oracle_spark_attention.
 *
 * parity pins: see tests/test_oracle_pins.py and tests/test_oracle_attention_pins.py
 * (sorted top-m, closed-form theta,
 * textbook quantiles, GELU vs x*Phi(x), invariants, degenerate rows, reduction
 * of the FFN to GELU(SoftThreshold) for identity-like K2/V).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 is the top 16 bits of an IEEE binary32; widening is exact. */
double oracle_bf16_to_f64(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Standard normal upper tail P(Z > z) = erfc(z / sqrt 2) / 2 (host libm). */
double oracle_normal_upper_tail(double z)
{
    return 0.5 * erfc(z / sqrt(2.0));
}

/*
 * Q(1 - k/d): the z with P(Z > z) = k/d, found by plain bisection on the upper
 * tail (monotone decreasing in z).  "Statistical Top-k": Q is the
 * standard-normal quantile function evaluated at 1 - k/d.
 * Returns NAN unless 0 < k < d.
 */
double oracle_topk_quantile(double k, double d)
{
    if (!(k > 0.0) || !(k < d)) return NAN;
    double tail = k / d;
    double lo = -40.0, hi = 40.0; /* upper_tail(lo) ~ 1 > tail > upper_tail(hi) ~ 0 */
    for (int it = 0; it < 400 && hi - lo > 1e-15; ++it) {
        double mid = 0.5 * (lo + hi);
        if (oracle_normal_upper_tail(mid) > tail)
            lo = mid; /* too much mass above mid: threshold must move up */
        else
            hi = mid;
    }
    return 0.5 * (lo + hi);
}

/* Population mean and standard deviation of x[0..d), two passes. */
void oracle_row_stats(const double *x, long d, double *mean_out, double *std_out)
{
    double sum = 0.0;
    for (long i = 0; i < d; ++i) sum += x[i];
    double mean = sum / (double)d;
    double ss = 0.0;
    for (long i = 0; i < d; ++i) {
        double c = x[i] - mean;
        ss += c * c;
    }
    *mean_out = mean;
    *std_out = sqrt(ss / (double)d);
}

/* theta(x,k) = mean(x) + std(x) * Q(1 - k/d)  ("Statistical Top-k"). */
double oracle_theta(const double *x, long d, long k, double *mean_out, double *std_out)
{
    double mean, sd;
    oracle_row_stats(x, d, &mean, &sd);
    if (mean_out) *mean_out = mean;
    if (std_out) *std_out = sd;
    return mean + sd * oracle_topk_quantile((double)k, (double)d);
}

/* GELU, tanh form: 0.5 s (1 + tanh(sqrt(2/pi) (s + 0.044715 s^3))). */
double oracle_gelu_tanh(double s)
{
    const double c = sqrt(2.0 / M_PI);
    return 0.5 * s * (1.0 + tanh(c * (s + 0.044715 * s * s * s)));
}

/* GELU, exact form: s * Phi(s) = s * erfc(-s / sqrt 2) / 2. */
double oracle_gelu_erf(double s)
{
    return s * 0.5 * erfc(-s / sqrt(2.0));
}

static double gelu_of_kind(double s, int kind)
{
    return kind == 1 ? oracle_gelu_erf(s) : oracle_gelu_tanh(s);
}

/*
 * Standalone statistical top-k with soft threshold on fp32 rows:
 * out[row][i] = max(x[row][i] - theta_row, 0).
 * theta/mean/std outputs are optional (NULL to skip).  Rows run in parallel
 * when n_threads > 1; each row is computed exactly as above.
 * Returns 0, or -1 when 0 < k < d does not hold.
 */
int oracle_stat_topk(const float *x, long rows, long d, long k, double *out,
                     double *theta_out, double *mean_out, double *std_out, int n_threads)
{
    if (!(k > 0 && k < d) || rows < 0) return -1;
    if (n_threads < 1) n_threads = 1;
#pragma omp parallel for schedule(static) num_threads(n_threads)
    for (long row = 0; row < rows; ++row) {
        double *xr = (double *)malloc(sizeof(double) * (size_t)d);
        for (long i = 0; i < d; ++i) xr[i] = (double)x[row * d + i];
        double mean, sd;
        double theta = oracle_theta(xr, d, k, &mean, &sd);
        for (long i = 0; i < d; ++i) {
            double s = xr[i] - theta;
            out[row * d + i] = s > 0.0 ? s : 0.0;
        }
        if (theta_out) theta_out[row] = theta;
        if (mean_out) mean_out[row] = mean;
        if (std_out) std_out[row] = sd;
        free(xr);
    }
    return 0;
}

/*
 * Huber-smoothed statistical top-k ("Statistical Top-k", Theorem 3.2: after
 * smoothing with a Huber function the operator is continuously
 * differentiable).  Reading: the kink of Soft-Threshold, max{z, 0} at z = 0,
 * is replaced by the Huber-smoothed ramp of width delta >= 0
 *   rho(z) = 0                 for z <= 0
 *          = z^2 / (2 delta)   for 0 < z < delta
 *          = z - delta / 2     for z >= delta
 * (delta = 0: rho(z) = max{z, 0}, the plain operator), with z = x - theta(x),
 * theta(x) = mean(x) + std(x) Q(1 - k/d), population std, as everywhere here.
 */
static double huber_ramp(double z, double delta)
{
    if (z <= 0.0) return 0.0;
    if (z < delta) return z * z / (2.0 * delta);
    return z - 0.5 * delta;
}

/* rho'(z): 0, z / delta, 1 on the three pieces (0 at the kink when delta = 0). */
static double huber_ramp_slope(double z, double delta)
{
    if (z <= 0.0) return 0.0;
    if (z < delta) return z / delta;
    return 1.0;
}

/* Forward on fp64 rows: out = rho(x - theta(x)).  Returns 0, or -1 unless
 * 0 < k < d and delta >= 0. */
int oracle_stat_topk_huber(const double *x, long rows, long d, long k, double delta, double *out,
                           double *theta_out)
{
    if (!(k > 0 && k < d) || rows < 0 || !(delta >= 0.0)) return -1;
    for (long row = 0; row < rows; ++row) {
        const double *xr = x + row * d;
        double mean, sd;
        double theta = oracle_theta(xr, d, k, &mean, &sd);
        for (long i = 0; i < d; ++i) out[row * d + i] = huber_ramp(xr[i] - theta, delta);
        if (theta_out) theta_out[row] = theta;
    }
    return 0;
}

/*
 * Backward (vector-Jacobian product) of the forward above for an upstream
 * gradient g = dL/dout.  By the chain rule, with w_i = g_i rho'(z_i) and
 * W = sum_i w_i,
 *   dL/dx_j = w_j - W dtheta/dx_j,
 *   dtheta/dx_j = 1/d + Q(1 - k/d) (x_j - mean) / (d std)
 * (d mean/dx_j = 1/d; d std/dx_j = (x_j - mean) / (d std)).  A row with zero
 * spread has every z = 0, so w = 0 and the result is 0 (the std term is not
 * evaluated there).  Returns 0, or -1 on invalid arguments.
 */
int oracle_stat_topk_huber_backward(const double *x, const double *g, long rows, long d, long k, double delta,
                                    double *grad_x)
{
    if (!(k > 0 && k < d) || rows < 0 || !(delta >= 0.0)) return -1;
    const double Q = oracle_topk_quantile((double)k, (double)d);
    double *w = (double *)malloc(sizeof(double) * (size_t)d);
    for (long row = 0; row < rows; ++row) {
        const double *xr = x + row * d;
        const double *gr = g + row * d;
        double mean, sd;
        double theta = oracle_theta(xr, d, k, &mean, &sd);
        double W = 0.0;
        for (long i = 0; i < d; ++i) {
            w[i] = gr[i] * huber_ramp_slope(xr[i] - theta, delta);
            W += w[i];
        }
        for (long j = 0; j < d; ++j) {
            double dtheta = 1.0 / (double)d;
            if (sd > 0.0) dtheta += Q * (xr[j] - mean) / ((double)d * sd);
            grad_x[row * d + j] = w[j] - W * dtheta;
        }
    }
    free(w);
    return 0;
}

/*
 * Statistical top-k with soft threshold on causally masked score rows (the
 * attention-shaped case of "Statistical Top-k" under a causal mask; "Spark
 * Attention": each token attends to at most k_attn tokens, so the work is
 * min{k_attn, n_ctx} per query).
 *   Row i is query number i mod n_q of its head, at position
 *   pos = offset + (i mod n_q); it sees keys 0..pos, i.e. the first
 *   n = min(d, pos + 1) entries of the row; the rest are masked.
 *   If k < n: theta = mean + std * Q(1 - k/n) over the n visible entries
 *     (population std), out[j] = max(x[j] - theta, 0) for j < n.
 *   If k >= n: every visible entry is kept (the threshold formula has no
 *     finite value there, Q(1 - k/n) = -inf): theta = -inf and out[j] = x[j]
 *     for j < n (the scores pass through unshifted).
 *   Masked entries (j >= n) are 0 in both cases.
 * theta_out optional (NULL to skip).  Returns 0, or -1 unless k >= 1, n_q >= 1,
 * offset >= 0, d >= 1, rows >= 0.
 */
int oracle_stat_topk_causal(const float *x, long rows, long d, long k, long n_q, long offset, double *out,
                            double *theta_out, int n_threads)
{
    if (k < 1 || n_q < 1 || offset < 0 || d < 1 || rows < 0) return -1;
    if (n_threads < 1) n_threads = 1;
#pragma omp parallel for schedule(static) num_threads(n_threads)
    for (long row = 0; row < rows; ++row) {
        const long pos = offset + row % n_q;
        const long n = pos + 1 < d ? pos + 1 : d;
        double *xr = (double *)malloc(sizeof(double) * (size_t)n);
        for (long j = 0; j < n; ++j) xr[j] = (double)x[row * d + j];
        double theta = -INFINITY;
        if (k < n) {
            double mean, sd;
            theta = oracle_theta(xr, n, k, &mean, &sd);
            for (long j = 0; j < n; ++j) {
                double s = xr[j] - theta;
                out[row * d + j] = s > 0.0 ? s : 0.0;
            }
        } else {
            for (long j = 0; j < n; ++j) out[row * d + j] = xr[j];
        }
        for (long j = n; j < d; ++j) out[row * d + j] = 0.0;
        if (theta_out) theta_out[row] = theta;
        free(xr);
    }
    return 0;
}

/*
 * Spark FFN forward over T tokens ("Spark FFN" in 关键设计):
 *   x_i   = sum_{j<r} K1[i][j] q[j]                       (predictor, K1 is d_ff x r)
 *   theta = mean(x) + std(x) Q(1 - k/d_ff)                 (statistical top-k)
 *   A     = { i : x_i > theta }                            (soft-threshold support)
 *   g_i   = GELU(max(x_i - theta, 0))                      (sigma after Top_k)
 *   a_i   = sum_{j<d_model-r} K2[i][j] q[r+j]              (K2 is d_ff x (d_model-r))
 *   out   = sum_{i in A} g_i a_i V[i][:]                   (V is d_ff x d_model)
 * Inputs are bf16 bit patterns, row-major.  out is fp64 [T][d_model].
 *
 * override_active (optional, [T][d_ff] bytes): when given, A is taken from it
 * instead of from x > theta; g_i still uses max(x_i - theta, 0).  This lets the
 * caller evaluate the output on another implementation's active set.
 * x_out [T][d_ff], theta/mean/std [T], active_out [T][d_ff] are optional.
 * gelu_kind: 0 = tanh form, 1 = exact erf form.
 * Returns 0, or -1 on invalid sizes (need 0<r<d_model, 0<k<d_ff, T>=0).
 */
int oracle_spark_ffn(const uint16_t *q, const uint16_t *K1, const uint16_t *K2,
                     const uint16_t *V, long T, long d_model, long r, long d_ff, long k,
                     int gelu_kind, const uint8_t *override_active, double *out,
                     double *x_out, double *theta_out, double *mean_out, double *std_out,
                     uint8_t *active_out, int n_threads)
{
    if (!(r > 0 && r < d_model) || !(k > 0 && k < d_ff) || T < 0) return -1;
    if (n_threads < 1) n_threads = 1;
    const long d2 = d_model - r;
#pragma omp parallel for schedule(static) num_threads(n_threads)
    for (long t = 0; t < T; ++t) {
        const uint16_t *qt = q + t * d_model;
        double *x = (double *)malloc(sizeof(double) * (size_t)d_ff);
        /* predictor: x = K1^T q[:r] in the page's notation (K1 stored d_ff x r) */
        for (long i = 0; i < d_ff; ++i) {
            double acc = 0.0;
            for (long j = 0; j < r; ++j)
                acc += oracle_bf16_to_f64(K1[i * r + j]) * oracle_bf16_to_f64(qt[j]);
            x[i] = acc;
        }
        double mean, sd;
        double theta = oracle_theta(x, d_ff, k, &mean, &sd);
        double *o = out + t * d_model;
        for (long c = 0; c < d_model; ++c) o[c] = 0.0;
        for (long i = 0; i < d_ff; ++i) {
            int active = override_active ? (override_active[t * d_ff + i] != 0) : (x[i] > theta);
            if (active_out) active_out[t * d_ff + i] = (uint8_t)(x[i] > theta);
            if (!active) continue;
            double s = x[i] - theta;
            if (s < 0.0) s = 0.0;
            double g = gelu_of_kind(s, gelu_kind);
            double a = 0.0;
            for (long j = 0; j < d2; ++j)
                a += oracle_bf16_to_f64(K2[i * d2 + j]) * oracle_bf16_to_f64(qt[r + j]);
            double h = g * a;
            for (long c = 0; c < d_model; ++c) o[c] += h * oracle_bf16_to_f64(V[i * d_model + c]);
        }
        if (x_out)
            for (long i = 0; i < d_ff; ++i) x_out[t * d_ff + i] = x[i];
        if (theta_out) theta_out[t] = theta;
        if (mean_out) mean_out[t] = mean;
        if (std_out) std_out[t] = sd;
        free(x);
    }
    return 0;
}

/* softplus(a) = log(1 + e^a), evaluated without overflow. */
double oracle_softplus(double a)
{
    return a > 0.0 ? a + log1p(exp(-a)) : log1p(exp(a));
}

/*
 * Spark Attention for one decoding position ("Spark Attention" in 关键设计): the
 * key vectors are split like the FFN's K into K1 (the first r dimensions, used
 * to predict) and K2 (the rest); each query attends to at most k_attn keys
 * chosen by statistical top-k on the predictor scores; sigma_1 = softmax and
 * sigma_2 = softplus.  For query head h (key/value head g = h / (n_heads /
 * n_kv_heads)):
 *   s_j   = scale * sum_{i<r} K[g][j][i] q[h][i]                (j < n_ctx)
 *   theta = mean(s) + std(s) Q(1 - k_attn/n_ctx); A = { j : s_j > theta }
 *           (k_attn >= n_ctx: every key, the min{k_attn, n_ctx} of the FLOP count)
 *   p_j   = exp(s_j) / sum_{l in A} exp(s_l)                       (j in A)
 *   a_j   = sum_{i<d_head-r} K[g][j][r+i] q[h][r+i]
 *   out[h] = sum_{j in A} p_j softplus(a_j) V[g][j][:]
 * Readings: the softmax runs over the selected keys only (a softmax over all
 * n_ctx soft-thresholded scores would give every unselected key the weight
 * e^0 and attend densely); softmax is shift-invariant, so it is the same on s_j
 * and on the soft-thresholded s_j - theta; `scale` is the attention temperature,
 * which the page leaves open (callers pass 1/sqrt(d_head) by default); an
 * empty A (zero spread) gives out = 0.
 * Layouts: q [n_heads][d_head], K and V [n_kv_heads][n_ctx][d_head] bf16 bits;
 * out fp64 [n_heads][d_head].  s_out [n_heads][n_ctx], theta_out [n_heads],
 * active_out [n_heads][n_ctx] are optional; override_active ([n_heads][n_ctx])
 * replaces A (the weights are then renormalised over the given set).
 * Returns 0, or -1 on invalid sizes.
 */
int oracle_spark_attention(const uint16_t *q, const uint16_t *K, const uint16_t *V, long n_heads,
                           long n_kv_heads, long n_ctx, long d_head, long r, long k_attn, double scale,
                           const uint8_t *override_active, double *out, double *s_out, double *theta_out,
                           uint8_t *active_out, int n_threads)
{
    if (n_heads < 1 || n_kv_heads < 1 || n_heads % n_kv_heads != 0 || n_ctx < 1 || !(r > 0 && r < d_head) ||
        k_attn < 1)
        return -1;
    if (n_threads < 1) n_threads = 1;
    const long group = n_heads / n_kv_heads;
#pragma omp parallel for schedule(static) num_threads(n_threads)
    for (long h = 0; h < n_heads; ++h) {
        const long g = h / group;
        const uint16_t *qh = q + h * d_head;
        const uint16_t *Kg = K + g * n_ctx * d_head;
        const uint16_t *Vg = V + g * n_ctx * d_head;
        double *s = (double *)malloc(sizeof(double) * (size_t)n_ctx);
        for (long j = 0; j < n_ctx; ++j) {
            double acc = 0.0;
            for (long i = 0; i < r; ++i)
                acc += oracle_bf16_to_f64(Kg[j * d_head + i]) * oracle_bf16_to_f64(qh[i]);
            s[j] = scale * acc;
        }
        double theta = -INFINITY;
        if (k_attn < n_ctx) theta = oracle_theta(s, n_ctx, k_attn, NULL, NULL);
        double smax = -INFINITY;
        for (long j = 0; j < n_ctx; ++j) {
            int act = override_active ? (override_active[h * n_ctx + j] != 0) : (s[j] > theta);
            if (active_out) active_out[h * n_ctx + j] = (uint8_t)(s[j] > theta);
            if (act && s[j] > smax) smax = s[j];
        }
        double *o = out + h * d_head;
        for (long c = 0; c < d_head; ++c) o[c] = 0.0;
        double z = 0.0;
        for (long j = 0; j < n_ctx; ++j) {
            int act = override_active ? (override_active[h * n_ctx + j] != 0) : (s[j] > theta);
            if (!act) continue;
            double w = exp(s[j] - smax);
            double a = 0.0;
            for (long i = 0; i < d_head - r; ++i)
                a += oracle_bf16_to_f64(Kg[j * d_head + r + i]) * oracle_bf16_to_f64(qh[r + i]);
            double f = w * oracle_softplus(a);
            for (long c = 0; c < d_head; ++c) o[c] += f * oracle_bf16_to_f64(Vg[j * d_head + c]);
            z += w;
        }
        if (z > 0.0)
            for (long c = 0; c < d_head; ++c) o[c] /= z;
        if (s_out)
            for (long j = 0; j < n_ctx; ++j) s_out[h * n_ctx + j] = s[j];
        if (theta_out) theta_out[h] = theta;
        free(s);
    }
    return 0;
}

/*
 * RMSNorm with unit gain used between the layers of a decoder stack:
 * y = h / sqrt(mean(h^2) + eps).  Not from the pages: it is the standard
 * pre-norm of a Gemma-style residual stack, used to chain layers.
 */
void oracle_rmsnorm(const double *h, long d, double eps, double *y)
{
    double ss = 0.0;
    for (long i = 0; i < d; ++i) ss += h[i] * h[i];
    double inv = 1.0 / sqrt(ss / (double)d + eps);
    for (long i = 0; i < d; ++i) y[i] = h[i] * inv;
}

int oracle_num_threads_available(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
