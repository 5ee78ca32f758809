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
 * parity pins: see tests/test_oracle_pins.py (sorted top-m, closed-form theta,
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
