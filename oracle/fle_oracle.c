/*
 * CPU oracle for the fused Linear + epilogue path.  TEST INFRASTRUCTURE ONLY.
 *
 * This file is the plain, slow, obviously correct definition that the CUDA
 * library is checked against.  Only the test suite, the package's smoke()
 * entry and the benchmark's CPU-baseline / reference leg may load it.  It
 * shares no code, header, table or constant with the CUDA path, and the CUDA
 * path never calls it.
 *
 * Arithmetic: every input is fp32 (as the pages' nn.Linear problems are);
 * every product and sum is carried in fp64, the dot product runs over k in
 * ascending order, the epilogue is evaluated in fp64 with libm erf/exp, and
 * the result is rounded to fp32 once, at the end.
 *
 * What it computes (the three problems the pages restate):
 *   linear  y[m][n] = b[n] + sum_k x[m][k] * W[n][k]
 *           -- nn.Linear applied to a row-major x [M,K] with weight W [N,K]
 *              and bias b [N] (page "Kimi-K2.6 l2_p98", problem restatement,
 *              step 1; page "Kimi-K2.6 l2_p53", task statement, step 1).
 *   (a)     t = clamp(s*y, lo, hi);  out = t * Phi(t),  Phi(t) = (1+erf(t/sqrt2))/2
 *           -- multiply by the constant, Hardtanh, then GELU in its exact
 *              erf form, in that order (page "Kimi-K2.6 l2_p53", task
 *              statement steps 2-4, and its check of PyTorch's default GELU).
 *   (b)     out = y * sigmoid(y) * s,  sigmoid(y) = 1/(1+exp(-y))
 *           -- Swish, then the scaling factor (page "Kimi-K2.6 l2_p59",
 *              problem analysis, items 2-3 and the combined formula after them).
 *   (c)     p_j = (1/k) sum_{t<k} y[m][j*stride + t]  for j < P,
 *           P = floor((N - k)/stride) + 1  (AvgPool1d, no padding, floor mode),
 *           g_j = s * GELU(p_j),  out[m] = max_j g_j
 *           -- AvgPool1d(k) over the feature axis, GELU, scale, maximum over
 *              dim 1 (page "Kimi-K2.6 l2_p98", problem restatement steps 2-5,
 *              including its output-length check for N=8192, k=16).
 *   none    out = y  (the Linear alone; used to check the contraction itself).
 *
 * Option (a), (c): GELU in its tanh form instead of the erf form,
 *           GELU_tanh(v) = v/2 * (1 + tanh(sqrt(2/pi) * (v + 0.044715 v^3)))
 *           -- the approximation page "Kimi-K2.6 l2_p53" writes into its first
 *              fused elementwise kernel and then weighs against the exact form
 *              (gelu_tanh = 1 below).
 *
 * Build: gcc -O2 -fopenmp -fPIC -shared (no -ffast-math: the fp64
 * evaluation must not be reassociated).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Epilogue selectors of the oracle (its own numbering, not the library's). */
#define ORC_EPI_SCALE_HARDTANH_GELU 0
#define ORC_EPI_SWISH_SCALE 1
#define ORC_EPI_AVGPOOL_GELU_SCALE_ROWMAX 2
#define ORC_EPI_NONE 3

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Standard normal CDF, Phi(v) = (1 + erf(v / sqrt 2)) / 2. */
static double orc_phi(double v) { return 0.5 * (1.0 + erf(v / sqrt(2.0))); }

/* Exact GELU: v * Phi(v) (PyTorch's default approximate='none'). */
double orc_gelu(double v) { return v * orc_phi(v); }

/* GELU in its tanh form: v/2 * (1 + tanh(sqrt(2/pi) * (v + 0.044715 v^3))). */
double orc_gelu_tanh(double v) {
    const double c = sqrt(2.0 / acos(-1.0));
    return 0.5 * v * (1.0 + tanh(c * (v + 0.044715 * v * v * v)));
}

/* The GELU of the selected form (0: erf, 1: tanh). */
static double orc_gelu_form(double v, int gelu_tanh) { return gelu_tanh ? orc_gelu_tanh(v) : orc_gelu(v); }

/* Epilogue (a) on one linear output. */
double orc_scale_hardtanh_gelu_form(double y, double s, double lo, double hi, int gelu_tanh) {
    double t = s * y;
    t = fmin(fmax(t, lo), hi);
    return orc_gelu_form(t, gelu_tanh);
}

double orc_scale_hardtanh_gelu(double y, double s, double lo, double hi) {
    return orc_scale_hardtanh_gelu_form(y, s, lo, hi, 0);
}

/* Epilogue (b) on one linear output. */
double orc_swish_scale(double y, double s) {
    double sig = 1.0 / (1.0 + exp(-y));
    return (y * sig) * s;
}

/* Number of AvgPool1d windows over a length-N row (padding 0, floor mode). */
int64_t orc_pool_windows(int64_t N, int64_t k, int64_t stride) {
    if (k <= 0 || stride <= 0 || N < k) return 0;
    return (N - k) / stride + 1;
}

/* Epilogue (c) on one full linear row y[0..N). */
double orc_pool_gelu_scale_max_form(const double* yrow, int64_t N, int64_t k,
                                    int64_t stride, double s, int gelu_tanh) {
    int64_t P = orc_pool_windows(N, k, stride);
    double best = -INFINITY;
    for (int64_t j = 0; j < P; ++j) {
        double acc = 0.0;
        for (int64_t t = 0; t < k; ++t) acc += yrow[j * stride + t];
        double p = acc / (double)k;
        double g = s * orc_gelu_form(p, gelu_tanh);
        if (g > best) best = g;
    }
    return best;
}

double orc_pool_gelu_scale_max(const double* yrow, int64_t N, int64_t k,
                               int64_t stride, double s) {
    return orc_pool_gelu_scale_max_form(yrow, N, k, stride, s, 0);
}

/* The linear part for a list of rows: y[r*N + n] for r < nrows. */
void orc_linear_rows(const float* x, const float* W, const float* b,
                     int64_t M, int64_t K, int64_t N,
                     const int64_t* rows, int64_t nrows, double* y) {
    (void)M;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t r = 0; r < nrows; ++r) {
        for (int64_t n = 0; n < N; ++n) {
            const float* xr = x + rows[r] * K;
            const float* wn = W + n * K;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += (double)xr[k] * (double)wn[k];
            if (b) acc += (double)b[n];
            y[r * N + n] = acc;
        }
    }
}

/*
 * The whole path for a list of rows.  out has nrows*N floats for kinds (a),
 * (b) and none, and nrows floats for (c).  y_scratch, when not NULL, must hold
 * nrows*N doubles and receives the linear outputs.  gelu_tanh selects the
 * tanh form of GELU for (a) and (c).  Returns 0, or -1 on a shape/argument
 * error (no windows for (c), unknown kind, bad row index).
 */
int orc_forward_rows(const float* x, const float* W, const float* b,
                     int64_t M, int64_t K, int64_t N, int kind,
                     double scale, double clamp_lo, double clamp_hi,
                     int64_t pool_k, int64_t pool_stride, int gelu_tanh,
                     const int64_t* rows, int64_t nrows,
                     float* out, double* y_scratch) {
    if (M < 0 || K < 0 || N <= 0 || nrows < 0) return -1;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= M) return -1;
    if (kind == ORC_EPI_AVGPOOL_GELU_SCALE_ROWMAX &&
        orc_pool_windows(N, pool_k, pool_stride) <= 0)
        return -1;
    if (kind < 0 || kind > ORC_EPI_NONE) return -1;

    double* y = y_scratch;
    if (!y) {
        y = (double*)malloc((size_t)(nrows > 0 ? nrows : 1) * (size_t)N * sizeof(double));
        if (!y) return -1;
    }
    orc_linear_rows(x, W, b, M, K, N, rows, nrows, y);

#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < nrows; ++r) {
        const double* yr = y + r * N;
        if (kind == ORC_EPI_AVGPOOL_GELU_SCALE_ROWMAX) {
            out[r] = (float)orc_pool_gelu_scale_max_form(yr, N, pool_k, pool_stride, scale, gelu_tanh);
            continue;
        }
        for (int64_t n = 0; n < N; ++n) {
            double o;
            if (kind == ORC_EPI_SCALE_HARDTANH_GELU)
                o = orc_scale_hardtanh_gelu_form(yr[n], scale, clamp_lo, clamp_hi, gelu_tanh);
            else if (kind == ORC_EPI_SWISH_SCALE)
                o = orc_swish_scale(yr[n], scale);
            else
                o = yr[n];
            out[r * N + n] = (float)o;
        }
    }
    if (!y_scratch) free(y);
    return 0;
}
