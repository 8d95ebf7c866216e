/*
 * oracle.c -- plain CPU oracle for activation-sparse FFN decode.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg load this file's library.  The CUDA library
 * never calls it, and it shares no code, header or table with the CUDA path.
 *
 * What it computes, step by step, in double precision (every stored fp16 or
 * fp32 parameter is first converted exactly to double):
 *
 *   predictor   h_j = max(0, sum_k x_k A[k][j])          (k ascending)
 *               z_i = sum_j h_j B[j][i] + c_i              (j ascending)
 *               i is predicted active  iff  sigmoid(z_i) > 0.5  iff  z_i > 0
 *   FFN         ReLU : a_i = max(0, W_up[i].x + b_i)
 *               ReGLU: a_i = max(0, W_gate[i].x + b_i) * (W_up[i].x)
 *               y_j = sum_{i in S, ascending} a_i W_down[j][i]
 *
 * Sources.  Only predicted-active neurons are computed, inactive ones are
 * skipped: 53ai.com "sparsity for LLM inference" page, PowerInfer overview
 * (section "概述") and the single-layer example (section "单层计算优化").
 * Inactive rows contribute exactly zero to the down projection, which is why
 * they need not be read: same page, section "激活稀疏" (activation sparsity).
 * A small per-layer MLP predicts the active MLP neurons: same page, section
 * "自适应稀疏预测器" (adaptive sparse predictor).  The predictor's form here is
 * a rank-r two-layer MLP, sigmoid(relu(x.A).B + c), thresholded at 0.5.
 * Because sigmoid is strictly increasing with sigmoid(0) = 1/2, the threshold
 * is evaluated as z > 0 (no exponential is taken); a tie z == 0 and a NaN are
 * inactive.
 *
 * Layouts are PyTorch's: w_up/w_gate [n][d], w_down [d][n], A [d][r],
 * B [r][n], b/c [n], x [d].  dt selects the stored element type
 * (0 = fp32, 1 = IEEE fp16 bits).  nthreads > 1 runs independent outputs in
 * parallel with OpenMP; every output's sum keeps the order above.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F32 = 0, OR_F16 = 1 };
enum { OR_RELU = 0, OR_REGLU = 1 };

/* IEEE 754 binary16 -> double, exact: sign, 5-bit exponent (bias 15), 10-bit fraction. */
static double half_to_double(uint16_t bits) {
    int sign = bits >> 15;
    int expo = (bits >> 10) & 0x1f;
    int frac = bits & 0x3ff;
    double v;
    if (expo == 0)
        v = ldexp((double)frac, -24); /* subnormal: frac * 2^-14 * 2^-10 */
    else if (expo == 31)
        v = frac ? NAN : INFINITY;
    else
        v = ldexp((double)(frac | 0x400), expo - 25); /* 1.frac * 2^(expo-15) */
    return sign ? -v : v;
}

static double g_half_table[65536];
static int g_half_table_ready = 0;

static void init_table(void) {
    if (g_half_table_ready) return;
    for (int i = 0; i < 65536; ++i) g_half_table[i] = half_to_double((uint16_t)i);
    g_half_table_ready = 1;
}

static inline double ld(const void *p, int dt, size_t i) {
    return dt == OR_F16 ? g_half_table[((const uint16_t *)p)[i]] : (double)((const float *)p)[i];
}

static void set_threads(int nthreads) {
#ifdef _OPENMP
    omp_set_num_threads(nthreads > 0 ? nthreads : 1);
#else
    (void)nthreads;
#endif
}

/* Convert `count` stored elements to double (exposes the decoding for its own pin). */
void oracle_decode(const void *src, int dt, int64_t count, double *dst) {
    init_table();
    for (int64_t i = 0; i < count; ++i) dst[i] = ld(src, dt, (size_t)i);
}

/* Predictor: h [r], z [n], mask [n] (1 = predicted active).  Returns |S|. */
int32_t oracle_predictor(int32_t d, int32_t r, int32_t n, int32_t dt, const void *x, const void *A,
                         const void *B, const void *c, double *h, double *z, uint8_t *mask,
                         int32_t nthreads) {
    init_table();
    set_threads(nthreads);
#pragma omp parallel for schedule(static)
    for (int32_t j = 0; j < r; ++j) {
        double u = 0.0;
        for (int32_t k = 0; k < d; ++k) u += ld(x, dt, k) * ld(A, dt, (size_t)k * r + j);
        h[j] = u > 0.0 ? u : 0.0;
    }
#pragma omp parallel for schedule(static)
    for (int32_t i = 0; i < n; ++i) {
        double s = 0.0;
        for (int32_t j = 0; j < r; ++j) s += h[j] * ld(B, dt, (size_t)j * n + i);
        z[i] = s + ld(c, dt, i);
    }
    int32_t count = 0;
    for (int32_t i = 0; i < n; ++i) {
        mask[i] = z[i] > 0.0 ? 1 : 0; /* NaN compares false: inactive */
        count += mask[i];
    }
    return count;
}

/* Pre-activation of the ReLU'd projection for every neuron: g_i = W[i].x + b_i with
 * W = w_up (ReLU) or w_gate (ReGLU).  The exact active set is {i : g_i > 0}. */
void oracle_preact(int32_t d, int32_t n, int32_t act, int32_t dt, const void *x, const void *w_up,
                   const void *w_gate, const void *bias, double *g, int32_t nthreads) {
    init_table();
    set_threads(nthreads);
    const void *w = act == OR_REGLU ? w_gate : w_up;
#pragma omp parallel for schedule(static)
    for (int32_t i = 0; i < n; ++i) {
        double s = 0.0;
        for (int32_t k = 0; k < d; ++k) s += ld(w, dt, (size_t)i * d + k) * ld(x, dt, k);
        g[i] = s + ld(bias, dt, i);
    }
}

/* FFN restricted to the neurons with mask[i] != 0: a [n] (0 outside the set), y [d]. */
void oracle_ffn_masked(int32_t d, int32_t n, int32_t act, int32_t dt, const void *x, const void *w_up,
                       const void *w_gate, const void *bias, const void *w_down, const uint8_t *mask,
                       double *a, double *y, int32_t nthreads) {
    init_table();
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 16)
    for (int32_t i = 0; i < n; ++i) {
        if (!mask[i]) {
            a[i] = 0.0;
            continue;
        }
        double up = 0.0;
        for (int32_t k = 0; k < d; ++k) up += ld(w_up, dt, (size_t)i * d + k) * ld(x, dt, k);
        if (act == OR_RELU) {
            double g = up + ld(bias, dt, i);
            a[i] = g > 0.0 ? g : 0.0;
        } else {
            double g = 0.0;
            for (int32_t k = 0; k < d; ++k) g += ld(w_gate, dt, (size_t)i * d + k) * ld(x, dt, k);
            g += ld(bias, dt, i);
            a[i] = (g > 0.0 ? g : 0.0) * up;
        }
    }
    /* active list in ascending neuron order */
    int32_t *list = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n > 0 ? n : 1));
    int32_t k = 0;
    for (int32_t i = 0; i < n; ++i)
        if (mask[i]) list[k++] = i;
#pragma omp parallel for schedule(static)
    for (int32_t j = 0; j < d; ++j) {
        double s = 0.0;
        for (int32_t t = 0; t < k; ++t) s += a[list[t]] * ld(w_down, dt, (size_t)j * n + list[t]);
        y[j] = s;
    }
    free(list);
}

/* One decode step: predictor, then the FFN over the predicted set.  Returns |S|. */
int32_t oracle_forward(int32_t d, int32_t n, int32_t r, int32_t act, int32_t dt, const void *x,
                       const void *w_up, const void *w_gate, const void *bias, const void *w_down,
                       const void *A, const void *B, const void *c, double *h, double *z, uint8_t *mask,
                       double *a, double *y, int32_t nthreads) {
    int32_t count = oracle_predictor(d, r, n, dt, x, A, B, c, h, z, mask, nthreads);
    oracle_ffn_masked(d, n, act, dt, x, w_up, w_gate, bias, w_down, mask, a, y, nthreads);
    return count;
}

/*
 * Weight-only int8 and int4 rows (a NEXT step of the method: PowerInfer runs its weights
 * in INT4 on the smaller PC, 53ai.com page, section on evaluation; only the rows'
 * storage changes, the arithmetic stays that of the FFN above).
 *
 * Quantisation of `units` units of `len` elements each (element k of unit i at
 * w[i*unit_stride + k*elem_stride]) to symmetric codes in [-qmax, qmax] (qmax = 127 for
 * int8, 7 for int4): in IEEE fp32, scale_i = max_k |w_ik| / qmax and
 * q_ik = round-to-nearest-even(w_ik / scale_i), clamped to [-qmax, qmax]; an all-zero
 * unit has scale 0 and codes 0.  The decision is taken in fp32 so that any fp32
 * implementation of the same rule gives the same codes.  q is unit-major, one code per
 * byte whatever qmax.
 */
void oracle_quantize(int32_t units, int32_t len, int32_t dt, const void *w, int64_t unit_stride,
                     int64_t elem_stride, int32_t qmax, int8_t *q, float *scale) {
    init_table();
    for (int32_t i = 0; i < units; ++i) {
        float amax = 0.0f;
        for (int32_t k = 0; k < len; ++k) {
            const float v = fabsf((float)ld(w, dt, (size_t)(i * unit_stride + k * elem_stride)));
            if (v > amax) amax = v;
        }
        const float s = amax / (float)qmax;
        scale[i] = s;
        for (int32_t k = 0; k < len; ++k) {
            int32_t c = 0;
            if (s > 0.0f) {
                const float v = (float)ld(w, dt, (size_t)(i * unit_stride + k * elem_stride));
                c = (int32_t)rintf(v / s);
                c = c > qmax ? qmax : (c < -qmax ? -qmax : c);
            }
            q[(size_t)i * len + k] = (int8_t)c;
        }
    }
}

/* The FFN of oracle_ffn_masked with quantised rows: every weight is q * scale (exact in
 * double).  q_up/q_gate [n][d] with scales [n]; q_down [n][d] neuron-major (neuron i's
 * down row, i.e. column i of w_down) with scales [n].  x and b in dt. */
void oracle_ffn_masked_q(int32_t d, int32_t n, int32_t act, int32_t dt, const void *x, const int8_t *q_up,
                         const float *s_up, const int8_t *q_gate, const float *s_gate, const void *bias,
                         const int8_t *q_down, const float *s_down, const uint8_t *mask, double *a, double *y,
                         int32_t nthreads) {
    init_table();
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 16)
    for (int32_t i = 0; i < n; ++i) {
        if (!mask[i]) {
            a[i] = 0.0;
            continue;
        }
        double up = 0.0;
        for (int32_t k = 0; k < d; ++k) up += ((double)q_up[(size_t)i * d + k] * (double)s_up[i]) * ld(x, dt, k);
        if (act == OR_RELU) {
            const double pre = up + ld(bias, dt, i);
            a[i] = pre > 0.0 ? pre : 0.0;
        } else {
            double gate = 0.0;
            for (int32_t k = 0; k < d; ++k)
                gate += ((double)q_gate[(size_t)i * d + k] * (double)s_gate[i]) * ld(x, dt, k);
            gate += ld(bias, dt, i);
            a[i] = (gate > 0.0 ? gate : 0.0) * up;
        }
    }
    int32_t *list = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n > 0 ? n : 1));
    int32_t k = 0;
    for (int32_t i = 0; i < n; ++i)
        if (mask[i]) list[k++] = i;
#pragma omp parallel for schedule(static)
    for (int32_t j = 0; j < d; ++j) {
        double s = 0.0;
        for (int32_t t = 0; t < k; ++t) {
            const int32_t i = list[t];
            s += a[i] * ((double)q_down[(size_t)i * d + j] * (double)s_down[i]);
        }
        y[j] = s;
    }
    free(list);
}

int32_t oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
