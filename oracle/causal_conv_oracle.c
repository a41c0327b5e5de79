/*
 * Oracle for the causal sequence convolution -- TEST INFRASTRUCTURE ONLY.
 *
 * This file is the plain, slow, obviously-correct CPU statement of what the
 * GPU path computes.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark load it; the product library never links or
 * calls it, and it shares no code, header or constant with the CUDA sources.
 *
 * Definition followed (Caracal: Causal Architecture via Spectral Mixing,
 * section "Key design 1: Multi-Head Fourier module" and "Key design 2:
 * frequency-domain causal mask"): per (batch b, channel d) row,
 *
 *     r_t = sum_{j=0}^{t} v_j * g_{t-j},      0 <= t < L,
 *
 * which the pages state is exactly what zero-padding to 2L, FFT, pointwise
 * product, inverse FFT and truncation to L produce.  The oracle therefore
 * evaluates the sum itself, term by term in ascending j, with no transform.
 *
 * Float rows are widened to double (products of two float32 values are exact
 * in double) and summed in double.  For the float error bound the oracle also
 * returns den_t = sum_j |v_j * g_{t-j}|.  Integer rows (the number-theoretic
 * variant of "Catastrophic Token Leakage in Convolutional Sequence Modeling
 * and How to Mitigate It", abstract) are summed exactly in int64.
 *
 * Layout: every array is [B, L, D] row-major ("channel-last"): element
 * (b, t, d) sits at (b*L + t)*D + d.  Points for the sampled variants are
 * given as n triples (b, t, d), flattened.
 *
 * Backward (gradient of a scalar loss through r, given dr = dLoss/dr): the
 * derivatives of the sum above are, per row,
 *
 *     dv_j = sum_{t=j}^{L-1} dr_t * g_{t-j},     dg_k = sum_{t=k}^{L-1} dr_t * v_{t-k},
 *
 * again evaluated term by term (ascending t) in double, with the matching
 * error-bound denominators sum |dr_t g_{t-j}| and sum |dr_t v_{t-k}|.
 *
 * Parity pins: see tests/test_oracle_pins.py (delta inputs, closed-form sums,
 * commutativity/bilinearity/shift, causality, wrap-around, brute force, and
 * for the backward: the adjoint identity, numpy.convolve on reversed rows,
 * torch autograd).
 */
#include <stdint.h>
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define IDX(b, t, d) (((int64_t)(b) * L + (t)) * D + (d))

/* r[b,t,d] and den[b,t,d] for one point, float64 inputs. */
static void point_f64(const double *v, const double *g, int64_t L, int64_t D,
                      int64_t b, int64_t t, int64_t d, double *r, double *den)
{
    double acc = 0.0, mag = 0.0;
    for (int64_t j = 0; j <= t; ++j) {
        double p = v[IDX(b, j, d)] * g[IDX(b, t - j, d)];
        acc += p;
        mag += fabs(p);
    }
    *r = acc;
    *den = mag;
}

/* Same, float32 inputs widened to double on use. */
static void point_f32in(const float *v, const float *g, int64_t L, int64_t D,
                        int64_t b, int64_t t, int64_t d, double *r, double *den)
{
    double acc = 0.0, mag = 0.0;
    for (int64_t j = 0; j <= t; ++j) {
        double p = (double)v[IDX(b, j, d)] * (double)g[IDX(b, t - j, d)];
        acc += p;
        mag += fabs(p);
    }
    *r = acc;
    *den = mag;
}

static int64_t point_i32in(const int32_t *v, const int32_t *g, int64_t L, int64_t D,
                           int64_t b, int64_t t, int64_t d)
{
    int64_t acc = 0;
    for (int64_t j = 0; j <= t; ++j)
        acc += (int64_t)v[IDX(b, j, d)] * (int64_t)g[IDX(b, t - j, d)];
    return acc;
}

/* ---- full outputs ------------------------------------------------------ */

void oracle_conv_f64(const double *v, const double *g, int64_t B, int64_t L, int64_t D,
                     double *r, double *den)
{
    int64_t n = B * L * D;
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t i = 0; i < n; ++i) {
        int64_t d = i % D, t = (i / D) % L, b = i / (D * L);
        point_f64(v, g, L, D, b, t, d, &r[i], &den[i]);
    }
}

void oracle_conv_f32in(const float *v, const float *g, int64_t B, int64_t L, int64_t D,
                       double *r, double *den)
{
    int64_t n = B * L * D;
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t i = 0; i < n; ++i) {
        int64_t d = i % D, t = (i / D) % L, b = i / (D * L);
        point_f32in(v, g, L, D, b, t, d, &r[i], &den[i]);
    }
}

void oracle_conv_i32in(const int32_t *v, const int32_t *g, int64_t B, int64_t L, int64_t D,
                       int64_t *r)
{
    int64_t n = B * L * D;
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t i = 0; i < n; ++i) {
        int64_t d = i % D, t = (i / D) % L, b = i / (D * L);
        r[i] = point_i32in(v, g, L, D, b, t, d);
    }
}

/* ---- sampled outputs: pts = n x (b, t, d) ------------------------------ */

void oracle_conv_f64_points(const double *v, const double *g, int64_t B, int64_t L, int64_t D,
                            const int64_t *pts, int64_t n, double *r, double *den)
{
    (void)B;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t i = 0; i < n; ++i)
        point_f64(v, g, L, D, pts[3 * i], pts[3 * i + 1], pts[3 * i + 2], &r[i], &den[i]);
}

void oracle_conv_f32in_points(const float *v, const float *g, int64_t B, int64_t L, int64_t D,
                              const int64_t *pts, int64_t n, double *r, double *den)
{
    (void)B;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t i = 0; i < n; ++i)
        point_f32in(v, g, L, D, pts[3 * i], pts[3 * i + 1], pts[3 * i + 2], &r[i], &den[i]);
}

void oracle_conv_i32in_points(const int32_t *v, const int32_t *g, int64_t B, int64_t L, int64_t D,
                              const int64_t *pts, int64_t n, int64_t *r)
{
    (void)B;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t i = 0; i < n; ++i)
        r[i] = point_i32in(v, g, L, D, pts[3 * i], pts[3 * i + 1], pts[3 * i + 2]);
}

/* ---- backward ---------------------------------------------------------- */

/* dv[b,j,d] (with den) for one point: sum over t >= j of dr_t g_{t-j}. */
static void point_bwd_f32in(const float *dr, const float *k, int64_t L, int64_t D,
                            int64_t b, int64_t j, int64_t d, double *out, double *den)
{
    double acc = 0.0, mag = 0.0;
    for (int64_t t = j; t < L; ++t) {
        double p = (double)dr[IDX(b, t, d)] * (double)k[IDX(b, t - j, d)];
        acc += p;
        mag += fabs(p);
    }
    *out = acc;
    *den = mag;
}

/* Full gradients: dv from (dr, g), dg from (dr, v). */
void oracle_conv_bwd_f32in(const float *dr, const float *v, const float *g, int64_t B, int64_t L, int64_t D,
                           double *dv, double *den_dv, double *dg, double *den_dg)
{
    int64_t n = B * L * D;
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t i = 0; i < n; ++i) {
        int64_t d = i % D, j = (i / D) % L, b = i / (D * L);
        point_bwd_f32in(dr, g, L, D, b, j, d, &dv[i], &den_dv[i]);
        point_bwd_f32in(dr, v, L, D, b, j, d, &dg[i], &den_dg[i]);
    }
}

void oracle_conv_bwd_f32in_points(const float *dr, const float *v, const float *g, int64_t B, int64_t L,
                                  int64_t D, const int64_t *pts, int64_t n, double *dv, double *den_dv,
                                  double *dg, double *den_dg)
{
    (void)B;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t i = 0; i < n; ++i) {
        point_bwd_f32in(dr, g, L, D, pts[3 * i], pts[3 * i + 1], pts[3 * i + 2], &dv[i], &den_dv[i]);
        point_bwd_f32in(dr, v, L, D, pts[3 * i], pts[3 * i + 1], pts[3 * i + 2], &dg[i], &den_dg[i]);
    }
}

/* Number of OpenMP threads the loops above use (for the baseline report). */
int oracle_num_threads(void)
{
    int n = 1;
#ifdef _OPENMP
#pragma omp parallel
    {
#pragma omp single
        n = omp_get_num_threads();
    }
#endif
    return n;
}
