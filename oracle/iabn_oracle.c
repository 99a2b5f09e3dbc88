/*
 * iabn_oracle.c -- plain fp64 CPU oracle for In-Place Activated BatchNorm.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE (see iabn_oracle.h for the sources,
 * the layout convention and the readings taken where the pages are silent).
 *
 * Everything here is deliberately the plain definition: one loop per
 * formula, fp64 throughout, no blocking, fusion or reordering.  The per-
 * channel sums visit the elements of a channel in (n, h, w) order.
 */
#include "iabn_oracle.h"

#include <math.h>
#include <stdlib.h>

/* Built with -fopenmp (the benchmark's multi-core CPU baseline), the loops
 * over channels (and over the elements of orc_round) are split across the
 * host's cores.  Every iteration writes only its own channel's outputs, in
 * the same order, so both builds give identical bits. */
#ifdef _OPENMP
#define ORC_PARALLEL_FOR _Pragma("omp parallel for schedule(static)")
#else
#define ORC_PARALLEL_FOR
#endif

/* ---------------------------------------------------------------- layout */

static int64_t at(int layout, int64_t C, int64_t HW, int64_t n, int64_t c, int64_t p) {
    return layout == ORC_NCHW ? (n * C + c) * HW + p : (n * HW + p) * C + c;
}

static int check_geom(int64_t n, int64_t c, int64_t h, int64_t w, int layout) {
    if (n <= 0 || c <= 0 || h <= 0 || w <= 0) return -1;
    if (layout != ORC_NCHW && layout != ORC_NHWC) return -1;
    return 0;
}

/* ------------------------------------------------------------ activation */
/* [ABN] section 3, "INPLACE-ABN": the activation must be invertible; section
 * 4, "Experimental setup": leaky-ReLU with slope a = 0.01.  ELU (alpha > 0)
 * is the other invertible activation the layer is asked to support. */

#define ORC_ELU_FLOOR_LOG2 (-24)

double orc_act(double y, int act, double p) {
    switch (act) {
    case ORC_LEAKY_RELU: return y > 0.0 ? y : p * y;
    case ORC_ELU:        return y > 0.0 ? y : p * expm1(y);
    case ORC_IDENTITY:   return y;
    default:             return NAN;
    }
}

double orc_act_inv(double z, int act, double p) {
    switch (act) {
    case ORC_LEAKY_RELU: return z > 0.0 ? z : z / p;
    case ORC_ELU: {
        if (z > 0.0) return z;
        double t = z / p;
        double floor_u = ldexp(1.0, ORC_ELU_FLOOR_LOG2);
        if (1.0 + t <= floor_u) return log(floor_u);
        return log1p(t);
    }
    case ORC_IDENTITY:   return z;
    default:             return NAN;
    }
}

double orc_act_dy_from_z(double z, double dz, int act, double p) {
    switch (act) {
    case ORC_LEAKY_RELU: return z > 0.0 ? dz : p * dz;
    case ORC_ELU: {
        /* phi'(y) = alpha*e^y = z + alpha on the negative branch. */
        if (z > 0.0) return dz;
        double s = z + p;
        return s > 0.0 ? dz * s : 0.0;
    }
    case ORC_IDENTITY:   return dz;
    default:             return NAN;
    }
}

double orc_act_deriv_from_y(double y, int act, double p) {
    switch (act) {
    case ORC_LEAKY_RELU: return y > 0.0 ? 1.0 : p;
    case ORC_ELU:        return y > 0.0 ? 1.0 : p * exp(y);
    case ORC_IDENTITY:   return 1.0;
    default:             return NAN;
    }
}

/* -------------------------------------------------------------- rounding */
/* Round to nearest, ties to even, into a binary format with `prec`
 * significand bits (hidden bit included) and exponent range [emin, emax]
 * (IEEE 754-2008, section 4.3.1 and 7.4).  Subnormals keep the fixed
 * quantum 2^(emin - prec + 1); a result of magnitude >= 2^(emax + 1)
 * overflows to infinity. */
static double round_format(double v, int prec, int emin, int emax) {
    if (isnan(v) || isinf(v) || v == 0.0) return v;
    double a = fabs(v);
    int k;
    frexp(a, &k);              /* a = m * 2^k, m in [0.5, 1) */
    int e = k - 1;             /* a in [2^e, 2^(e+1)) */
    if (e < emin) e = emin;    /* subnormal range: fixed quantum */
    double q = ldexp(a, prec - 1 - e);   /* exact: a scaled so the quantum is 1 */
    double r = rint(q);                   /* default mode: nearest, ties to even */
    double res = ldexp(r, e - (prec - 1));
    if (res >= ldexp(1.0, emax + 1)) res = INFINITY;
    return copysign(res, v);
}

int orc_round(const double* in, double* out, int64_t count, int dtype) {
    int prec, emin, emax;
    switch (dtype) {
    case ORC_F32:  prec = 24; emin = -126; emax = 127; break;
    case ORC_BF16: prec = 8;  emin = -126; emax = 127; break;
    case ORC_F16:  prec = 11; emin = -14;  emax = 15;  break;
    default: return -1;
    }
    ORC_PARALLEL_FOR
    for (int64_t i = 0; i < count; ++i) out[i] = round_format(in[i], prec, emin, emax);
    return 0;
}

/* ------------------------------------------------------------ statistics */
/* [ABN] section 3, "Batch Normalization Review"; [BN] Algorithm 1: the
 * minibatch statistics are the empirical per-channel mean and variance. */

static void channel_stats(int64_t N, int64_t C, int64_t HW, int layout, const double* x,
                          int64_t c, double* mean, double* var) {
    const double M = (double)(N * HW);
    double s = 0.0;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t p = 0; p < HW; ++p) s += x[at(layout, C, HW, n, c, p)];
    double mu = s / M;
    double ss = 0.0;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t p = 0; p < HW; ++p) {
            double d = x[at(layout, C, HW, n, c, p)] - mu;
            ss += d * d;
        }
    *mean = mu;
    *var = ss / M;
}

int orc_forward(int64_t n, int64_t c, int64_t h, int64_t w, int layout,
                const double* x, const double* gamma, const double* beta,
                double eps, int act, double act_param,
                double* mean_out, double* var_out,
                double* xhat_out, double* y_out, double* z_out) {
    if (check_geom(n, c, h, w, layout)) return -1;
    const int64_t HW = h * w;
    ORC_PARALLEL_FOR
    for (int64_t ch = 0; ch < c; ++ch) {
        double mu, var;
        channel_stats(n, c, HW, layout, x, ch, &mu, &var);
        double rstd = 1.0 / sqrt(var + eps);
        if (mean_out) mean_out[ch] = mu;
        if (var_out) var_out[ch] = var;
        for (int64_t i = 0; i < n; ++i)
            for (int64_t p = 0; p < HW; ++p) {
                int64_t k = at(layout, c, HW, i, ch, p);
                double xhat = (x[k] - mu) * rstd;      /* whitening */
                double y = gamma[ch] * xhat + beta[ch]; /* scale and shift */
                if (xhat_out) xhat_out[k] = xhat;
                if (y_out) y_out[k] = y;
                if (z_out) z_out[k] = orc_act(y, act, act_param);
            }
    }
    return 0;
}

/* ------------------------------------------------------------- backward */

int orc_backward_standard(int64_t n, int64_t c, int64_t h, int64_t w, int layout,
                          const double* x, const double* dz,
                          const double* gamma, const double* beta,
                          double eps, int act, double act_param,
                          double* dx, double* dgamma, double* dbeta) {
    if (check_geom(n, c, h, w, layout)) return -1;
    const int64_t HW = h * w;
    const double M = (double)(n * HW);
    ORC_PARALLEL_FOR
    for (int64_t ch = 0; ch < c; ++ch) {
        double mu, var;
        channel_stats(n, c, HW, layout, x, ch, &mu, &var);
        double rstd = 1.0 / sqrt(var + eps);
        double s1 = 0.0, s2 = 0.0;
        for (int64_t i = 0; i < n; ++i)
            for (int64_t p = 0; p < HW; ++p) {
                int64_t k = at(layout, c, HW, i, ch, p);
                double xhat = (x[k] - mu) * rstd;
                double y = gamma[ch] * xhat + beta[ch];
                double dy = dz[k] * orc_act_deriv_from_y(y, act, act_param);
                s1 += dy;
                s2 += dy * xhat;
            }
        dbeta[ch] = s1;
        dgamma[ch] = s2;
        for (int64_t i = 0; i < n; ++i)
            for (int64_t p = 0; p < HW; ++p) {
                int64_t k = at(layout, c, HW, i, ch, p);
                double xhat = (x[k] - mu) * rstd;
                double y = gamma[ch] * xhat + beta[ch];
                double dy = dz[k] * orc_act_deriv_from_y(y, act, act_param);
                dx[k] = gamma[ch] * rstd * (dy - s1 / M - xhat * s2 / M);
            }
    }
    return 0;
}

int orc_backward_inplace_1(int64_t n, int64_t c, int64_t h, int64_t w, int layout,
                           const double* z, const double* dz,
                           const double* gamma, const double* beta,
                           const double* var, double eps, int act, double act_param,
                           double* dx, double* dgamma, double* dbeta) {
    if (check_geom(n, c, h, w, layout)) return -1;
    const int64_t HW = h * w;
    const double M = (double)(n * HW);
    ORC_PARALLEL_FOR
    for (int64_t ch = 0; ch < c; ++ch) {
        double rstd = 1.0 / sqrt(var[ch] + eps);
        double s1 = 0.0, s2 = 0.0;
        for (int64_t i = 0; i < n; ++i)
            for (int64_t p = 0; p < HW; ++p) {
                int64_t k = at(layout, c, HW, i, ch, p);
                double y = orc_act_inv(z[k], act, act_param);        /* invert phi */
                double dy = orc_act_dy_from_z(z[k], dz[k], act, act_param);
                double xhat = (y - beta[ch]) / gamma[ch];            /* invert the affine */
                s1 += dy;
                if (dy != 0.0) s2 += dy * xhat;                      /* 0*anything = 0 */
            }
        dbeta[ch] = s1;
        dgamma[ch] = s2;
        for (int64_t i = 0; i < n; ++i)
            for (int64_t p = 0; p < HW; ++p) {
                int64_t k = at(layout, c, HW, i, ch, p);
                double y = orc_act_inv(z[k], act, act_param);
                double dy = orc_act_dy_from_z(z[k], dz[k], act, act_param);
                double xhat = (y - beta[ch]) / gamma[ch];
                dx[k] = gamma[ch] * rstd * (dy - s1 / M - xhat * s2 / M);
            }
        if (!(fabs(gamma[ch]) >= 1.17549435082228750797e-38)) { /* FLT_MIN */
            dbeta[ch] = NAN;
            dgamma[ch] = NAN;
            for (int64_t i = 0; i < n; ++i)
                for (int64_t p = 0; p < HW; ++p) dx[at(layout, c, HW, i, ch, p)] = NAN;
        }
    }
    return 0;
}

int orc_backward_inplace_2(int64_t n, int64_t c, int64_t h, int64_t w, int layout,
                           const double* z, const double* dz,
                           const double* gamma, const double* beta,
                           const double* var, double eps, int act, double act_param,
                           double* dx, double* dgamma, double* dbeta) {
    if (check_geom(n, c, h, w, layout)) return -1;
    const int64_t HW = h * w;
    const double M = (double)(n * HW);
    ORC_PARALLEL_FOR
    for (int64_t ch = 0; ch < c; ++ch) {
        double rstd = 1.0 / sqrt(var[ch] + eps);
        double s1 = 0.0, sy = 0.0;
        for (int64_t i = 0; i < n; ++i)
            for (int64_t p = 0; p < HW; ++p) {
                int64_t k = at(layout, c, HW, i, ch, p);
                double y = orc_act_inv(z[k], act, act_param);
                double dy = orc_act_dy_from_z(z[k], dz[k], act, act_param);
                s1 += dy;
                if (dy != 0.0) sy += dy * y;
            }
        double db = s1;
        double dg = (sy - beta[ch] * s1) / gamma[ch];
        dbeta[ch] = db;
        dgamma[ch] = dg;
        for (int64_t i = 0; i < n; ++i)
            for (int64_t p = 0; p < HW; ++p) {
                int64_t k = at(layout, c, HW, i, ch, p);
                double y = orc_act_inv(z[k], act, act_param);
                double dy = orc_act_dy_from_z(z[k], dz[k], act, act_param);
                dx[k] = rstd * (gamma[ch] * dy - gamma[ch] * db / M - (y - beta[ch]) * dg / M);
            }
        if (!(fabs(gamma[ch]) >= 1.17549435082228750797e-38)) { /* FLT_MIN */
            dbeta[ch] = NAN;
            dgamma[ch] = NAN;
            for (int64_t i = 0; i < n; ++i)
                for (int64_t p = 0; p < HW; ++p) dx[at(layout, c, HW, i, ch, p)] = NAN;
        }
    }
    return 0;
}

/* --------------------------------------------------- checkpointing (xhat) */
/* [ABN] section 3, "Proposed Checkpointing": the stored buffer is xhat; the
 * backward reaches y through the scale and shift only and uses the stored
 * xhat in the BN backward as it stands. */

int orc_backward_checkpoint(int64_t n, int64_t c, int64_t h, int64_t w, int layout,
                            const double* xhat, const double* dz,
                            const double* gamma, const double* beta,
                            const double* var, double eps, int act, double act_param,
                            double* dx, double* dgamma, double* dbeta) {
    if (check_geom(n, c, h, w, layout)) return -1;
    const int64_t HW = h * w;
    const double M = (double)(n * HW);
    ORC_PARALLEL_FOR
    for (int64_t ch = 0; ch < c; ++ch) {
        double rstd = 1.0 / sqrt(var[ch] + eps);
        double s1 = 0.0, s2 = 0.0;
        for (int64_t i = 0; i < n; ++i)
            for (int64_t p = 0; p < HW; ++p) {
                int64_t k = at(layout, c, HW, i, ch, p);
                double y = gamma[ch] * xhat[k] + beta[ch];           /* scale and shift */
                double dy = dz[k] * orc_act_deriv_from_y(y, act, act_param);
                s1 += dy;
                s2 += dy * xhat[k];
            }
        dbeta[ch] = s1;
        dgamma[ch] = s2;
        for (int64_t i = 0; i < n; ++i)
            for (int64_t p = 0; p < HW; ++p) {
                int64_t k = at(layout, c, HW, i, ch, p);
                double y = gamma[ch] * xhat[k] + beta[ch];
                double dy = dz[k] * orc_act_deriv_from_y(y, act, act_param);
                dx[k] = gamma[ch] * rstd * (dy - s1 / M - xhat[k] * s2 / M);
            }
    }
    return 0;
}

int orc_checkpoint_recompute(int64_t n, int64_t c, int64_t h, int64_t w, int layout,
                             const double* xhat, const double* gamma, const double* beta,
                             int act, double act_param, double* z_out) {
    if (check_geom(n, c, h, w, layout)) return -1;
    const int64_t HW = h * w;
    ORC_PARALLEL_FOR
    for (int64_t ch = 0; ch < c; ++ch)
        for (int64_t i = 0; i < n; ++i)
            for (int64_t p = 0; p < HW; ++p) {
                int64_t k = at(layout, c, HW, i, ch, p);
                z_out[k] = orc_act(gamma[ch] * xhat[k] + beta[ch], act, act_param);
            }
    return 0;
}

/* ----------------------------------------------------- running statistics */
/* ------------------------------------------------------------ inference */
/* [BN] Algorithm 2 (the inference network): the batch statistics are
 * replaced by fixed estimates of the population's, here the running
 * averages; then the same scale, shift and activation as in training. */

int orc_inference(int64_t n, int64_t c, int64_t h, int64_t w, int layout,
                  const double* x, const double* gamma, const double* beta,
                  const double* running_mean, const double* running_var,
                  double eps, int act, double act_param, double* z_out) {
    if (check_geom(n, c, h, w, layout)) return -1;
    const int64_t HW = h * w;
    ORC_PARALLEL_FOR
    for (int64_t ch = 0; ch < c; ++ch) {
        double rstd = 1.0 / sqrt(running_var[ch] + eps);
        for (int64_t i = 0; i < n; ++i)
            for (int64_t p = 0; p < HW; ++p) {
                int64_t k = at(layout, c, HW, i, ch, p);
                double xhat = (x[k] - running_mean[ch]) * rstd;
                double y = gamma[ch] * xhat + beta[ch];
                z_out[k] = orc_act(y, act, act_param);
            }
    }
    return 0;
}

/* [BN] Algorithm 2 uses the unbiased variance for inference; the momentum
 * form of the running average is the usual framework convention. */
int orc_running_update(int64_t c, int64_t count, const double* mean, const double* var,
                       double momentum, double* running_mean, double* running_var) {
    if (c <= 0 || count < 2) return -1;
    const double unbias = (double)count / (double)(count - 1);
    ORC_PARALLEL_FOR
    for (int64_t ch = 0; ch < c; ++ch) {
        running_mean[ch] = (1.0 - momentum) * running_mean[ch] + momentum * mean[ch];
        running_var[ch] = (1.0 - momentum) * running_var[ch] + momentum * var[ch] * unbias;
    }
    return 0;
}
