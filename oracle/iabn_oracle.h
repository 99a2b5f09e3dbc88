/*
 * iabn_oracle.h -- plain fp64 CPU oracle for In-Place Activated BatchNorm.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test-suite, the smoke
 * check and the CPU-baseline leg of the benchmark may load this library.  It
 * shares no code, header, table or helper with the CUDA library.
 *
 * Sources (web pages about the method):
 *   [ABN]  "In-Place Activated BatchNorm for Memory-Optimized Training of
 *          DNNs", section-by-section summary (paperlayer.ai), section 3
 *          "In-Place Activated Batch Normalization" with its bullets
 *          "Batch Normalization Review", "Standard and Checkpointed
 *          Computation", "INPLACE-ABN" and "INPLACE-ABN II"; section 4
 *          "Experimental setup" (leaky-ReLU, slope 0.01).
 *   [BN]   Ioffe & Szegedy, "Batch Normalization: Accelerating Deep Network
 *          Training by Reducing Internal Covariate Shift", cited in the
 *          reference list of the same paper (app.cochat.ai page).
 *
 * Tensor layout: element (n, c, p) with p = h*W + w lives at
 *   NCHW: ((n*C + c)*HW + p)        NHWC: ((n*HW + p)*C + c)
 * All floating-point arrays are double.  M = N*H*W values per channel.
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes of the repository):
 *   - variance for normalisation is the biased one (divide by M);
 *   - rstd = 1/sqrt(var + eps);
 *   - the positive branch of both activations is taken iff its argument is
 *     strictly positive;
 *   - ELU inverse: with t = z/alpha, y = log1p(t) when 1 + t > 2^-24, else
 *     y = log(2^-24) (a saturated, rounded z carries no more information);
 *     its slope is taken from z as max(z + alpha, 0);
 *   - gamma is used with its sign; a channel with |gamma| below the smallest
 *     normal float gives NaN gradients (the affine is not invertible there);
 *   - running statistics: r <- (1-m) r + m s, with the unbiased variance
 *     var*M/(M-1) for the running variance.
 */
#ifndef IABN_ORACLE_H
#define IABN_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_NCHW = 0, ORC_NHWC = 1 };
enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_F16 = 2 };
enum { ORC_LEAKY_RELU = 0, ORC_ELU = 1, ORC_IDENTITY = 2 };

/* Activation phi, its inverse, and dL/dy = dL/dz * phi'(y) taken from z.
 * Return NaN for an unknown activation kind. */
double orc_act(double y, int act, double p);
double orc_act_inv(double z, int act, double p);
double orc_act_dy_from_z(double z, double dz, int act, double p);
/* phi'(y) evaluated from the pre-activation (textbook form). */
double orc_act_deriv_from_y(double y, int act, double p);

/* Round each value to the nearest value of the storage type (ties to even),
 * written from the IEEE-754 definition; result returned as an exact double.
 * Returns 0 on success, -1 for an unknown dtype. */
int orc_round(const double* in, double* out, int64_t count, int dtype);

/* Forward, training mode: per-channel batch mean and biased variance
 * (two passes: the mean first, then the sum of squared deviations), then
 * xhat = (x - mean) * rstd, y = gamma*xhat + beta, z = phi(y).
 * xhat_out and y_out may be NULL.  Returns 0, or -1 on a bad argument. */
int orc_forward(int64_t n, int64_t c, int64_t h, int64_t w, int layout,
                const double* x, const double* gamma, const double* beta,
                double eps, int act, double act_param,
                double* mean_out, double* var_out,
                double* xhat_out, double* y_out, double* z_out);

/* Standard BN+ACT backward, computed from the stored input x (the layer
 * that keeps x and z, [ABN] "Standard and Checkpointed Computation"):
 * recompute the statistics, xhat and y from x; dy = dz*phi'(y);
 * dbeta = sum dy; dgamma = sum dy*xhat;
 * dx = gamma*rstd*(dy - dbeta/M - xhat*dgamma/M). */
int orc_backward_standard(int64_t n, int64_t c, int64_t h, int64_t w, int layout,
                          const double* x, const double* dz,
                          const double* gamma, const double* beta,
                          double eps, int act, double act_param,
                          double* dx, double* dgamma, double* dbeta);

/* INPLACE-ABN I ([ABN] "INPLACE-ABN"): from z only.  y = phi^-1(z);
 * dy = dz*phi'(y) (from z); xhat = (y - beta)/gamma; then the BN backward
 * in xhat as above, with rstd from the saved (biased) variance. */
int orc_backward_inplace_1(int64_t n, int64_t c, int64_t h, int64_t w, int layout,
                           const double* z, const double* dz,
                           const double* gamma, const double* beta,
                           const double* var, double eps, int act, double act_param,
                           double* dx, double* dgamma, double* dbeta);

/* INPLACE-ABN II ([ABN] "INPLACE-ABN II"): the gradients written directly
 * in terms of y; xhat is never formed:
 *   dbeta = sum dy,  dgamma = (sum dy*y - beta*dbeta)/gamma,
 *   dx = rstd*(gamma*dy - gamma*dbeta/M - (y - beta)*dgamma/M). */
int orc_backward_inplace_2(int64_t n, int64_t c, int64_t h, int64_t w, int layout,
                           const double* z, const double* dz,
                           const double* gamma, const double* beta,
                           const double* var, double eps, int act, double act_param,
                           double* dx, double* dgamma, double* dbeta);

/* Optimized checkpointing ([ABN] section 3, "Proposed Checkpointing"): the
 * layer keeps the normalised xhat (the forward's xhat_out) instead of x.  The
 * backward recovers y = gamma*xhat + beta by the scale and shift alone,
 * dy = dz*phi'(y), and runs the BN backward on the stored xhat (nothing is
 * recomputed from x):
 *   dbeta = sum dy,  dgamma = sum dy*xhat,
 *   dx = gamma*rstd*(dy - dbeta/M - xhat*dgamma/M),  rstd from the saved
 *   (biased) variance. */
int orc_backward_checkpoint(int64_t n, int64_t c, int64_t h, int64_t w, int layout,
                            const double* xhat, const double* dz,
                            const double* gamma, const double* beta,
                            const double* var, double eps, int act, double act_param,
                            double* dx, double* dgamma, double* dbeta);

/* The activation output the layer after it needs, recovered from the stored
 * xhat ([ABN] "Proposed Checkpointing": scale and shift, then the
 * activation):  z = phi(gamma*xhat + beta). */
int orc_checkpoint_recompute(int64_t n, int64_t c, int64_t h, int64_t w, int layout,
                             const double* xhat, const double* gamma, const double* beta,
                             int act, double act_param, double* z_out);

/* Inference (evaluation mode): the layer with fixed statistics in place of
 * the batch's ([BN] Algorithm 2, the inference network: normalise with the
 * population mean and variance the running averages estimate; [ABN] section
 * 3, "Batch Normalization Review": scale and shift by gamma and beta):
 *   xhat = (x - running_mean) / sqrt(running_var + eps),
 *   y = gamma*xhat + beta,  z = phi(y).
 * Returns 0, or -1 on a bad argument. */
int orc_inference(int64_t n, int64_t c, int64_t h, int64_t w, int layout,
                  const double* x, const double* gamma, const double* beta,
                  const double* running_mean, const double* running_var,
                  double eps, int act, double act_param, double* z_out);

/* Running statistics (momentum form, unbiased running variance), in place. */
int orc_running_update(int64_t c, int64_t count, const double* mean, const double* var,
                       double momentum, double* running_mean, double* running_var);

#ifdef __cplusplus
}
#endif
#endif /* IABN_ORACLE_H */
