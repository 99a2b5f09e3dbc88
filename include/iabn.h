/*
 * iabn.h -- C ABI of libiabn.so: In-Place Activated BatchNorm (InPlace-ABN)
 * for NVIDIA B200 (sm_100a), training mode, one GPU.
 *
 * The layer fuses batch normalisation and an invertible activation and keeps
 * a single buffer: the forward overwrites its input x with the activated
 * output z; the backward recovers what it needs from z alone by inverting
 * the activation and the scale-and-shift, and overwrites the incoming
 * gradient dz with dx.
 *
 * Sources (web pages about the method; cited by title and section):
 *   [ABN] "In-Place Activated BatchNorm for Memory-Optimized Training of
 *         DNNs" (Rota Bulo, Porzi, Kontschieder; CVPR 2018), the
 *         section-by-section summary on paperlayer.ai: section 3 "In-Place
 *         Activated Batch Normalization" -- bullets "INPLACE-ABN" (one buffer,
 *         invertible activation and scale-and-shift), "Batch Normalization
 *         Review" (empirical mean and variance, learnable gamma and beta),
 *         "INPLACE-ABN II" (gradients written in terms of y); section 4
 *         "Experimental setup" (leaky-ReLU, slope 0.01).  The abstract (same
 *         title, codewithpapers.app and app.cochat.ai pages) calls it a single
 *         plugin layer for existing frameworks.
 *   [BN]  Ioffe & Szegedy, "Batch Normalization ...", cited in that paper's
 *         reference list: batch statistics and the BN backward.
 *
 * Conventions for every call
 *   - Every pointer argument except `stream` is a DEVICE pointer to memory
 *     owned by the caller.  No call allocates memory.  Between calls the
 *     library keeps only per-device launch settings, and one 8 MiB array of
 *     device memory on every GPU that loads it: the scratch of
 *     iabn_forward_static_ws, held until the process exits.
 *   - All calls are asynchronous and ordered on `stream` (a cudaStream_t;
 *     NULL means the legacy default stream), except iabn_get_device_status.
 *   - Arguments are checked on the host before anything is launched; a
 *     rejected call launches nothing and returns the error.
 *   - Element (n, c, h, w) of a tensor lives at ((n*C + c)*H + h)*W + w for
 *     IABN_NCHW and ((n*H + h)*W + w)*C + c for IABN_NHWC.  M = N*H*W is the
 *     number of values per channel.
 *   - Activation tensors (x/z, dz/dx) use the storage type `dtype`; gamma,
 *     beta, statistics and parameter gradients are always float32 [C].  All
 *     arithmetic is float32 (statistics combined in float64), with one
 *     round-to-nearest-even into the storage type per written element.
 *   - Activation tensors must start on a 16-byte boundary
 *     (IABN_ERR_MISALIGNED otherwise).
 *   - One workspace may serve only one call in flight at a time.  It must be
 *     zero-filled once before its first use; each call leaves it reusable.
 *     Its size is given by iabn_workspace_size and depends only on the
 *     descriptor.
 *   - Errors found on the device never trap: they set a sticky status word
 *     in the workspace that iabn_get_device_status reads.
 */
#ifndef IABN_H
#define IABN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    IABN_OK = 0,
    IABN_ERR_INVALID_ARG = 1,    /* null pointer, bad dimension, M < 2, bad parameter */
    IABN_ERR_UNSUPPORTED = 2,    /* valid but not supported (e.g. sizes beyond int64) */
    IABN_ERR_MISALIGNED = 3,     /* an activation tensor is not 16-byte aligned */
    IABN_ERR_WORKSPACE = 4,      /* workspace missing or smaller than iabn_workspace_size */
    IABN_ERR_CUDA = 5,           /* a CUDA runtime call failed (launch, copy, ...) */
    IABN_ERR_TIMEOUT = 6,        /* device: a bounded wait inside a kernel ran out */
    IABN_ERR_SINGULAR_GAMMA = 7  /* device: |gamma_c| < FLT_MIN in a backward call */
} iabn_status;

typedef enum { IABN_NCHW = 0, IABN_NHWC = 1 } iabn_layout;
typedef enum { IABN_F32 = 0, IABN_BF16 = 1, IABN_F16 = 2 } iabn_dtype;

/* The activation phi.  The positive branch is taken iff its argument is > 0.
 *   IABN_ACT_LEAKY_RELU: phi(y) = y (y > 0), a*y otherwise; act_param = a > 0.
 *   IABN_ACT_ELU:        phi(y) = y (y > 0), alpha*(e^y - 1) otherwise;
 *                        act_param = alpha > 0.
 *   IABN_ACT_IDENTITY:   phi(y) = y (plain batch normalisation); act_param unused. */
typedef enum { IABN_ACT_LEAKY_RELU = 0, IABN_ACT_ELU = 1, IABN_ACT_IDENTITY = 2 } iabn_act;

/* Tensor descriptor: logical shape N x C x H x W, memory layout and storage
 * type (iabn_layout / iabn_dtype values). */
typedef struct {
    int64_t n, c, h, w;
    int32_t layout;
    int32_t dtype;
} iabn_desc;

/* Bytes of workspace the forward and backward calls of every layer need for
 * descriptor `d` (a multiple of 256).  Returns 0 if the descriptor is
 * invalid; M = 1 is valid here (iabn_inference takes it, the training calls
 * do not).  Host-only. */
size_t iabn_workspace_size(const iabn_desc* d);

/* Forward, training mode ([ABN] section 3, "Batch Normalization Review" and
 * "INPLACE-ABN"; [BN] Algorithm 1).
 *   mean_c = (1/M) sum x,  var_c = (1/M) sum (x - mean_c)^2   (biased),
 *   xhat = (x - mean_c) / sqrt(var_c + eps),  y = gamma_c*xhat + beta_c,
 *   z = phi(y), written over x_inout.
 * x_inout   [N,C,H,W] in `d->layout`/`d->dtype`: x on entry, z on return.
 * gamma, beta [C] float32 (gamma may be negative; it must be nonzero for the
 *           backward to be defined).
 * eps >= 0.
 * save_mean, save_var [C] float32, written: the batch mean and the biased
 *           variance; iabn_backward and iabn_update_running_stats take them.
 * workspace, ws_bytes: scratch of at least iabn_workspace_size(d) bytes.
 * stream:   cudaStream_t the work is ordered on. */
iabn_status iabn_forward(const iabn_desc* d, void* x_inout,
                         const float* gamma, const float* beta, float eps,
                         int32_t act, float act_param,
                         float* save_mean, float* save_var,
                         void* workspace, size_t ws_bytes, void* stream);

/* iabn_forward and iabn_update_running_stats(C, M, ...) in one call: the
 * running statistics are updated by the forward's own finalize (the same
 * fp32 arithmetic, so the same bits as the two calls), which saves the
 * update's kernel launch.
 * running_mean, running_var [C] float32, updated in place; momentum in
 * [0, 1].  Other arguments, errors and the workspace as for iabn_forward. */
iabn_status iabn_forward_with_running_stats(const iabn_desc* d, void* x_inout,
                                            const float* gamma, const float* beta, float eps,
                                            int32_t act, float act_param,
                                            float* save_mean, float* save_var,
                                            float* running_mean, float* running_var,
                                            float momentum,
                                            void* workspace, size_t ws_bytes, void* stream);

/* Backward from the stored output only ([ABN] section 3, "INPLACE-ABN" and
 * "INPLACE-ABN II"; appendix "Derivation of Gradient dL").
 *   y = phi^-1(z); dy = dz * phi'(y) (phi' read from z);
 *   xhat = (y - beta_c)/gamma_c;  rstd = 1/sqrt(save_var_c + eps);
 *   dbeta_c = sum dy,  dgamma_c = sum dy*xhat,
 *   dx = gamma_c*rstd*(dy - dbeta_c/M - xhat*dgamma_c/M), written over dz.
 * ELU inverse: with t = z/alpha, y = log1p(t) when 1 + t > 2^-24, else
 *   y = ln(2^-24); its slope is max(z + alpha, 0).
 * z         [N,C,H,W]: exactly the tensor iabn_forward produced (not modified).
 * dz_inout  [N,C,H,W]: dL/dz on entry, dL/dx on return.  Must not alias z.
 * gamma, beta, save_var, eps, act, act_param: as passed to / returned by the
 *           forward call.
 * dgamma, dbeta [C] float32: written (not accumulated).
 * A channel with |gamma_c| < FLT_MIN gets NaN in dx, dgamma_c, dbeta_c and
 * sets IABN_ERR_SINGULAR_GAMMA in the workspace status word. */
iabn_status iabn_backward(const iabn_desc* d, const void* z, void* dz_inout,
                          const float* gamma, const float* beta,
                          const float* save_var, float eps,
                          int32_t act, float act_param,
                          float* dgamma, float* dbeta,
                          void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * The standard BN+ACT layer ([ABN] section 3, "Standard and Checkpointed
 * Computation"): it keeps both its input x (for the BN backward) and its
 * output z (for the activation's and the next layer's backward) -- the
 * layer InPlace-ABN is measured against.  Same statistics, arithmetic and
 * rounding as iabn_forward / iabn_backward; only what is stored differs.
 * ------------------------------------------------------------------------ */

/* Standard forward: as iabn_forward, but x is only read and z is written to
 * its own buffer.
 * x      [N,C,H,W] input, not modified.
 * z_out  [N,C,H,W] output; must not overlap x (IABN_ERR_INVALID_ARG) and
 *        must start on a 16-byte boundary (IABN_ERR_MISALIGNED).
 * Other arguments, errors and the workspace as for iabn_forward. */
iabn_status iabn_forward_standard(const iabn_desc* d, const void* x, void* z_out,
                                  const float* gamma, const float* beta, float eps,
                                  int32_t act, float act_param,
                                  float* save_mean, float* save_var,
                                  void* workspace, size_t ws_bytes, void* stream);

/* Standard backward from the stored input x ([BN] backward; [ABN]
 * "Standard and Checkpointed Computation"):
 *   rstd = 1/sqrt(save_var_c + eps),  xhat = (x - save_mean_c)*rstd,
 *   y = gamma_c*xhat + beta_c,  dy = dz*phi'(y),
 *   dbeta_c = sum dy,  dgamma_c = sum dy*xhat,
 *   dx = gamma_c*rstd*(dy - dbeta_c/M - xhat*dgamma_c/M), written over dz.
 * x         [N,C,H,W]: the forward's input (not modified).
 * dz_inout  [N,C,H,W]: dL/dz on entry, dL/dx on return; must not overlap x.
 * save_mean, save_var [C]: as returned by the forward.
 * gamma may be zero here (nothing is divided by it).  Other arguments and
 * errors as for iabn_backward. */
iabn_status iabn_backward_standard(const iabn_desc* d, const void* x, void* dz_inout,
                                   const float* gamma, const float* beta,
                                   const float* save_mean, const float* save_var, float eps,
                                   int32_t act, float act_param,
                                   float* dgamma, float* dbeta,
                                   void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * The optimized-checkpointing layer ([ABN] section 3, "Proposed
 * Checkpointing"): it keeps the normalised xhat in place of x; the backward
 * reaches y by the scale and shift alone and uses xhat in the BN backward as
 * it stands; z, which the next layer's backward needs, is recomputed from
 * xhat (iabn_checkpoint_recompute).
 * ------------------------------------------------------------------------ */

/* Checkpointing forward: the statistics of iabn_forward, then
 *   xhat = (x - mean_c)*rstd, written over x (storage type, one rounding),
 *   z = phi(gamma_c*xhat + beta_c), written to z_out.
 * x_inout [N,C,H,W]: x on entry, xhat on return.
 * z_out   [N,C,H,W]: must not overlap x_inout; 16-byte aligned.
 * Other arguments, errors and the workspace as for iabn_forward. */
iabn_status iabn_forward_checkpoint(const iabn_desc* d, void* x_inout, void* z_out,
                                    const float* gamma, const float* beta, float eps,
                                    int32_t act, float act_param,
                                    float* save_mean, float* save_var,
                                    void* workspace, size_t ws_bytes, void* stream);

/* z = phi(gamma_c*xhat + beta_c) from the stored xhat, for the layer that
 * follows (one elementwise pass; no statistics, no workspace).  M >= 1.
 * xhat    [N,C,H,W]: not modified unless z_out is the same buffer.
 * z_out   [N,C,H,W]: xhat itself or a buffer that does not overlap it. */
iabn_status iabn_checkpoint_recompute(const iabn_desc* d, const void* xhat, void* z_out,
                                      const float* gamma, const float* beta,
                                      int32_t act, float act_param, void* stream);

/* Checkpointing backward from the stored xhat:
 *   y = gamma_c*xhat + beta_c,  dy = dz*phi'(y),
 *   dbeta_c = sum dy,  dgamma_c = sum dy*xhat,
 *   dx = gamma_c*rstd*(dy - dbeta_c/M - xhat*dgamma_c/M), written over dz,
 *   rstd = 1/sqrt(save_var_c + eps).
 * xhat      [N,C,H,W]: as the checkpointing forward left it (not modified).
 * dz_inout  [N,C,H,W]: dL/dz on entry, dL/dx on return; must not overlap xhat.
 * gamma may be zero.  Other arguments and errors as for iabn_backward. */
iabn_status iabn_backward_checkpoint(const iabn_desc* d, const void* xhat, void* dz_inout,
                                     const float* gamma, const float* beta,
                                     const float* save_var, float eps,
                                     int32_t act, float act_param,
                                     float* dgamma, float* dbeta,
                                     void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * INPLACE-ABNsync ([ABN] section 4, "Semantic segmentation": the
 * segmentation results use synchronised statistics across GPUs).  The batch
 * is split along N over `world` GPUs; each GPU holds its shard, and the
 * statistics are those of the whole batch.  Each direction is two calls with
 * the exchange between them, which the caller does (e.g. one all-gather of
 * the per-GPU records with NCCL):
 *   forward:  iabn_sync_forward_stats -> gather the records of all GPUs ->
 *             iabn_sync_forward_apply;
 *   backward: iabn_sync_backward_stats -> gather -> iabn_sync_backward_apply.
 * A record is 3 float64 per channel, record[c*3 + i]:
 *   forward  (n, mean, M2) of this GPU's values of channel c, M2 = sum (x - mean)^2;
 *   backward (n, sum dy, sum dy*xhat) over this GPU's values.
 * `gathered` is [world][C][3] float64 (device memory), the records of GPUs
 * 0 .. world-1 in rank order; every GPU must pass the same array so that all
 * of them compute the same statistics (they are combined in rank order in
 * float64, so they agree bitwise).  With world = 1 the layer is the plain
 * in-place layer (same arithmetic up to the summation order).
 * The descriptor of each call is this GPU's shard; shards may differ in N.
 * ------------------------------------------------------------------------ */

/* This GPU's forward record of x (n = N*H*W of the shard).
 * x [N,C,H,W]: not modified.  stats [C*3] float64, written. */
iabn_status iabn_sync_forward_stats(const iabn_desc* d, const void* x, double* stats,
                                    void* workspace, size_t ws_bytes, void* stream);

/* Combines the gathered forward records into the whole batch's
 *   mean_c = sum_r n_r mean_r / Mt,  var_c = M2_c / Mt  (Mt = sum_r n_r; biased),
 * writes save_mean, save_var (the whole batch's) and overwrites x with
 *   z = phi(gamma_c*(x - mean_c)/sqrt(var_c + eps) + beta_c)
 * as iabn_forward does.  world >= 1; the records' n must sum to >= 2.
 * Other arguments as for iabn_forward. */
iabn_status iabn_sync_forward_apply(const iabn_desc* d, void* x_inout, const double* gathered,
                                    int32_t world, const float* gamma, const float* beta,
                                    float eps, int32_t act, float act_param,
                                    float* save_mean, float* save_var,
                                    void* workspace, size_t ws_bytes, void* stream);

/* This GPU's backward record from z and dz (y and xhat recovered from z as
 * iabn_backward does; dy = dz*phi'(y)).  z, dz not modified.  stats [C*3]
 * float64, written.  gamma, beta, act, act_param as passed to the forward. */
iabn_status iabn_sync_backward_stats(const iabn_desc* d, const void* z, const void* dz,
                                     const float* gamma, const float* beta,
                                     int32_t act, float act_param, double* stats,
                                     void* workspace, size_t ws_bytes, void* stream);

/* Combines the gathered backward records (sums in rank order) into the whole
 * batch's dbeta_c = sum dy and dgamma_c = sum dy*xhat, writes them, and
 * overwrites dz with
 *   dx = gamma_c*rstd*(dy - dbeta_c/Mt - xhat*dgamma_c/Mt),  Mt = sum_r n_r,
 * rstd = 1/sqrt(save_var_c + eps) (save_var: the whole batch's, from
 * iabn_sync_forward_apply).  |gamma_c| < FLT_MIN: as for iabn_backward.
 * Other arguments as for iabn_backward. */
iabn_status iabn_sync_backward_apply(const iabn_desc* d, const void* z, void* dz_inout,
                                     const double* gathered, int32_t world,
                                     const float* gamma, const float* beta,
                                     const float* save_var, float eps,
                                     int32_t act, float act_param,
                                     float* dgamma, float* dbeta,
                                     void* workspace, size_t ws_bytes, void* stream);

/* Inference, i.e. evaluation mode ([BN] Algorithm 2, the inference network;
 * [ABN] section 3, "Batch Normalization Review" for the scale and shift):
 *   xhat = (x - running_mean_c) / sqrt(running_var_c + eps),
 *   z = phi(gamma_c*xhat + beta_c), written over x_inout.
 * No statistics are computed or written; M >= 1.
 * x_inout   [N,C,H,W] in `d->layout`/`d->dtype`: x on entry, z on return.
 * gamma, beta, running_mean, running_var [C] float32; running_var_c + eps
 *           must be > 0.
 * eps >= 0; act, act_param as for iabn_forward.
 * workspace, ws_bytes: checked as for iabn_forward but not used (the pass
 *           forms its coefficients itself).
 * One kernel launch.  Arguments are checked as for iabn_forward. */
iabn_status iabn_inference(const iabn_desc* d, void* x_inout,
                           const float* gamma, const float* beta,
                           const float* running_mean, const float* running_var, float eps,
                           int32_t act, float act_param,
                           void* workspace, size_t ws_bytes, void* stream);

/* Running statistics ([BN] Algorithm 2 uses the unbiased variance for
 * inference; the momentum form is the usual framework convention):
 *   running_mean <- (1 - momentum)*running_mean + momentum*save_mean,
 *   running_var  <- (1 - momentum)*running_var + momentum*save_var*count/(count - 1).
 * c: number of channels; count: M of the forward call (>= 2);
 * momentum in [0, 1].  running_mean, running_var [C] float32, updated in place. */
iabn_status iabn_update_running_stats(int64_t c, int64_t count,
                                      const float* save_mean, const float* save_var,
                                      float* running_mean, float* running_var,
                                      float momentum, void* stream);

/* Synchronises `stream`, reads the workspace's sticky device status and
 * clears it (resetting the workspace's control block for reuse).  Returns
 * IABN_OK, IABN_ERR_TIMEOUT, IABN_ERR_SINGULAR_GAMMA (the most severe
 * condition seen since the last read), or IABN_ERR_CUDA if the stream or a
 * copy failed.  After IABN_ERR_TIMEOUT the outputs of the call(s) that timed
 * out are undefined; the workspace itself stays usable (later calls are
 * correct whether or not the status has been read in between). */
iabn_status iabn_get_device_status(void* workspace, void* stream);

/* Diagnostics: the number of kernels this library has launched in this
 * process so far (all devices, all threads).  Host-only; never fails. */
uint64_t iabn_kernel_launches(void);

/* The calls iabn_describe_plan describes. */
typedef enum {
    IABN_CALL_FORWARD = 0,              /* iabn_forward */
    IABN_CALL_BACKWARD = 1,             /* iabn_backward */
    IABN_CALL_FORWARD_STANDARD = 2,     /* iabn_forward_standard */
    IABN_CALL_BACKWARD_STANDARD = 3,    /* iabn_backward_standard */
    IABN_CALL_FORWARD_CHECKPOINT = 4,   /* iabn_forward_checkpoint */
    IABN_CALL_BACKWARD_CHECKPOINT = 5   /* iabn_backward_checkpoint */
} iabn_call;

/* Launch plans (see iabn_describe_plan). */
typedef enum {
    IABN_PLAN_TWOPHASE = 0,   /* statistics, finalize, apply: three plain launches */
    IABN_PLAN_RESIDENT = 1    /* one cooperative persistent launch, one CTA per SM */
} iabn_plan;

/* Launch shape of one call; filled by iabn_describe_plan.  The fields after
 * `launches` describe the resident plan and are 0 for the two-phase plan. */
typedef struct {
    int32_t plan;               /* iabn_plan */
    int32_t launches;           /* kernels one iabn_forward / iabn_backward call launches */
    int32_t grid;               /* CTAs (at most one per SM) */
    int32_t threads;            /* threads per CTA */
    int32_t smem_bytes;         /* dynamic shared memory per CTA */
    int32_t tile_bytes;         /* bytes of each streamed tensor per full tile */
    int32_t slots;              /* tile slots in shared memory */
    int32_t ring;               /* slots the stream cycles through (<= slots) */
    int32_t vectors_per_row;    /* NHWC: 16-byte vectors in a row of C channels; NCHW: 0 */
    int32_t cols_per_thread;    /* NHWC: 16-byte columns each consumer thread owns */
    int32_t row_phases;         /* NHWC: consumer threads sharing one column */
    int32_t planes_per_unit;    /* NCHW: whole H*W planes per 16-byte aligned unit */
    int32_t stash_rows;         /* NHWC: rows per consumer thread kept in Tensor Memory
                                   between the two passes (0: none) */
    int32_t stash_copy_engine;  /* 1: tcgen05.cp fills that stash from shared memory */
} iabn_plan_info;

/* Which plan the training call `call` (an iabn_call value) takes for
 * descriptor d, and its launch shape, as decided on the host; the same
 * environment settings apply (IABN_FORCE_PLAN=twophase, tile and ring
 * sizes).  A layer's two calls take the same plan.  A resident launch the driver refuses at run time (e.g. too few
 * co-resident CTAs) still falls back to the two-phase plan; that is not
 * predicted here.
 * sm_count, smem_optin: the device's SM count and opt-in shared memory per
 * block in bytes (B200: 148 and 232448); both 0 = query the current device
 * (IABN_ERR_CUDA if there is none).  With both given no CUDA call is made.
 * Returns the descriptor errors of iabn_forward, IABN_ERR_INVALID_ARG for a
 * null `out`, an unknown call or a negative or half-given limit pair, else
 * IABN_OK with *out filled. */
iabn_status iabn_describe_plan(const iabn_desc* d, int32_t call, int32_t sm_count,
                               int32_t smem_optin, iabn_plan_info* out);

/* iabn_forward without a caller-supplied workspace.  The paper has no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory -- e.g. a plugin inside a framework whose own allocator owns
 * the GPU's memory, or a real-time loop that forbids allocation after
 * start-up.  They still pass x_inout, gamma, beta, save_mean and save_var
 * exactly as for iabn_forward; the scratch comes from an 8 MiB array of
 * device memory that the library reserves on every GPU that loads it, held
 * until the process exits.  No call allocates or frees memory.
 *   - Descriptors whose iabn_workspace_size exceeds 8 MiB (8388608 bytes) are
 *     rejected with IABN_ERR_WORKSPACE before anything is launched; other
 *     argument errors are reported as by iabn_forward.
 *   - The first call on a device (that device current) looks up the array's
 *     device address and keeps it for the life of the process; make that
 *     first call before any stream capture.  A cudaDeviceReset of the device
 *     discards the array: do not call this entry point on that device after
 *     one.
 *   - All calls on a device share the one array: calls that overlap on the
 *     GPU (other streams, other host threads) race and give wrong results.
 *     Each call zeroes the array's control block on `stream` before its
 *     kernels, so device-side conditions of one call (a bounded wait that ran
 *     out) are not carried into the next; iabn_get_static_ws_status reads
 *     them after the call. */
iabn_status iabn_forward_static_ws(const iabn_desc* d, void* x_inout,
                                   const float* gamma, const float* beta, float eps,
                                   int32_t act, float act_param,
                                   float* save_mean, float* save_var, void* stream);

/* The device status of the iabn_forward_static_ws calls on the current
 * device since its last call or the last read: synchronises `stream`, then
 * reads and clears the status word of the library's own scratch, as
 * iabn_get_device_status does for a caller's workspace (same return values;
 * IABN_OK before any such call).  Each iabn_forward_static_ws call starts
 * from a cleared status, so read it after the call that matters. */
iabn_status iabn_get_static_ws_status(void* stream);

#ifdef __cplusplus
}
#endif
#endif /* IABN_H */
