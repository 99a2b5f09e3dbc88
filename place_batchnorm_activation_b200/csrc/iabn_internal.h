// iabn_internal.h -- host-side types shared by the C-ABI layer and the two
// launch plans (split "two-phase" and co-resident "resident").
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace iabn {

struct Control;

// Validated geometry of one call.
struct Geom {
    int64_t N, C, HW;
    int64_t R;       // N*HW: rows of the NHWC matrix [R x C]
    int64_t M;       // values per channel (= R)
    int64_t E;       // N*C*HW elements
    int layout;      // kNCHW / kNHWC
    int dtype;       // kF32 / kBF16 / kF16
    int esize;       // bytes per stored element
};

// Workspace carve-up: [Control | trace | partials (double2) | coef (2 float4
// records per channel)].
struct Workspace {
    Control* ctl;
    unsigned long long* trace;
    double2* part;
    float4* coef;
};

// Layers: which buffer each keeps for its backward.
//   kLayerInPlace   z only (INPLACE-ABN): forward kModeFwd over x, backward kModeBwdZ
//   kLayerStandard  x and z: forward kModeFwd into its own buffer, backward kModeBwdX
//   kLayerCkpt      xhat: forward kModeFwdCkpt, backward kModeBwdXhat
enum : int { kLayerInPlace = 0, kLayerStandard = 1, kLayerCkpt = 2 };

struct FwdArgs {
    const void* x;
    void* dst;            // z (kModeFwd) or xhat (kModeFwdCkpt)
    void* dst2;           // kModeFwdCkpt: z
    int mode;             // kModeFwd or kModeFwdCkpt
    int layer;            // kLayer*
    const float* gamma;
    const float* beta;
    float eps;
    int act;
    float act_param;
    float* save_mean;
    float* save_var;
    // optional: the running statistics, updated in the finalize with the
    // arithmetic of running_update (count M); null: not updated
    float* running_mean = nullptr;
    float* running_var = nullptr;
    float momentum = 0.f;
};

struct BwdArgs {
    const void* src;      // z (kModeBwdZ), x (kModeBwdX) or xhat (kModeBwdXhat)
    void* dz;
    int mode;
    int layer;
    const float* gamma;
    const float* beta;
    const float* save_mean;   // kModeBwdX
    const float* save_var;
    float eps;
    int act;
    float act_param;
    float* dgamma;
    float* dbeta;
};

struct InfArgs {
    void* x;
    const float* gamma;
    const float* beta;
    const float* running_mean;
    const float* running_var;
    float eps;
    int act;
    float act_param;
};

// Host-side count of kernel launches (diagnostics; see iabn_kernel_launches).
void count_launches(int n);

// Number of double2 partial slots the workspace reserves for geometry g.
int64_t partial_slots(const Geom& g);

cudaError_t forward_twophase(const Geom& g, const FwdArgs& a, const Workspace& w,
                             cudaStream_t s, int sms);
cudaError_t backward_twophase(const Geom& g, const BwdArgs& a, const Workspace& w,
                              cudaStream_t s, int sms);
// One-launch elementwise passes (iabn_elementwise.cu): evaluation mode from
// the running statistics; the checkpointing layer's z = phi(gamma*xhat +
// beta); the two-phase forward's apply from its finalize's coefficients.
cudaError_t inference_pass(const Geom& g, const InfArgs& a, cudaStream_t s, int sms);
cudaError_t recompute_pass(const Geom& g, const void* xhat, void* z, const float* gamma,
                           const float* beta, int act, float act_param, cudaStream_t s,
                           int sms);
cudaError_t forward_apply_pass(const Geom& g, const FwdArgs& f, const float4* coef,
                               cudaStream_t s, int sms, int nseg = 0);
// INPLACE-ABNsync (iabn_twophase.cu): this GPU's per-channel record (3
// doubles per channel), and the apply from the records of all GPUs
// ([world][C][3], rank order).
cudaError_t sync_forward_stats(const Geom& g, const void* x, double* rec, const Workspace& w,
                               cudaStream_t s, int sms);
cudaError_t sync_forward_apply(const Geom& g, const FwdArgs& a, const double* gathered,
                               int world, const Workspace& w, cudaStream_t s, int sms);
cudaError_t sync_backward_stats(const Geom& g, const BwdArgs& a, double* rec,
                                const Workspace& w, cudaStream_t s, int sms);
cudaError_t sync_backward_apply(const Geom& g, const BwdArgs& a, const double* gathered,
                                int world, const Workspace& w, cudaStream_t s, int sms);
cudaError_t running_update(int64_t C, int64_t count, const float* mean, const float* var,
                           float* rmean, float* rvar, float momentum, cudaStream_t s);

// Resident plan: returns cudaErrorNotSupported when the shape is outside what
// it handles (the caller then uses the two-phase plan), or the launch error.
cudaError_t forward_resident(const Geom& g, const FwdArgs& a, const Workspace& w,
                             cudaStream_t s);
cudaError_t backward_resident(const Geom& g, const BwdArgs& a, const Workspace& w,
                              cudaStream_t s);
// Both calls of the layer qualify for the resident plan on the current device.
bool resident_supported(const Geom& g, int layer);

// Launch shape of the resident plan in one direction (iabn_describe_plan).
struct ResidentShape {
    int grid, threads, smem_bytes, tile_bytes, slots, ring;
    int vectors_per_row, cols_per_thread, row_phases, planes_per_unit;
    int stash_rows, stash_copy_engine;
};

// True, with `out` filled for direction dir (0 forward, 1 backward) of
// `layer`, if the calls on g take the resident plan on a device with `sms`
// SMs and `smem_optin` bytes of opt-in shared memory per block (both calls of
// the layer must qualify, as in resident_supported).  Host only: no CUDA call.
bool resident_shape(const Geom& g, int layer, int dir, int sms, int smem_optin,
                    ResidentShape& out);

}  // namespace iabn
