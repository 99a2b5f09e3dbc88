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

// Workspace carve-up: [Control | trace | partials (double2) | coef (float4)].
struct Workspace {
    Control* ctl;
    unsigned long long* trace;
    double2* part;
    float4* coef;
};

struct FwdArgs {
    void* x;
    const float* gamma;
    const float* beta;
    float eps;
    int act;
    float act_param;
    float* save_mean;
    float* save_var;
};

struct BwdArgs {
    const void* z;
    void* dz;
    const float* gamma;
    const float* beta;
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
// Evaluation mode: coefficients from the running statistics, then the
// forward's elementwise pass (two launches).
cudaError_t inference_twophase(const Geom& g, const InfArgs& a, const Workspace& w,
                               cudaStream_t s, int sms);
cudaError_t running_update(int64_t C, int64_t count, const float* mean, const float* var,
                           float* rmean, float* rvar, float momentum, cudaStream_t s);

// Resident plan: returns cudaErrorNotSupported when the shape is outside what
// it handles (the caller then uses the two-phase plan), or the launch error.
cudaError_t forward_resident(const Geom& g, const FwdArgs& a, const Workspace& w,
                             cudaStream_t s);
cudaError_t backward_resident(const Geom& g, const BwdArgs& a, const Workspace& w,
                              cudaStream_t s);
bool resident_supported(const Geom& g);

// Launch shape of the resident plan in one direction (iabn_describe_plan).
struct ResidentShape {
    int grid, threads, smem_bytes, tile_bytes, slots, ring;
    int vectors_per_row, cols_per_thread, row_phases, planes_per_unit;
    int stash_rows, stash_copy_engine;
};

// True, with `out` filled for direction dir (0 forward, 1 backward), if the
// calls on g take the resident plan on a device with `sms` SMs and
// `smem_optin` bytes of opt-in shared memory per block (both directions must
// qualify, as in resident_supported).  Host only: no CUDA call.
bool resident_shape(const Geom& g, int dir, int sms, int smem_optin, ResidentShape& out);

}  // namespace iabn
