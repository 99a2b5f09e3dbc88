// iabn_api.cu -- the extern "C" entry points declared in include/iabn.h:
// argument checks, workspace carve-up, plan choice and launch.
//
// Plan choice: the resident plan (one co-resident grid per call, data staged
// through shared memory, grid-wide statistics) when the shape qualifies,
// else the split two-phase plan.  IABN_FORCE_PLAN=twophase|resident in the
// environment forces one (a shape the resident plan does not take still runs
// two-phase; a resident launch that fails is then reported, not replaced).
// IABN_DEBUG=1 prints CUDA errors to stderr.
#include <cuda_runtime.h>
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "iabn.h"
#include "iabn_device.cuh"
#include "iabn_internal.h"

namespace iabn {

static std::atomic<uint64_t> g_launches{0};

void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

int64_t partial_slots(const Geom& g) {
    return g.layout == kNHWC ? (int64_t)kMaxPartialBlocks * g.C : g.N * g.C;
}

static size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

static size_t workspace_bytes(const Geom& g) {
    return round_up(sizeof(Control) + kTraceBytes + (size_t)partial_slots(g) * sizeof(double2) +
                        (size_t)g.C * sizeof(float4),
                    256);
}

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Checks the descriptor; fills g.  Returns IABN_OK or the error.  min_m is
// the least number of values per channel the call accepts: 2 for the
// training calls (a variance needs two values), 1 for inference.
static iabn_status make_geom(const iabn_desc* d, Geom& g, int64_t min_m = 2) {
    if (!d) return IABN_ERR_INVALID_ARG;
    if (d->n <= 0 || d->c <= 0 || d->h <= 0 || d->w <= 0) return IABN_ERR_INVALID_ARG;
    if (d->layout != IABN_NCHW && d->layout != IABN_NHWC) return IABN_ERR_INVALID_ARG;
    if (d->dtype != IABN_F32 && d->dtype != IABN_BF16 && d->dtype != IABN_F16)
        return IABN_ERR_INVALID_ARG;
    const int64_t lim = (int64_t)1 << 40;
    if (d->n > lim || d->c > lim || d->h > lim || d->w > lim) return IABN_ERR_UNSUPPORTED;
    // launch-grid limit: the NHWC reductions of the two-phase plan put blocks of
    // 256 channels on the grid's y dimension (at most 65535)
    if (d->c > (int64_t)65535 * 256) return IABN_ERR_UNSUPPORTED;
    const __int128 hw = (__int128)d->h * d->w;
    const __int128 m = hw * d->n;
    const __int128 e = m * d->c;
    if (e * 4 > (__int128)INT64_MAX / 2) return IABN_ERR_UNSUPPORTED;
    if (m < min_m) return IABN_ERR_INVALID_ARG;
    // Partial slots and the count of values per channel must stay exact.
    if ((__int128)d->n * d->c > ((__int128)1 << 40)) return IABN_ERR_UNSUPPORTED;
    if (m > ((__int128)1 << 52)) return IABN_ERR_UNSUPPORTED;
    g.N = d->n;
    g.C = d->c;
    g.HW = (int64_t)hw;
    g.R = (int64_t)m;
    g.M = (int64_t)m;
    g.E = (int64_t)e;
    g.layout = d->layout;
    g.dtype = d->dtype;
    g.esize = d->dtype == IABN_F32 ? 4 : 2;
    return IABN_OK;
}

static iabn_status check_act(int32_t act, float p) {
    if (act == IABN_ACT_IDENTITY) return IABN_OK;
    if (act != IABN_ACT_LEAKY_RELU && act != IABN_ACT_ELU) return IABN_ERR_INVALID_ARG;
    if (!(p > 0.f) || !isfinite(p)) return IABN_ERR_INVALID_ARG;
    return IABN_OK;
}

static Workspace carve(void* ws, const Geom& g) {
    Workspace w;
    char* base = static_cast<char*>(ws);
    w.ctl = reinterpret_cast<Control*>(base);
    w.trace = reinterpret_cast<unsigned long long*>(base + sizeof(Control));
    w.part = reinterpret_cast<double2*>(base + sizeof(Control) + kTraceBytes);
    w.coef = reinterpret_cast<float4*>(base + sizeof(Control) + kTraceBytes +
                                       (size_t)partial_slots(g) * sizeof(double2));
    return w;
}

// Per-device SM count, queried once per device.
static int device_sms(int dev) {
    static std::mutex mu;
    static int cache[64] = {0};
    if (dev < 0 || dev >= 64) return 148;
    std::lock_guard<std::mutex> lock(mu);
    if (cache[dev] == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            v <= 0)
            v = 148;
        cache[dev] = v;
    }
    return cache[dev];
}

enum Plan { kAuto = 0, kTwoPhase = 1, kResident = 2 };

static Plan forced_plan() {
    const char* s = getenv("IABN_FORCE_PLAN");
    if (!s) return kAuto;
    if (strcmp(s, "twophase") == 0) return kTwoPhase;
    if (strcmp(s, "resident") == 0) return kResident;
    return kAuto;
}

static iabn_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return IABN_OK;
    cudaGetLastError();   // clear a sticky launch error so later calls are not blamed
    if (getenv("IABN_DEBUG")) fprintf(stderr, "iabn: CUDA error %d: %s\n", (int)e,
                                      cudaGetErrorString(e));
    return IABN_ERR_CUDA;
}

// Launch-configuration errors after which nothing ran, so the two-phase plan
// may run instead.
static bool resident_declined(cudaError_t e) {
    return e == cudaErrorNotSupported || e == cudaErrorCooperativeLaunchTooLarge ||
           e == cudaErrorInvalidValue || e == cudaErrorLaunchOutOfResources ||
           e == cudaErrorInvalidConfiguration;
}

}  // namespace iabn

using namespace iabn;

extern "C" size_t iabn_workspace_size(const iabn_desc* d) {
    Geom g;
    if (make_geom(d, g, 1) != IABN_OK) return 0;
    return workspace_bytes(g);
}

extern "C" iabn_status iabn_forward(const iabn_desc* d, void* x_inout, const float* gamma,
                                    const float* beta, float eps, int32_t act, float act_param,
                                    float* save_mean, float* save_var, void* workspace,
                                    size_t ws_bytes, void* stream) {
    Geom g;
    iabn_status st = make_geom(d, g);
    if (st != IABN_OK) return st;
    if (!x_inout || !gamma || !beta || !save_mean || !save_var) return IABN_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !isfinite(eps)) return IABN_ERR_INVALID_ARG;
    if ((st = check_act(act, act_param)) != IABN_OK) return st;
    if (!aligned16(x_inout)) return IABN_ERR_MISALIGNED;
    if (!workspace || ws_bytes < workspace_bytes(g) || !aligned16(workspace))
        return IABN_ERR_WORKSPACE;
    FwdArgs a{x_inout, gamma, beta, eps, (int)act, act_param, save_mean, save_var};
    const Workspace w = carve(workspace, g);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return from_cuda(cudaErrorNoDevice);
    const Plan plan = forced_plan();
    if (plan != kTwoPhase && resident_supported(g)) {
        cudaError_t e = forward_resident(g, a, w, s);
        if (e == cudaSuccess || plan == kResident || !resident_declined(e)) return from_cuda(e);
        cudaGetLastError();
    }
    return from_cuda(forward_twophase(g, a, w, s, device_sms(dev)));
}

extern "C" iabn_status iabn_backward(const iabn_desc* d, const void* z, void* dz_inout,
                                     const float* gamma, const float* beta,
                                     const float* save_var, float eps, int32_t act,
                                     float act_param, float* dgamma, float* dbeta,
                                     void* workspace, size_t ws_bytes, void* stream) {
    Geom g;
    iabn_status st = make_geom(d, g);
    if (st != IABN_OK) return st;
    if (!z || !dz_inout || !gamma || !beta || !save_var || !dgamma || !dbeta)
        return IABN_ERR_INVALID_ARG;
    if (z == dz_inout) return IABN_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !isfinite(eps)) return IABN_ERR_INVALID_ARG;
    if ((st = check_act(act, act_param)) != IABN_OK) return st;
    if (!aligned16(z) || !aligned16(dz_inout)) return IABN_ERR_MISALIGNED;
    if (!workspace || ws_bytes < workspace_bytes(g) || !aligned16(workspace))
        return IABN_ERR_WORKSPACE;
    BwdArgs a{z, dz_inout, gamma, beta, save_var, eps, (int)act, act_param, dgamma, dbeta};
    const Workspace w = carve(workspace, g);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return from_cuda(cudaErrorNoDevice);
    const Plan plan = forced_plan();
    if (plan != kTwoPhase && resident_supported(g)) {
        cudaError_t e = backward_resident(g, a, w, s);
        if (e == cudaSuccess || plan == kResident || !resident_declined(e)) return from_cuda(e);
        cudaGetLastError();
    }
    return from_cuda(backward_twophase(g, a, w, s, device_sms(dev)));
}

extern "C" iabn_status iabn_inference(const iabn_desc* d, void* x_inout, const float* gamma,
                                      const float* beta, const float* running_mean,
                                      const float* running_var, float eps, int32_t act,
                                      float act_param, void* workspace, size_t ws_bytes,
                                      void* stream) {
    Geom g;
    iabn_status st = make_geom(d, g, 1);
    if (st != IABN_OK) return st;
    if (!x_inout || !gamma || !beta || !running_mean || !running_var) return IABN_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !isfinite(eps)) return IABN_ERR_INVALID_ARG;
    if ((st = check_act(act, act_param)) != IABN_OK) return st;
    if (!aligned16(x_inout)) return IABN_ERR_MISALIGNED;
    if (!workspace || ws_bytes < workspace_bytes(g) || !aligned16(workspace))
        return IABN_ERR_WORKSPACE;
    InfArgs a{x_inout, gamma, beta, running_mean, running_var, eps, (int)act, act_param};
    const Workspace w = carve(workspace, g);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return from_cuda(cudaErrorNoDevice);
    return from_cuda(inference_twophase(g, a, w, static_cast<cudaStream_t>(stream),
                                        device_sms(dev)));
}

extern "C" iabn_status iabn_update_running_stats(int64_t c, int64_t count,
                                                 const float* save_mean, const float* save_var,
                                                 float* running_mean, float* running_var,
                                                 float momentum, void* stream) {
    if (c <= 0 || count < 2) return IABN_ERR_INVALID_ARG;
    if (!save_mean || !save_var || !running_mean || !running_var) return IABN_ERR_INVALID_ARG;
    if (!(momentum >= 0.f && momentum <= 1.f)) return IABN_ERR_INVALID_ARG;
    return from_cuda(running_update(c, count, save_mean, save_var, running_mean, running_var,
                                    momentum, static_cast<cudaStream_t>(stream)));
}

extern "C" iabn_status iabn_get_device_status(void* workspace, void* stream) {
    if (!workspace) return IABN_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Control* ctl = static_cast<Control*>(workspace);
    uint32_t bits = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess) return from_cuda(cudaErrorUnknown);
    if (cudaMemcpyAsync(&bits, &ctl->status, sizeof(bits), cudaMemcpyDeviceToHost, s) !=
        cudaSuccess)
        return from_cuda(cudaErrorUnknown);
    if (cudaMemsetAsync(ctl, 0, sizeof(Control), s) != cudaSuccess)
        return from_cuda(cudaErrorUnknown);
    if (cudaStreamSynchronize(s) != cudaSuccess) return from_cuda(cudaErrorUnknown);
    if (bits & kStTimeout) return IABN_ERR_TIMEOUT;
    if (bits & kStSingular) return IABN_ERR_SINGULAR_GAMMA;
    return IABN_OK;
}

extern "C" uint64_t iabn_kernel_launches(void) {
    return g_launches.load(std::memory_order_relaxed);
}

extern "C" iabn_status iabn_describe_plan(const iabn_desc* d, int32_t direction,
                                          int32_t sm_count, int32_t smem_optin,
                                          iabn_plan_info* out) {
    Geom g;
    iabn_status st = make_geom(d, g);
    if (st != IABN_OK) return st;
    if (!out || (direction != 0 && direction != 1)) return IABN_ERR_INVALID_ARG;
    if (sm_count < 0 || smem_optin < 0 || (sm_count == 0) != (smem_optin == 0))
        return IABN_ERR_INVALID_ARG;
    if (sm_count == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return from_cuda(cudaErrorNoDevice);
        int sms = 0, smem = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
                cudaSuccess)
            return from_cuda(cudaErrorUnknown);
        sm_count = sms;
        smem_optin = smem;
    }
    memset(out, 0, sizeof(*out));
    ResidentShape r;
    if (forced_plan() != kTwoPhase && resident_shape(g, direction, sm_count, smem_optin, r)) {
        out->plan = IABN_PLAN_RESIDENT;
        out->launches = 1;
        out->grid = r.grid;
        out->threads = r.threads;
        out->smem_bytes = r.smem_bytes;
        out->tile_bytes = r.tile_bytes;
        out->slots = r.slots;
        out->ring = r.ring;
        out->vectors_per_row = r.vectors_per_row;
        out->cols_per_thread = r.cols_per_thread;
        out->row_phases = r.row_phases;
        out->planes_per_unit = r.planes_per_unit;
        out->stash_rows = r.stash_rows;
        out->stash_copy_engine = r.stash_copy_engine;
    } else {
        out->plan = IABN_PLAN_TWOPHASE;
        out->launches = 3;
    }
    return IABN_OK;
}
