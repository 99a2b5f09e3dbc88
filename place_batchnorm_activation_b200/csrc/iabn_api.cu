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
                        2 * (size_t)g.C * sizeof(float4),
                    256);
}

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// True if the two activation tensors of g at a and b share any byte.
static bool overlap(const Geom& g, const void* a, const void* b) {
    const uintptr_t n = (uintptr_t)g.E * (uintptr_t)g.esize;
    const uintptr_t pa = (uintptr_t)a, pb = (uintptr_t)b;
    return pa < pb + n && pb < pa + n;
}

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

// Checks shared by the training forward calls; fills g.  z_out: the separate
// output of the standard and checkpointing forwards (nullptr for the in-place
// one, which writes over x).
static iabn_status check_forward(const iabn_desc* d, Geom& g, const void* x, const void* z_out,
                                 bool separate_out, const float* gamma, const float* beta,
                                 float eps, int32_t act, float act_param,
                                 const float* save_mean, const float* save_var,
                                 const void* workspace, size_t ws_bytes, int64_t min_m = 2) {
    iabn_status st = make_geom(d, g, min_m);
    if (st != IABN_OK) return st;
    if (!x || !gamma || !beta || !save_mean || !save_var) return IABN_ERR_INVALID_ARG;
    if (separate_out && (!z_out || overlap(g, x, z_out))) return IABN_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !isfinite(eps)) return IABN_ERR_INVALID_ARG;
    if ((st = check_act(act, act_param)) != IABN_OK) return st;
    if (!aligned16(x) || (separate_out && !aligned16(z_out))) return IABN_ERR_MISALIGNED;
    if (!workspace || ws_bytes < workspace_bytes(g) || !aligned16(workspace))
        return IABN_ERR_WORKSPACE;
    return IABN_OK;
}

// Checks shared by the backward calls; fills g.  src is z, x or xhat.
static iabn_status check_backward(const iabn_desc* d, Geom& g, const void* src, const void* dz,
                                  const float* gamma, const float* beta, const float* save_var,
                                  float eps, int32_t act, float act_param, const float* dgamma,
                                  const float* dbeta, const void* workspace, size_t ws_bytes,
                                  bool need_mean = false, const float* save_mean = nullptr,
                                  int64_t min_m = 2) {
    iabn_status st = make_geom(d, g, min_m);
    if (st != IABN_OK) return st;
    if (!src || !dz || !gamma || !beta || !save_var || !dgamma || !dbeta)
        return IABN_ERR_INVALID_ARG;
    if (need_mean && !save_mean) return IABN_ERR_INVALID_ARG;
    if (overlap(g, src, dz)) return IABN_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !isfinite(eps)) return IABN_ERR_INVALID_ARG;
    if ((st = check_act(act, act_param)) != IABN_OK) return st;
    if (!aligned16(src) || !aligned16(dz)) return IABN_ERR_MISALIGNED;
    if (!workspace || ws_bytes < workspace_bytes(g) || !aligned16(workspace))
        return IABN_ERR_WORKSPACE;
    return IABN_OK;
}

// The resident plan when both calls of the layer qualify, else (or when the
// driver declines the launch) the two-phase plan.
static iabn_status run_forward(const Geom& g, const FwdArgs& a, void* workspace,
                               cudaStream_t s) {
    const Workspace w = carve(workspace, g);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return from_cuda(cudaErrorNoDevice);
    const Plan plan = forced_plan();
    if (plan != kTwoPhase && resident_supported(g, a.layer)) {
        cudaError_t e = forward_resident(g, a, w, s);
        if (e == cudaSuccess || plan == kResident || !resident_declined(e)) return from_cuda(e);
        cudaGetLastError();
    }
    return from_cuda(forward_twophase(g, a, w, s, device_sms(dev)));
}

static iabn_status run_backward(const Geom& g, const BwdArgs& a, void* workspace,
                                cudaStream_t s) {
    const Workspace w = carve(workspace, g);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return from_cuda(cudaErrorNoDevice);
    const Plan plan = forced_plan();
    if (plan != kTwoPhase && resident_supported(g, a.layer)) {
        cudaError_t e = backward_resident(g, a, w, s);
        if (e == cudaSuccess || plan == kResident || !resident_declined(e)) return from_cuda(e);
        cudaGetLastError();
    }
    return from_cuda(backward_twophase(g, a, w, s, device_sms(dev)));
}

extern "C" iabn_status iabn_forward(const iabn_desc* d, void* x_inout, const float* gamma,
                                    const float* beta, float eps, int32_t act, float act_param,
                                    float* save_mean, float* save_var, void* workspace,
                                    size_t ws_bytes, void* stream) {
    Geom g;
    const iabn_status st = check_forward(d, g, x_inout, nullptr, false, gamma, beta, eps, act,
                                         act_param, save_mean, save_var, workspace, ws_bytes);
    if (st != IABN_OK) return st;
    const FwdArgs a{x_inout, x_inout, nullptr, kModeFwd, kLayerInPlace, gamma, beta, eps,
                    (int)act, act_param, save_mean, save_var};
    return run_forward(g, a, workspace, static_cast<cudaStream_t>(stream));
}

extern "C" iabn_status iabn_forward_with_running_stats(
    const iabn_desc* d, void* x_inout, const float* gamma, const float* beta, float eps,
    int32_t act, float act_param, float* save_mean, float* save_var, float* running_mean,
    float* running_var, float momentum, void* workspace, size_t ws_bytes, void* stream) {
    if (!running_mean || !running_var) return IABN_ERR_INVALID_ARG;
    if (!(momentum >= 0.f && momentum <= 1.f)) return IABN_ERR_INVALID_ARG;
    Geom g;
    const iabn_status st = check_forward(d, g, x_inout, nullptr, false, gamma, beta, eps, act,
                                         act_param, save_mean, save_var, workspace, ws_bytes);
    if (st != IABN_OK) return st;
    FwdArgs a{x_inout, x_inout, nullptr, kModeFwd, kLayerInPlace, gamma, beta, eps, (int)act,
              act_param, save_mean, save_var};
    a.running_mean = running_mean;
    a.running_var = running_var;
    a.momentum = momentum;
    return run_forward(g, a, workspace, static_cast<cudaStream_t>(stream));
}

extern "C" iabn_status iabn_forward_standard(const iabn_desc* d, const void* x, void* z_out,
                                             const float* gamma, const float* beta, float eps,
                                             int32_t act, float act_param, float* save_mean,
                                             float* save_var, void* workspace, size_t ws_bytes,
                                             void* stream) {
    Geom g;
    const iabn_status st = check_forward(d, g, x, z_out, true, gamma, beta, eps, act, act_param,
                                         save_mean, save_var, workspace, ws_bytes);
    if (st != IABN_OK) return st;
    const FwdArgs a{x, z_out, nullptr, kModeFwd, kLayerStandard, gamma, beta, eps, (int)act,
                    act_param, save_mean, save_var};
    return run_forward(g, a, workspace, static_cast<cudaStream_t>(stream));
}

extern "C" iabn_status iabn_forward_checkpoint(const iabn_desc* d, void* x_inout, void* z_out,
                                               const float* gamma, const float* beta, float eps,
                                               int32_t act, float act_param, float* save_mean,
                                               float* save_var, void* workspace,
                                               size_t ws_bytes, void* stream) {
    Geom g;
    const iabn_status st = check_forward(d, g, x_inout, z_out, true, gamma, beta, eps, act,
                                         act_param, save_mean, save_var, workspace, ws_bytes);
    if (st != IABN_OK) return st;
    const FwdArgs a{x_inout, x_inout, z_out, kModeFwdCkpt, kLayerCkpt, gamma, beta, eps,
                    (int)act, act_param, save_mean, save_var};
    return run_forward(g, a, workspace, static_cast<cudaStream_t>(stream));
}

extern "C" iabn_status iabn_backward(const iabn_desc* d, const void* z, void* dz_inout,
                                     const float* gamma, const float* beta,
                                     const float* save_var, float eps, int32_t act,
                                     float act_param, float* dgamma, float* dbeta,
                                     void* workspace, size_t ws_bytes, void* stream) {
    Geom g;
    const iabn_status st = check_backward(d, g, z, dz_inout, gamma, beta, save_var, eps, act,
                                          act_param, dgamma, dbeta, workspace, ws_bytes);
    if (st != IABN_OK) return st;
    const BwdArgs a{z, dz_inout, kModeBwdZ, kLayerInPlace, gamma, beta, nullptr, save_var, eps,
                    (int)act, act_param, dgamma, dbeta};
    return run_backward(g, a, workspace, static_cast<cudaStream_t>(stream));
}

extern "C" iabn_status iabn_backward_standard(const iabn_desc* d, const void* x, void* dz_inout,
                                              const float* gamma, const float* beta,
                                              const float* save_mean, const float* save_var,
                                              float eps, int32_t act, float act_param,
                                              float* dgamma, float* dbeta, void* workspace,
                                              size_t ws_bytes, void* stream) {
    Geom g;
    const iabn_status st = check_backward(d, g, x, dz_inout, gamma, beta, save_var, eps, act,
                                          act_param, dgamma, dbeta, workspace, ws_bytes, true,
                                          save_mean);
    if (st != IABN_OK) return st;
    const BwdArgs a{x, dz_inout, kModeBwdX, kLayerStandard, gamma, beta, save_mean, save_var,
                    eps, (int)act, act_param, dgamma, dbeta};
    return run_backward(g, a, workspace, static_cast<cudaStream_t>(stream));
}

extern "C" iabn_status iabn_backward_checkpoint(const iabn_desc* d, const void* xhat,
                                                void* dz_inout, const float* gamma,
                                                const float* beta, const float* save_var,
                                                float eps, int32_t act, float act_param,
                                                float* dgamma, float* dbeta, void* workspace,
                                                size_t ws_bytes, void* stream) {
    Geom g;
    const iabn_status st = check_backward(d, g, xhat, dz_inout, gamma, beta, save_var, eps, act,
                                          act_param, dgamma, dbeta, workspace, ws_bytes);
    if (st != IABN_OK) return st;
    const BwdArgs a{xhat, dz_inout, kModeBwdXhat, kLayerCkpt, gamma, beta, nullptr, save_var,
                    eps, (int)act, act_param, dgamma, dbeta};
    return run_backward(g, a, workspace, static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------ INPLACE-ABNsync
// (the shard of one call may hold a single value per channel: M >= 1)

static bool aligned8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }

extern "C" iabn_status iabn_sync_forward_stats(const iabn_desc* d, const void* x, double* stats,
                                               void* workspace, size_t ws_bytes,
                                               void* stream) {
    Geom g;
    const iabn_status st = make_geom(d, g, 1);
    if (st != IABN_OK) return st;
    if (!x || !stats || !aligned8(stats)) return IABN_ERR_INVALID_ARG;
    if (!aligned16(x)) return IABN_ERR_MISALIGNED;
    if (!workspace || ws_bytes < workspace_bytes(g) || !aligned16(workspace))
        return IABN_ERR_WORKSPACE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return from_cuda(cudaErrorNoDevice);
    return from_cuda(sync_forward_stats(g, x, stats, carve(workspace, g),
                                        static_cast<cudaStream_t>(stream), device_sms(dev)));
}

extern "C" iabn_status iabn_sync_forward_apply(const iabn_desc* d, void* x_inout,
                                               const double* gathered, int32_t world,
                                               const float* gamma, const float* beta, float eps,
                                               int32_t act, float act_param, float* save_mean,
                                               float* save_var, void* workspace,
                                               size_t ws_bytes, void* stream) {
    if (!gathered || !aligned8(gathered) || world < 1) return IABN_ERR_INVALID_ARG;
    Geom g;
    const iabn_status st = check_forward(d, g, x_inout, nullptr, false, gamma, beta, eps, act,
                                         act_param, save_mean, save_var, workspace, ws_bytes, 1);
    if (st != IABN_OK) return st;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return from_cuda(cudaErrorNoDevice);
    const FwdArgs a{x_inout, x_inout, nullptr, kModeFwd, kLayerInPlace, gamma, beta, eps,
                    (int)act, act_param, save_mean, save_var};
    return from_cuda(sync_forward_apply(g, a, gathered, (int)world, carve(workspace, g),
                                        static_cast<cudaStream_t>(stream), device_sms(dev)));
}

extern "C" iabn_status iabn_sync_backward_stats(const iabn_desc* d, const void* z, const void* dz,
                                                const float* gamma, const float* beta,
                                                int32_t act, float act_param, double* stats,
                                                void* workspace, size_t ws_bytes,
                                                void* stream) {
    Geom g;
    iabn_status st = make_geom(d, g, 1);
    if (st != IABN_OK) return st;
    if (!z || !dz || !gamma || !beta || !stats || !aligned8(stats)) return IABN_ERR_INVALID_ARG;
    if ((st = check_act(act, act_param)) != IABN_OK) return st;
    if (!aligned16(z) || !aligned16(dz)) return IABN_ERR_MISALIGNED;
    if (!workspace || ws_bytes < workspace_bytes(g) || !aligned16(workspace))
        return IABN_ERR_WORKSPACE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return from_cuda(cudaErrorNoDevice);
    const BwdArgs a{z, const_cast<void*>(dz), kModeBwdZ, kLayerInPlace, gamma, beta, nullptr,
                    nullptr, 0.f, (int)act, act_param, nullptr, nullptr};
    return from_cuda(sync_backward_stats(g, a, stats, carve(workspace, g),
                                         static_cast<cudaStream_t>(stream), device_sms(dev)));
}

extern "C" iabn_status iabn_sync_backward_apply(const iabn_desc* d, const void* z, void* dz_inout,
                                                const double* gathered, int32_t world,
                                                const float* gamma, const float* beta,
                                                const float* save_var, float eps, int32_t act,
                                                float act_param, float* dgamma, float* dbeta,
                                                void* workspace, size_t ws_bytes,
                                                void* stream) {
    if (!gathered || !aligned8(gathered) || world < 1) return IABN_ERR_INVALID_ARG;
    Geom g;
    const iabn_status st = check_backward(d, g, z, dz_inout, gamma, beta, save_var, eps, act,
                                          act_param, dgamma, dbeta, workspace, ws_bytes, false,
                                          nullptr, 1);
    if (st != IABN_OK) return st;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return from_cuda(cudaErrorNoDevice);
    const BwdArgs a{z, dz_inout, kModeBwdZ, kLayerInPlace, gamma, beta, nullptr, save_var, eps,
                    (int)act, act_param, dgamma, dbeta};
    return from_cuda(sync_backward_apply(g, a, gathered, (int)world, carve(workspace, g),
                                         static_cast<cudaStream_t>(stream), device_sms(dev)));
}

extern "C" iabn_status iabn_checkpoint_recompute(const iabn_desc* d, const void* xhat,
                                                 void* z_out, const float* gamma,
                                                 const float* beta, int32_t act,
                                                 float act_param, void* stream) {
    Geom g;
    iabn_status st = make_geom(d, g, 1);
    if (st != IABN_OK) return st;
    if (!xhat || !z_out || !gamma || !beta) return IABN_ERR_INVALID_ARG;
    if ((st = check_act(act, act_param)) != IABN_OK) return st;
    if (!aligned16(xhat) || !aligned16(z_out)) return IABN_ERR_MISALIGNED;
    if (xhat != z_out && overlap(g, xhat, z_out)) return IABN_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return from_cuda(cudaErrorNoDevice);
    return from_cuda(recompute_pass(g, xhat, z_out, gamma, beta, (int)act, act_param,
                                    static_cast<cudaStream_t>(stream), device_sms(dev)));
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
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return from_cuda(cudaErrorNoDevice);
    return from_cuda(inference_pass(g, a, static_cast<cudaStream_t>(stream), device_sms(dev)));
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

extern "C" iabn_status iabn_describe_plan(const iabn_desc* d, int32_t call, int32_t sm_count,
                                          int32_t smem_optin, iabn_plan_info* out) {
    Geom g;
    iabn_status st = make_geom(d, g);
    if (st != IABN_OK) return st;
    if (!out || call < IABN_CALL_FORWARD || call > IABN_CALL_BACKWARD_CHECKPOINT)
        return IABN_ERR_INVALID_ARG;
    const int layer = call / 2, direction = call % 2;
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
    if (forced_plan() != kTwoPhase &&
        resident_shape(g, layer, direction, sm_count, smem_optin, r)) {
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
