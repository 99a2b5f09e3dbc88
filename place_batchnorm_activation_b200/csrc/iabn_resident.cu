// iabn_resident.cu -- host side of the resident plan: which shapes qualify,
// how a call is tiled over the SMs and their shared memory, and the launch.
//
// Shapes that qualify:
//   NHWC: a row of C channels is a multiple of 16 bytes and at most 16 KiB
//         (C % 8 == 0 and C <= 8192 for 16-bit storage; C % 4 == 0 and
//         C <= 4096 for fp32).
//   NCHW: with g = 16 / gcd(16, H*W*s) planes per unit every unit starts on a
//         16-byte boundary; N*C must be a multiple of g and one unit must fit
//         in 32 KiB.
// Everything else runs the two-phase plan.
//
// Tuning knobs read from the environment (defaults in brackets):
//   IABN_L2_HINTS [1]       L2 evict-last on tiles phase B reloads, evict-first
//                           on the rest; 0 = no hints.
//   IABN_TILE_KB_FWD, IABN_TILE_KB_BWD [48, 24] KiB per tensor per tile.
//   IABN_RING_FWD, IABN_RING_BWD       [4, 4]   slots cycled by the stream.
//   IABN_BARRIER_BUDGET_NS  [1e9] time budget of each bounded wait.
//   IABN_WAIT_CONS, IABN_WAIT_PROD [0]  mbarrier wait mode of the consumer warps
//                           and of the producer: 0 try_wait, 1 test_wait spin,
//                           2 try_wait with a 32 ns suspend hint.
//   IABN_TRACE    [0]       1: every CTA writes %globaltimer stamps at its phase
//                           boundaries into the workspace (bytes 256 .. 256 +
//                           32 KiB, [CTA][16] u64; see k_resident).
#include <stdlib.h>

#include <mutex>

#include <algorithm>

#include "iabn_resident.cuh"

namespace iabn {

namespace {

struct DeviceLimits {
    int sms = 0;
    int smem_optin = 0;
};

DeviceLimits device_limits() {
    static std::mutex mu;
    static DeviceLimits cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DeviceLimits{};
    std::lock_guard<std::mutex> lock(mu);
    DeviceLimits& d = cache[dev];
    if (d.sms == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
            d.sms = v;
        v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) ==
            cudaSuccess)
            d.smem_optin = v;
    }
    return d;
}

long env_long(const char* name, long dflt) {
    const char* s = getenv(name);
    if (!s || !*s) return dflt;
    char* end = nullptr;
    const long v = strtol(s, &end, 10);
    return (end && *end == 0) ? v : dflt;
}

int gcd_int(int64_t a, int64_t b) {
    while (b) {
        const int64_t t = a % b;
        a = b;
        b = t;
    }
    return (int)a;
}

int round_up_int(int v, int a) { return (v + a - 1) / a * a; }

int layer_mode(int layer, int dir) {
    if (layer == kLayerStandard) return dir == 0 ? kModeFwd : kModeBwdX;
    if (layer == kLayerCkpt) return dir == 0 ? kModeFwdCkpt : kModeBwdXhat;
    return dir == 0 ? kModeFwd : kModeBwdZ;
}

// Fills P for call mode `mode`; false if the shape does not qualify or the
// device cannot hold the tiles.
bool make_plan(const Geom& g, int mode, const DeviceLimits& dl, ResPlan& P, int& cpt) {
    if (dl.sms <= 0 || dl.smem_optin <= 0) return false;
    const int dir = mode_dir(mode);
    // coefficient records per channel in phase B
    const int nrec = mode == kModeBwdX || mode == kModeBwdXhat ? 2 : 1;
    const int s = g.esize;
    const int NT = dir == 0 ? 1 : 2;
    const int target =
        (int)env_long(dir == 0 ? "IABN_TILE_KB_FWD" : "IABN_TILE_KB_BWD", dir == 0 ? 48 : 24) * 1024;
    if (target < 1024 || target > 65536) return false;
    P = ResPlan{};
    cpt = 1;
    int scratch = 0;   // bytes of shared memory the per-CTA merge needs
    if (g.layout == kNHWC) {
        const int64_t rby = g.C * s;
        if (rby % 16 != 0 || rby > 16 * 4 * kConsumers) return false;
        P.VC = (int)(rby / 16);
        cpt = P.VC <= kConsumers ? 1 : (P.VC <= 2 * kConsumers ? 2 : 4);
        // the standard backward and the checkpointing calls run with one
        // 16-byte column per thread
        if (cpt > 1 && mode != kModeFwd && mode != kModeBwdZ) return false;
        P.RP = cpt == 1 ? kConsumers / P.VC : 1;
        P.unit_bytes = (int)rby;
        P.units = g.R;
        int tr = target / (int)rby;
        if (tr < 1) tr = 1;
        if (P.RP > 1) tr = tr < P.RP ? P.RP : tr / P.RP * P.RP;
        P.tile_units = tr;
        P.g = 1;
        P.L = 1;
        // merge: RP-1 row phases x VC columns x per channel pair, forward two
        // double2 (mean, M2), backward one float4 (sum dy, sum dy*y)
        if (cpt == 1 && P.RP > 1) scratch = (P.RP - 1) * P.VC * (8 / s) * (dir == 0 ? 32 : 16);
        // TMEM stash: 1 KB (64 vectors) per consumer thread; TMEM accesses are
        // warp-wide, so every warp must hold a single row phase
        if (env_long("IABN_TMEM_STASH", 1) != 0) {
            if (P.RP * P.VC == kConsumers * cpt && env_long("IABN_STASH_CP", 1) != 0) {
                P.stash = 64 / (cpt * NT);   // copy engine: 8 columns per 4 KB piece
                P.stash_cp = 1;
            } else if (cpt > 1 || P.VC % 32 == 0) {
                P.stash = 64 / (cpt * NT);
            }
        }
    } else {
        const int64_t pb = g.HW * s;
        const int gq = 16 / gcd_int(pb, 16);
        if ((g.N * g.C) % gq != 0) return false;
        if (gq * pb > 32768) return false;
        if (g.HW > (1 << 30)) return false;
        P.unit_bytes = (int)(gq * pb);
        P.units = g.N * g.C / gq;
        int tu = target / P.unit_bytes;
        if (tu < 1) tu = 1;
        P.g = gq;
        // lanes per plane: one for small planes (no shuffles), else enough for
        // ~8 elements each
        int L = 1;
        if (g.HW > 64)
            while (L < 32 && L * 8 < g.HW) L *= 2;
        if (dir == 0) {
            // the forward's 480 consumer threads: more lanes while a tile holds
            // fewer planes than they take at once (nc / L), so none is idle,
            // and a tile of whole rounds of nc / L planes where the target
            // size holds one
            const int nc = res_consumers(kNCHW, 0);
            while (L < 32 && nc / L > (int64_t)tu * gq) L *= 2;
            const int gp = nc / L;
            const int m = gp / gcd_int(gp, gq);
            if (tu >= m) tu = tu / m * m;
        }
        P.tile_units = tu;
        P.L = L;
        P.VC = 1;
        P.RP = 1;
    }
    P.tile_bytes = P.tile_units * P.unit_bytes;
    P.half_bytes = round_up_int(P.tile_bytes, 128);
    P.slot_bytes = P.half_bytes * NT;
    int ring = (int)env_long(dir == 0 ? "IABN_RING_FWD" : "IABN_RING_BWD", 4);
    if (ring < 2) ring = 2;
    if (g.layout == kNCHW) {
        // phase B coefficients of the CTA's channel window, if they fit next to
        // the ring: min(C, planes of the largest CTA range) records of nrec
        // float4s
        const int64_t G0 = g.N * g.C / P.g < dl.sms ? g.N * g.C / P.g : dl.sms;
        const int64_t planes = (P.units + G0 - 1) / G0 * P.g;
        const int64_t w = planes < g.C ? planes : g.C;
        const int64_t bytes = round_up_int((int)std::min<int64_t>(w * 16 * nrec, 1 << 20), 128);
        if (env_long("IABN_NCHW_SMEM_COEF", 1) != 0 &&
            1024 + kBarBytes + bytes + (int64_t)ring * P.slot_bytes <= dl.smem_optin) {
            P.ncoef = (int)w;
            scratch = (int)bytes;
        }
    }
    P.scratch_bytes = round_up_int(scratch, 128);
    const int budget = dl.smem_optin - 1024 - kBarBytes - P.scratch_bytes;
    int nslots = budget / P.slot_bytes;
    if (nslots > kMaxSlots) nslots = kMaxSlots;
    if (ring > nslots) return false;
    if (P.stash > 0) nslots = ring;   // the stash replaces resident tiles
    P.stash_first = P.stash_cp ? 1 : (int)env_long("IABN_STASH_FIRST", 1);
    P.nslots = nslots;
    P.ring = ring;
    P.smem_bytes = kBarBytes + P.scratch_bytes + nslots * P.slot_bytes;
    P.G = (int)(P.units < dl.sms ? P.units : dl.sms);
    if (P.G > kMaxResidentCtas) P.G = kMaxResidentCtas;
    // the kernel counts a CTA's units in 32 bits
    if ((P.units + P.G - 1) / P.G >= ((int64_t)1 << 31)) return false;
    P.hints = env_long("IABN_L2_HINTS", 1) != 0 ? 1 : 0;
    return true;
}

cudaError_t launch(const Geom& g, const ResArgs& a, int cpt, int act, int mode, int smem_optin,
                   cudaStream_t s) {
    const bool fwd = mode == kModeFwd || mode == kModeFwdCkpt;
    switch (g.dtype) {
    case kF32:
        return fwd ? launch_resident_f32_fwd(a, g.layout, cpt, act, mode, smem_optin, s)
                   : launch_resident_f32_bwd(a, g.layout, cpt, act, mode, smem_optin, s);
    case kBF16:
        return fwd ? launch_resident_bf16_fwd(a, g.layout, cpt, act, mode, smem_optin, s)
                   : launch_resident_bf16_bwd(a, g.layout, cpt, act, mode, smem_optin, s);
    default:
        return fwd ? launch_resident_f16_fwd(a, g.layout, cpt, act, mode, smem_optin, s)
                   : launch_resident_f16_bwd(a, g.layout, cpt, act, mode, smem_optin, s);
    }
}

ResArgs base_args(const Geom& g, const Workspace& w) {
    ResArgs a;
    a.N = g.N;
    a.C = g.C;
    a.HW = g.HW;
    a.M = (double)g.M;
    a.ctl = w.ctl;
    a.part = w.part;
    a.coef = w.coef;
    a.trace = env_long("IABN_TRACE", 0) != 0 ? w.trace : nullptr;
    const long b = env_long("IABN_BARRIER_BUDGET_NS", (long)kWaitBudgetNs);
    a.budget_ns = b > 0 ? (unsigned long long)b : kWaitBudgetNs;
    a.wait_cons = (int)env_long("IABN_WAIT_CONS", 0);
    a.wait_prod = (int)env_long("IABN_WAIT_PROD", 0);
    a.stall_cta = (int)env_long("IABN_TEST_STALL_CTA", -1);
    return a;
}

}  // namespace

bool resident_supported(const Geom& g, int layer) {
    const DeviceLimits dl = device_limits();
    ResPlan P;
    int cpt;
    return make_plan(g, layer_mode(layer, 0), dl, P, cpt) &&
           make_plan(g, layer_mode(layer, 1), dl, P, cpt);
}

bool resident_shape(const Geom& g, int layer, int dir, int sms, int smem_optin,
                    ResidentShape& out) {
    DeviceLimits dl;
    dl.sms = sms;
    dl.smem_optin = smem_optin;
    ResPlan P, Q;
    int cpt, cpt_other;
    if (!make_plan(g, layer_mode(layer, dir), dl, P, cpt) ||
        !make_plan(g, layer_mode(layer, 1 - dir), dl, Q, cpt_other))
        return false;
    const bool nhwc = g.layout == kNHWC;
    out.grid = P.G;
    out.threads = res_threads(g.layout, mode_dir(layer_mode(layer, dir)));
    out.smem_bytes = P.smem_bytes;
    out.tile_bytes = P.tile_bytes;
    out.slots = P.nslots;
    out.ring = P.ring;
    out.vectors_per_row = nhwc ? P.VC : 0;
    out.cols_per_thread = nhwc ? cpt : 0;
    out.row_phases = nhwc ? P.RP : 0;
    out.planes_per_unit = nhwc ? 0 : P.g;
    out.stash_rows = P.stash;
    out.stash_copy_engine = P.stash_cp;
    return true;
}

cudaError_t forward_resident(const Geom& g, const FwdArgs& f, const Workspace& w,
                             cudaStream_t s) {
    const DeviceLimits dl = device_limits();
    ResArgs a = base_args(g, w);
    int cpt;
    if (!make_plan(g, f.mode, dl, a.P, cpt)) return cudaErrorNotSupported;
    a.src0 = static_cast<const unsigned char*>(f.x);
    a.src1 = nullptr;
    a.dst = static_cast<unsigned char*>(f.dst);
    a.dst2 = static_cast<unsigned char*>(f.dst2);
    a.gamma = f.gamma;
    a.beta = f.beta;
    a.mean_in = nullptr;
    a.var_in = nullptr;
    a.out0 = f.save_mean;
    a.out1 = f.save_var;
    a.rmean = f.running_mean;
    a.rvar = f.running_var;
    a.momentum = f.momentum;
    a.unbias = (float)(g.M / (double)(g.M - 1));
    a.eps = f.eps;
    a.p = f.act_param;
    a.inv_p = f.act == kIdent ? 1.f : 1.f / f.act_param;
    return launch(g, a, cpt, f.act, f.mode, dl.smem_optin, s);
}

cudaError_t backward_resident(const Geom& g, const BwdArgs& b, const Workspace& w,
                              cudaStream_t s) {
    const DeviceLimits dl = device_limits();
    ResArgs a = base_args(g, w);
    int cpt;
    if (!make_plan(g, b.mode, dl, a.P, cpt)) return cudaErrorNotSupported;
    a.src0 = static_cast<const unsigned char*>(b.src);
    a.src1 = static_cast<const unsigned char*>(b.dz);
    a.dst = static_cast<unsigned char*>(b.dz);
    a.dst2 = nullptr;
    a.gamma = b.gamma;
    a.beta = b.beta;
    a.mean_in = b.save_mean;
    a.var_in = b.save_var;
    a.out0 = b.dgamma;
    a.out1 = b.dbeta;
    a.rmean = a.rvar = nullptr;
    a.momentum = a.unbias = 0.f;
    a.eps = b.eps;
    a.p = b.act_param;
    a.inv_p = b.act == kIdent ? 1.f : 1.f / b.act_param;
    return launch(g, a, cpt, b.act, b.mode, dl.smem_optin, s);
}

}  // namespace iabn
