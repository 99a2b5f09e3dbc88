// iabn_device.cuh -- device-side building blocks shared by the InPlace-ABN
// kernels: storage types, the activation and its inverse, the workspace
// control block, a bounded grid barrier and deterministic warp reductions.
//
// Method: "In-Place Activated BatchNorm for Memory-Optimized Training of
// DNNs" (paperlayer.ai summary), section 3 "INPLACE-ABN" (invertible
// activation and scale-and-shift) and section 4 "Experimental setup"
// (leaky-ReLU slope 0.01).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace iabn {

enum : int { kNCHW = 0, kNHWC = 1 };
enum : int { kF32 = 0, kBF16 = 1, kF16 = 2 };
enum : int { kLeaky = 0, kElu = 1, kIdent = 2 };

// What one call computes.  The in-place layer keeps only z; the standard
// BN+ACT layer keeps x (and z); the optimized-checkpointing layer keeps xhat.
//   kModeFwd       read x, write z (over x for the in-place layer, to its
//                  own buffer for the standard one)
//   kModeFwdCkpt   read x, write xhat over x and z to its own buffer
//   kModeBwdZ      read z and dz, write dx over dz (INPLACE-ABN)
//   kModeBwdX      read x and dz, write dx over dz (standard)
//   kModeBwdXhat   read xhat and dz, write dx over dz (checkpointing)
enum : int { kModeFwd = 0, kModeFwdCkpt = 1, kModeBwdZ = 2, kModeBwdX = 3, kModeBwdXhat = 4 };

// Sticky status bits written by kernels into the workspace control block.
constexpr uint32_t kStTimeout = 1u << 0;
constexpr uint32_t kStSingular = 1u << 1;

// First 256 bytes of every workspace.
struct Control {
    uint32_t status;     // sticky kSt* bits
    uint32_t bar_count;  // grid-barrier arrivals; a multiple of kBarStride between launches
    uint32_t never_set;  // a word no code writes (failure-injection wait target)
    uint32_t pad[61];
};
static_assert(sizeof(Control) == 256, "control block is 256 bytes");

// Largest number of blocks whose per-channel partials a workspace holds (NHWC).
constexpr int kMaxPartialBlocks = 512;

// Largest grid of the resident plan (one CTA per SM).
constexpr int kMaxResidentCtas = 256;

// Optional phase trace (IABN_TRACE=1): %globaltimer stamps, kTraceSlots per
// resident CTA, in the workspace right after the control block.
constexpr int kTraceSlots = 16;
constexpr size_t kTraceBytes = (size_t)kMaxResidentCtas * kTraceSlots * 8;

// Default time budget of one bounded wait (grid barrier, mbarrier): 1 s.
constexpr unsigned long long kWaitBudgetNs = 1000000000ull;

// ------------------------------------------------------------ storage types

template <int DT> struct Storage;
template <> struct Storage<kF32> {
    using T = float;
    static __device__ __forceinline__ float load(const T* p) { return *p; }
    static __device__ __forceinline__ void store(T* p, float v) { *p = v; }
};
template <> struct Storage<kBF16> {
    using T = __nv_bfloat16;
    static __device__ __forceinline__ float load(const T* p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void store(T* p, float v) { *p = __float2bfloat16_rn(v); }
};
template <> struct Storage<kF16> {
    using T = __half;
    static __device__ __forceinline__ float load(const T* p) { return __half2float(*p); }
    static __device__ __forceinline__ void store(T* p, float v) { *p = __float2half_rn(v); }
};

// ---------------------------------------------------------------- activation
// phi and its inverse.  The positive branch is taken iff the argument is > 0,
// so phi'(0) is the negative-branch slope.  For 16-bit storage the ELU uses
// the fast exponential / logarithm intrinsics: their error (a few fp32 ulp)
// is far below one storage ulp of z, which bounds what the inverse can
// recover anyway.  For fp32 storage the accurate library functions are used.

// ELU inverse floor: 1 + z/alpha is clamped at 2^-24, y = ln(2^-24).
constexpr float kEluFloorU = 5.9604644775390625e-08f;   // 2^-24
constexpr float kEluFloorY = -16.635532333438686f;      // ln(2^-24)

template <int ACT, int DT>
__device__ __forceinline__ float act_forward(float y, float p) {
    if (ACT == kLeaky) return y > 0.f ? y : p * y;
    if (ACT == kElu) {
        if (DT == kF32) return y > 0.f ? y : p * expm1f(y);
        // 16-bit storage: both branches, then a select (no divergence)
        const float e = p * (__expf(fminf(y, 0.f)) - 1.f);
        return y > 0.f ? y : e;
    }
    return y;
}

// From the stored z and the incoming dz: the pre-activation y and dy = dz*phi'(y).
template <int ACT, int DT>
__device__ __forceinline__ void act_backward(float z, float dz, float p, float inv_p,
                                             float& y, float& dy) {
    if (ACT == kLeaky) {
        const bool pos = z > 0.f;
        y = pos ? z : z * inv_p;
        dy = pos ? dz : dz * p;
    } else if (ACT == kElu) {
        if (DT == kF32) {
            if (z > 0.f) {
                y = z;
                dy = dz;
            } else {
                const float t = z * inv_p;
                y = 1.f + t <= kEluFloorU ? kEluFloorY : log1pf(t);
                dy = dz * fmaxf(z + p, 0.f);   // phi'(y) = alpha*e^y = z + alpha
            }
        } else {
            // 16-bit storage: both branches, then selects (no divergence)
            const float u = 1.f + z * inv_p;
            const float yn = u <= kEluFloorU ? kEluFloorY : __logf(fmaxf(u, kEluFloorU));
            const bool pos = z > 0.f;
            y = pos ? z : yn;
            dy = pos ? dz : dz * fmaxf(z + p, 0.f);
        }
    } else {
        y = z;
        dy = dz;
    }
}

// dy = dz * phi'(y) from the pre-activation y itself (the standard and the
// checkpointing layers, which recompute y): 1 on the positive branch, the
// slope a, or alpha*e^y for the ELU (y <= 0 there).
template <int ACT, int DT>
__device__ __forceinline__ float act_dy_from_y(float y, float dz, float p) {
    if (ACT == kLeaky) return y > 0.f ? dz : dz * p;
    if (ACT == kElu) {
        const float e = DT == kF32 ? expf(fminf(y, 0.f)) : __expf(fminf(y, 0.f));
        return y > 0.f ? dz : dz * (p * e);
    }
    return dz;
}

// Per-channel constants with which the standard and the checkpointing
// backward recover, from the stored value a (x or xhat),
//   xhat = a*xs + xb   and   y = a*ys + yb.
// Standard (from x, with the saved mean and variance): rstd =
// 1/sqrt(var + eps) and A = gamma*rstd in fp64, then xs = rstd,
// xb = -mean*rstd, ys = A, yb = beta - mean*A, each rounded once to fp32.
// Checkpointing (from xhat): xs = 1, xb = 0, ys = gamma, yb = beta.  Every
// kernel that recomputes y from a takes these same four floats, so its sign
// (the activation's branch) is decided identically in every pass.
template <int MODE>
__device__ __forceinline__ void src_affine(float g, float b, float mean, float var, float eps,
                                           float& xs, float& xb, float& ys, float& yb) {
    if (MODE == kModeBwdX) {
        const double r = 1.0 / sqrt((double)var + (double)eps);
        const double A = (double)g * r;
        xs = (float)r;
        xb = (float)(-(double)mean * r);
        ys = (float)A;
        yb = (float)((double)b - (double)mean * A);
    } else {
        xs = 1.f;
        xb = 0.f;
        ys = g;
        yb = b;
    }
}

// ------------------------------------------------------------ small helpers

// 16-byte global loads.  asm volatile keeps a batch of these in program
// order, so a batch is in flight before its values are used.
//   ldg_cg: cached in L2 only, normal eviction priority, so a later pass over
//           the same data can still find it there;
//   ldg_cs: streaming (evict-first).
__device__ __forceinline__ uint4 ldg_cg(const void* p) {
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}
__device__ __forceinline__ uint4 ldg_cs(const void* p) {
    uint4 v;
    asm volatile("ld.global.cs.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_gpu(uint32_t* p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t* p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;"
                 : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// Grid-wide barrier for a co-resident (cooperatively launched) grid, with a
// time budget.  The arrival counter only grows: each CTA adds 1 and waits
// until the counter reaches `target`, so the last arrival releases every
// poller directly.  Targets of one launch are base + G, base + 2G, ...; base
// is the counter at launch rounded down to a multiple of kBarStride (a CTA
// that starts late may already see up to G-1 early arrivals, and G <=
// kBarStride), and the launch pads the counter to base + 2*kBarStride before
// it ends (bar_pad), so the next launch again starts on a multiple.  The
// __syncthreads() before the arrival orders the CTA's writes before thread
// 0's release (a cumulative release after a CTA barrier).  *fail (shared
// memory) is the CTA's failure flag: a CTA that has failed still arrives (so
// the counter stays balanced for the next launch) but does not wait; a wait
// that runs out sets *fail and kStTimeout.  Every thread of the CTA must call
// it, and every CTA calls every barrier of the launch.
constexpr uint32_t kBarStride = 256;

__device__ __forceinline__ uint32_t bar_base(const Control* ctl) {
    return ld_acquire_gpu(&ctl->bar_count) & ~(kBarStride - 1u);
}

__device__ __forceinline__ bool grid_barrier(Control* ctl, uint32_t target,
                                             unsigned long long budget_ns, int* fail) {
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t arrived = atom_add_acq_rel_gpu(&ctl->bar_count, 1u) + 1u;
        if (*((volatile int*)fail) == 0 && arrived != target) {
            const unsigned long long t0 = global_ns();
            while ((int32_t)(ld_acquire_gpu(&ctl->bar_count) - target) < 0) {
                if (global_ns() - t0 > budget_ns) {
                    atomicOr(&ctl->status, kStTimeout);
                    *((volatile int*)fail) = 1;
                    break;
                }
            }
        }
    }
    __syncthreads();
    return *((volatile int*)fail) == 0;
}

// Called by one thread of one CTA after the launch's last barrier (nbar
// barriers of G arrivals each, every CTA arriving at each, failed or not):
// brings the counter to base + 2*kBarStride once all arrivals are in.
__device__ __forceinline__ void bar_pad(Control* ctl, uint32_t G, uint32_t nbar) {
    atomicAdd(&ctl->bar_count, 2u * kBarStride - nbar * G);
}

// One channel's running statistics step (momentum m, unbias = M/(M-1)):
//   running_mean <- (1 - m)*running_mean + m*mean,
//   running_var  <- (1 - m)*running_var + m*var*unbias,
// in fp32 from the fp32 batch statistics; the standalone update kernel and
// the forwards that fuse the update share it, so both give the same bits.
__device__ __forceinline__ void running_step(float* rmean, float* rvar, float mean, float var,
                                             float m, float unbias) {
    *rmean = fmaf(m, mean, (1.f - m) * *rmean);
    *rvar = fmaf(m, var * unbias, (1.f - m) * *rvar);
}

// ------------------------------------------------ channel of a flat index

// The channel of element i of a flat grid-stride loop, tracked incrementally
// (NHWC: i mod C; NCHW: (i div HW) mod C) so the loop has no division.
template <int LAYOUT>
struct ChannelWalker {
    int64_t c, rem, sc, sr, sq, C, HW;
    __device__ __forceinline__ void init(int64_t i, int64_t stride, int64_t C_, int64_t HW_) {
        C = C_; HW = HW_;
        if (LAYOUT == kNHWC) {
            c = i % C; sc = stride % C;
        } else {
            rem = i % HW; c = (i / HW) % C; sr = stride % HW; sq = (stride / HW) % C;
        }
    }
    __device__ __forceinline__ void advance() {
        if (LAYOUT == kNHWC) {
            c += sc;
            if (c >= C) c -= C;
        } else {
            rem += sr;
            int64_t carry = 0;
            if (rem >= HW) { rem -= HW; carry = 1; }
            c += sq + carry;
            if (c >= C) c -= C;
        }
    }
};

// Channel of a flat element index, moved without division: by one element
// (step) or by the grid-stride loop's fixed stride (jump).  NHWC: c = i mod C;
// NCHW: rem = i mod HW, c = (i div HW) mod C.
struct ChannelPos {
    int64_t c, rem;
};

template <int LAYOUT>
struct ChannelStride {
    int64_t C, HW, sc, sr, sq;
    __device__ __forceinline__ void setup(int64_t stride, int64_t C_, int64_t HW_) {
        C = C_;
        HW = HW_;
        sc = stride % C;
        sr = stride % HW;
        sq = (stride / HW) % C;
    }
    __device__ __forceinline__ ChannelPos at(int64_t i) const {
        ChannelPos q;
        if (LAYOUT == kNHWC) {
            q.c = i % C;
            q.rem = 0;
        } else {
            q.rem = i % HW;
            q.c = (i / HW) % C;
        }
        return q;
    }
    __device__ __forceinline__ void jump(ChannelPos& q) const {
        if (LAYOUT == kNHWC) {
            q.c += sc;
            if (q.c >= C) q.c -= C;
        } else {
            q.rem += sr;
            int64_t carry = 0;
            if (q.rem >= HW) {
                q.rem -= HW;
                carry = 1;
            }
            q.c += sq + carry;   // < 2C
            if (q.c >= C) q.c -= C;
        }
    }
    __device__ __forceinline__ void step(ChannelPos& q) const {
        if (LAYOUT == kNHWC) {
            if (++q.c == C) q.c = 0;
        } else if (++q.rem == HW) {
            q.rem = 0;
            if (++q.c == C) q.c = 0;
        }
    }
};

// Deterministic warp reductions (fixed shuffle-down tree; lane 0 holds the
// result, which is then broadcast so every lane sees the same bits).
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
    return __shfl_sync(0xffffffffu, v, 0);
}

// The same over each half of the warp (lanes 0-15, 16-31); every lane of the
// warp must call it.
__device__ __forceinline__ double half_warp_sum(double v) {
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o, 16);
    return __shfl_sync(0xffffffffu, v, 0, 16);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
    return __shfl_sync(0xffffffffu, v, 0);
}

// Chan et al. merge of two (count, mean, M2) summaries, in fp32.
__device__ __forceinline__ void chan_merge(float& n, float& mean, float& m2,
                                           float nb, float meanb, float m2b) {
    const float nt = n + nb;
    if (nb == 0.f) return;
    if (n == 0.f) {
        n = nb; mean = meanb; m2 = m2b;
        return;
    }
    const float d = meanb - mean;
    const float f = nb / nt;
    mean = fmaf(d, f, mean);
    m2 = m2 + m2b + d * d * n * f;
    n = nt;
}

}  // namespace iabn
