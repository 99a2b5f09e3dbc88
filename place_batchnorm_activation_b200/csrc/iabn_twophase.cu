// iabn_twophase.cu -- the split ("two-phase") plan of the InPlace-ABN layer:
// separate launches for the per-block statistics, the per-channel finalize
// and the elementwise apply.  It handles every shape, layout and alignment
// and needs no co-resident grid; the resident plan (iabn_resident.cu) is the
// fast path for the shapes it supports.
//
// Method: "In-Place Activated BatchNorm for Memory-Optimized Training of
// DNNs" (paperlayer.ai summary), section 3: "Batch Normalization Review"
// (per-channel batch mean and variance, gamma/beta), "INPLACE-ABN" (store
// only z; invert the activation and the scale-and-shift in the backward),
// "INPLACE-ABN II" (gradients in terms of y).
//
// Determinism: every reduction runs in a fixed order (fixed partition of the
// rows/planes, fixed trees), so results are bitwise reproducible.
#include <atomic>

#include "iabn_bulk.cuh"
#include "iabn_device.cuh"
#include "iabn_internal.h"

namespace iabn {

// Threads of the NHWC reductions: one column of W <= 256 channels per thread,
// kTpRowThreads / W row phases, so several rows are read at once.
constexpr int kTpRowThreads = 512;

// Loads issued together by every thread of the reductions before the
// values are used (the accumulation order stays row by row).
constexpr int kTpBatch = 8;

// Row blocks of the NHWC reductions over single channels (rows that are not
// whole 16-byte vectors).
static inline int nhwc_row_blocks(int64_t R) {
    return (int)(R < 256 ? R : 256);
}

// ---------------------------------------------------------------- forward

// Running Welford update of (n, mean, M2) with one value.
__device__ __forceinline__ void welford_add(float v, float& n, float& mean, float& m2) {
    n += 1.f;
    const float d = v - mean;
    mean += d / n;
    m2 = fmaf(d, v - mean, m2);
}

// NHWC: block (rb, cb) owns rows [rb*R/RB, (rb+1)*R/RB) and columns
// [cb*W, cb*W + W).  Thread t reads column t % W of rows phase, phase + RP,
// ... (coalesced along the channel dimension; kTpBatch rows loaded at once)
// with a running Welford update, then the RP row phases of each column merge
// in a fixed tree.
template <int DT>
__global__ void __launch_bounds__(kTpRowThreads, 2)
k_tp_stats_nhwc(const typename Storage<DT>::T* __restrict__ x, int64_t R, int64_t C, int RB,
                double2* __restrict__ part) {
    const int W = C < 256 ? (int)C : 256;
    const int RP = kTpRowThreads / W;
    const int t = threadIdx.x;
    const int lc = t % W, phase = t / W;
    const int64_t col = (int64_t)blockIdx.y * W + lc;
    const int64_t rb = blockIdx.x;
    const int64_t r0 = rb * R / RB, r1 = (rb + 1) * R / RB;
    float n = 0.f, mean = 0.f, m2 = 0.f;
    if (phase < RP && col < C) {
        const typename Storage<DT>::T* src = x + col;
        int64_t r = r0 + phase;
        for (; r + (kTpBatch - 1) * (int64_t)RP < r1; r += kTpBatch * (int64_t)RP) {
            float v[kTpBatch];
#pragma unroll
            for (int k = 0; k < kTpBatch; ++k)
                v[k] = Storage<DT>::load(src + (r + (int64_t)k * RP) * C);
#pragma unroll
            for (int k = 0; k < kTpBatch; ++k) welford_add(v[k], n, mean, m2);
        }
        for (; r < r1; r += RP) welford_add(Storage<DT>::load(src + r * C), n, mean, m2);
    }
    __shared__ float sn[kTpRowThreads], sm[kTpRowThreads], sq[kTpRowThreads];
    sn[t] = n; sm[t] = mean; sq[t] = m2;
    __syncthreads();
    for (int s = 1; s < RP; s <<= 1) {
        const bool act = phase < RP && (phase % (2 * s)) == 0 && phase + s < RP;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, b0 = 0.f, b1 = 0.f, b2 = 0.f;
        if (act) {
            a0 = sn[t]; a1 = sm[t]; a2 = sq[t];
            const int o = t + s * W;
            b0 = sn[o]; b1 = sm[o]; b2 = sq[o];
            chan_merge(a0, a1, a2, b0, b1, b2);
        }
        __syncthreads();
        if (act) { sn[t] = a0; sm[t] = a1; sq[t] = a2; }
        __syncthreads();
    }
    if (phase == 0 && col < C) part[rb * C + col] = make_double2(sm[t], sq[t]);
}

// NCHW: one warp per (n, c) plane of HW contiguous values; lanes run Welford
// over a strided share and merge in a fixed shuffle tree.  Partial slot of
// plane (n, c) is n*C + c.
template <int DT>
__global__ void __launch_bounds__(256)
k_tp_stats_nchw(const typename Storage<DT>::T* __restrict__ x, int64_t planes, int64_t HW,
                double2* __restrict__ part) {
    const int lane = threadIdx.x & 31;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t pl = gw; pl < planes; pl += nw) {
        const typename Storage<DT>::T* src = x + pl * HW;
        float n = 0.f, mean = 0.f, m2 = 0.f;
        int64_t i = lane;
        for (; i + 32 * (kTpBatch - 1) < HW; i += 32 * kTpBatch) {
            float v[kTpBatch];
#pragma unroll
            for (int k = 0; k < kTpBatch; ++k) v[k] = Storage<DT>::load(src + i + 32 * k);
#pragma unroll
            for (int k = 0; k < kTpBatch; ++k) welford_add(v[k], n, mean, m2);
        }
        // the rest of the plane: up to kTpBatch - 1 values per lane, all loaded first
        float v[kTpBatch - 1];
#pragma unroll
        for (int k = 0; k < kTpBatch - 1; ++k)
            v[k] = i + 32 * k < HW ? Storage<DT>::load(src + i + 32 * k) : 0.f;
#pragma unroll
        for (int k = 0; k < kTpBatch - 1; ++k)
            if (i + 32 * k < HW) welford_add(v[k], n, mean, m2);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float b0 = __shfl_down_sync(0xffffffffu, n, o);
            const float b1 = __shfl_down_sync(0xffffffffu, mean, o);
            const float b2 = __shfl_down_sync(0xffffffffu, m2, o);
            if (lane + o < 32) chan_merge(n, mean, m2, b0, b1, b2);
        }
        if (lane == 0) part[pl] = make_double2(mean, m2);
    }
}

// Count of values behind partial k of a channel.
__device__ __forceinline__ double partial_count(int layout, int64_t k, int64_t R, int RB,
                                                int64_t HW) {
    if (layout == kNHWC) return (double)((k + 1) * R / RB - k * R / RB);
    return (double)HW;
}

// The batch statistics of channel c and the forward's apply coefficients:
// record 0 (mean, scale, beta, beta - mean*scale), record 1 (rstd, for the
// checkpointing forward's xhat).
// Optionally (rmean != null) the running statistics' step.
struct RunUpd {
    float* rmean;
    float* rvar;
    float momentum, unbias;
};

__device__ __forceinline__ void fwd_coef_write(int64_t c, int64_t C, double mean, double var,
                                               const float* __restrict__ gamma,
                                               const float* __restrict__ beta, float eps,
                                               float* __restrict__ save_mean,
                                               float* __restrict__ save_var,
                                               float4* __restrict__ coef, const RunUpd& ru) {
    save_mean[c] = (float)mean;
    save_var[c] = (float)var;
    if (ru.rmean != nullptr)
        running_step(ru.rmean + c, ru.rvar + c, (float)mean, (float)var, ru.momentum, ru.unbias);
    const double rstd = 1.0 / sqrt(var + (double)eps);
    const double sc = (double)gamma[c] * rstd;
    coef[c] = make_float4((float)mean, (float)sc, beta[c], (float)((double)beta[c] - mean * sc));
    coef[C + c] = make_float4((float)rstd, 0.f, 0.f, 0.f);
}

// One warp per channel: combine the K partial summaries (count_k, mean_k,
// M2_k) in fp64 in one pass around r, the first partial's mean:
//   s1 = sum count_k (mean_k - r),  s2 = sum M2_k + count_k (mean_k - r)^2,
//   mean = r + s1/M,  M2 = s2 - s1^2/M,
// then write the batch statistics and the apply coefficients.
__global__ void __launch_bounds__(256)
k_tp_finalize_fwd(const double2* __restrict__ part, int layout, int64_t C, int64_t K,
                  int64_t R, int RB, int64_t HW, double M,
                  const float* __restrict__ gamma, const float* __restrict__ beta, float eps,
                  float* __restrict__ save_mean, float* __restrict__ save_var,
                  float4* __restrict__ coef, const RunUpd ru) {
    const int lane = threadIdx.x & 31;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t c = gw; c < C; c += nw) {
        const double r = part[c].x;
        double s1 = 0.0, s2 = 0.0;
#pragma unroll 4
        for (int64_t k = lane; k < K; k += 32) {
            const double2 pk = part[k * C + c];
            const double d = pk.x - r;
            const double w = partial_count(layout, k, R, RB, HW) * d;
            s1 += w;
            s2 += pk.y + w * d;
        }
        s1 = warp_sum(s1);
        s2 = warp_sum(s2);
        const double mean = r + s1 / M;
        const double var = fmax((s2 - s1 * (s1 / M)) / M, 0.0);
        if (lane == 0)
            fwd_coef_write(c, C, mean, var, gamma, beta, eps, save_mean, save_var, coef, ru);
    }
}

// --------------------------------------------------------------- backward

// Per-channel inputs of the backward reductions.
struct BwdIn {
    const float* gamma;
    const float* beta;
    const float* mean;   // standard backward
    const float* var;    // standard backward
    float eps, p, inv_p;
};

// One channel's view of an element (a, dz) of the backward: dy and xhat.
//   in-place (from z):       y = phi^-1(z), dy from z, xhat = (y - beta)/gamma
//   standard / checkpointing: xhat = a*xs + xb, y = a*ys + yb, dy from y
template <int MODE, int ACT, int DT>
struct ElemBwd {
    float ig, nb, xs, xb, ys, yb, p, inv_p;
    __device__ __forceinline__ void setup(const BwdIn& in, int64_t c) {
        p = in.p;
        inv_p = in.inv_p;
        if (MODE == kModeBwdZ) {
            ig = 1.f / in.gamma[c];
            nb = -in.beta[c] * ig;
        } else {
            src_affine<MODE>(in.gamma[c], in.beta[c], MODE == kModeBwdX ? in.mean[c] : 0.f,
                             MODE == kModeBwdX ? in.var[c] : 1.f, in.eps, xs, xb, ys, yb);
        }
    }
    __device__ __forceinline__ void eval(float a, float dz, float& xh, float& dy) const {
        if (MODE == kModeBwdZ) {
            float y;
            act_backward<ACT, DT>(a, dz, p, inv_p, y, dy);
            xh = fmaf(y, ig, nb);
        } else {
            xh = MODE == kModeBwdX ? fmaf(a, xs, xb) : a;
            dy = act_dy_from_y<ACT, DT>(fmaf(a, ys, yb), dz, p);
        }
    }
};

// Per-channel sums S1 = sum dy and S2 = sum dy*xhat, with xhat recovered from
// the stored value (ElemBwd).  Same partition and merge order as the
// statistics.
template <int DT, int ACT, int MODE>
__global__ void __launch_bounds__(kTpRowThreads, 2)
k_tp_reduce_nhwc(const typename Storage<DT>::T* __restrict__ z,
                 const typename Storage<DT>::T* __restrict__ dz, int64_t R, int64_t C, int RB,
                 const BwdIn in, double2* __restrict__ part) {
    const int W = C < 256 ? (int)C : 256;
    const int RP = kTpRowThreads / W;
    const int t = threadIdx.x;
    const int lc = t % W, phase = t / W;
    const int64_t col = (int64_t)blockIdx.y * W + lc;
    const int64_t rb = blockIdx.x;
    const int64_t r0 = rb * R / RB, r1 = (rb + 1) * R / RB;
    float s1 = 0.f, s2 = 0.f;
    if (phase < RP && col < C) {
        ElemBwd<MODE, ACT, DT> eb;
        eb.setup(in, col);
        auto add = [&](float zv, float dzv) {
            float xh, dy;
            eb.eval(zv, dzv, xh, dy);
            s1 += dy;
            s2 = fmaf(dy, xh, s2);
        };
        int64_t r = r0 + phase;
        for (; r + (kTpBatch - 1) * (int64_t)RP < r1; r += kTpBatch * (int64_t)RP) {
            float zv[kTpBatch], dzv[kTpBatch];
#pragma unroll
            for (int k = 0; k < kTpBatch; ++k) {
                const int64_t e = (r + (int64_t)k * RP) * C + col;
                zv[k] = Storage<DT>::load(z + e);
                dzv[k] = Storage<DT>::load(dz + e);
            }
#pragma unroll
            for (int k = 0; k < kTpBatch; ++k) add(zv[k], dzv[k]);
        }
        for (; r < r1; r += RP) {
            const int64_t e = r * C + col;
            add(Storage<DT>::load(z + e), Storage<DT>::load(dz + e));
        }
    }
    __shared__ float a[kTpRowThreads], b[kTpRowThreads];
    a[t] = s1; b[t] = s2;
    __syncthreads();
    for (int s = 1; s < RP; s <<= 1) {
        const bool act = phase < RP && (phase % (2 * s)) == 0 && phase + s < RP;
        float u = 0.f, v = 0.f;
        if (act) { u = a[t] + a[t + s * W]; v = b[t] + b[t + s * W]; }
        __syncthreads();
        if (act) { a[t] = u; b[t] = v; }
        __syncthreads();
    }
    if (phase == 0 && col < C) part[rb * C + col] = make_double2(a[t], b[t]);
}

template <int DT, int ACT, int MODE>
__global__ void __launch_bounds__(256)
k_tp_reduce_nchw(const typename Storage<DT>::T* __restrict__ z,
                 const typename Storage<DT>::T* __restrict__ dz, int64_t planes, int64_t C,
                 int64_t HW, const BwdIn in, double2* __restrict__ part) {
    const int lane = threadIdx.x & 31;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t pl = gw; pl < planes; pl += nw) {
        ElemBwd<MODE, ACT, DT> eb;
        eb.setup(in, pl % C);
        float s1 = 0.f, s2 = 0.f;
        auto add = [&](float zv, float dzv) {
            float xh, dy;
            eb.eval(zv, dzv, xh, dy);
            s1 += dy;
            s2 = fmaf(dy, xh, s2);
        };
        const typename Storage<DT>::T* zp = z + pl * HW;
        const typename Storage<DT>::T* dzp = dz + pl * HW;
        int64_t i = lane;
        for (; i + 32 * (kTpBatch - 1) < HW; i += 32 * kTpBatch) {
            float zv[kTpBatch], dzv[kTpBatch];
#pragma unroll
            for (int k = 0; k < kTpBatch; ++k) {
                zv[k] = Storage<DT>::load(zp + i + 32 * k);
                dzv[k] = Storage<DT>::load(dzp + i + 32 * k);
            }
#pragma unroll
            for (int k = 0; k < kTpBatch; ++k) add(zv[k], dzv[k]);
        }
        // the rest of the plane: up to kTpBatch - 1 pairs per lane, all loaded first
        float zv[kTpBatch - 1], dzv[kTpBatch - 1];
#pragma unroll
        for (int k = 0; k < kTpBatch - 1; ++k) {
            const bool in = i + 32 * k < HW;
            zv[k] = in ? Storage<DT>::load(zp + i + 32 * k) : 0.f;
            dzv[k] = in ? Storage<DT>::load(dzp + i + 32 * k) : 0.f;
        }
#pragma unroll
        for (int k = 0; k < kTpBatch - 1; ++k)
            if (i + 32 * k < HW) add(zv[k], dzv[k]);
        s1 = warp_sum(s1);
        s2 = warp_sum(s2);
        if (lane == 0) part[pl] = make_double2(s1, s2);
    }
}

// --------------------------------------------- NHWC rows of 16-byte vectors
// When a row of C channels is a whole number of 16-byte vectors (VC of them),
// the NHWC passes give every thread one fixed vector column: its VE = 16/s
// channels' constants stay in registers, every load and store is 16 bytes,
// and kRowBatch rows are loaded before any of them is used.  Block (rb, cb)
// owns rows [rb*R/RB, (rb+1)*R/RB) -- the partition the finalize counts -- and
// the columns [cb*W, cb*W + W); its RPB = threads/W row phases take rows
// phase, phase + RPB, ...  The reductions run one block of kRowThreads per SM
// (the partials are per block) with 16 loads in flight per thread (128 KiB
// per SM); the
// backward apply runs blocks of kApplyThreads, as many as fit, 8 loads in
// flight per thread.

constexpr int kRowThreads = 512;
constexpr int kRowBatch = 8;
constexpr int kStatsBatch = 16;
constexpr int kApplyThreads = 256;

template <int THREADS = kRowThreads>
struct RowTile {
    int W, RPB, phase;
    int64_t col, r0, r1;
    bool active;
    __device__ __forceinline__ RowTile(int VC, int64_t R, int RB) {
        W = VC < THREADS ? VC : THREADS;
        RPB = THREADS / W;
        phase = (int)threadIdx.x / W;
        col = (int64_t)blockIdx.y * W + (int)threadIdx.x % W;
        r0 = (int64_t)blockIdx.x * R / RB;
        r1 = ((int64_t)blockIdx.x + 1) * R / RB;
        active = phase < RPB && col < VC;
    }
    // rows of this thread in [r0, r1)
    __device__ __forceinline__ int64_t count() const {
        const int64_t n = r1 - r0;
        return active && n > phase ? (n - 1 - phase) / RPB + 1 : 0;
    }
};

// Forward statistics: each thread sums x - K and (x - K)^2 in fp32 around its
// own first value K of each channel, turns them into (mean, M2) in fp64, and
// the block's row phases combine around phase 0's mean in phase order; one
// (mean, M2) partial per (row block, channel).
template <int DT, bool KEEP>
__global__ void __launch_bounds__(kRowThreads, 1)
k_tp_stats_rows(const uint4* __restrict__ x, int64_t R, int VC, int RB, int64_t C,
                double2* __restrict__ part) {
    // KEEP: x is read again by the apply pass over these row segments, last
    // rows first; load it with normal L2 priority (else streaming)
    auto ld = [](const uint4* p) { return KEEP ? ldg_cg(p) : ldg_cs(p); };
    constexpr int VE = Vec<DT>::N;
    const RowTile<> rt(VC, R, RB);
    const int64_t n = rt.count();
    float piv[VE], s1[VE], s2[VE];
#pragma unroll
    for (int e = 0; e < VE; ++e) piv[e] = s1[e] = s2[e] = 0.f;
    if (n > 0) {
        const uint4* src = x + rt.col;
        Vec<DT>::unpack(src[(rt.r0 + rt.phase) * VC], piv);
        const int64_t step = rt.RPB;
        int64_t r = rt.r0 + rt.phase;
        auto add = [&](const uint4& v) {
            float f[VE];
            Vec<DT>::unpack(v, f);
#pragma unroll
            for (int e = 0; e < VE; ++e) {
                const float d = f[e] - piv[e];
                s1[e] += d;
                s2[e] = fmaf(d, d, s2[e]);
            }
        };
        for (; r + (kStatsBatch - 1) * step < rt.r1; r += kStatsBatch * step) {
            uint4 v[kStatsBatch];
#pragma unroll
            for (int k = 0; k < kStatsBatch; ++k) v[k] = ld(src + (r + k * step) * VC);
#pragma unroll
            for (int k = 0; k < kStatsBatch; ++k) add(v[k]);
        }
        for (; r < rt.r1; r += step) add(ld(src + r * VC));
    }
    // combine the row phases of each column, one channel of the vector at a
    // time (unrolled: the per-channel registers must not be indexed at run time)
    __shared__ double2 sm[kRowThreads];
    const double inv_n = n > 0 ? 1.0 / (double)n : 0.0;
    const int nrows = (int)(rt.r1 - rt.r0);   // a row block's rows fit in 32 bits
    const int pq = nrows / rt.RPB, pr = nrows - pq * rt.RPB;   // phase p has pq + (p < pr) rows
#pragma unroll
    for (int e = 0; e < VE; ++e) {
        const double a1 = s1[e];
        sm[threadIdx.x] = make_double2(n > 0 ? (double)piv[e] + a1 * inv_n : 0.0,
                                       n > 0 ? (double)s2[e] - a1 * a1 * inv_n : 0.0);
        __syncthreads();
        if (rt.active && rt.phase == 0) {
            const double R0 = sm[threadIdx.x].x;
            double q1 = 0.0, q2 = sm[threadIdx.x].y;
            for (int ph = 1; ph < rt.RPB && ph < nrows; ++ph) {
                const double2 v = sm[threadIdx.x + ph * rt.W];
                const double np = (double)(pq + (ph < pr ? 1 : 0));
                const double d = v.x - R0;
                q1 += np * d;
                q2 += v.y + np * d * d;
            }
            const double inv_rows = 1.0 / (double)nrows;
            part[(int64_t)blockIdx.x * C + rt.col * VE + e] =
                make_double2(R0 + q1 * inv_rows, q2 - q1 * q1 * inv_rows);
        }
        __syncthreads();
    }
}

// Backward sums S1 = sum dy and S2 = sum dy*xhat (ElemBwd), fp32 per thread,
// the row phases added in phase order; one partial per (row block, channel).
template <int DT, int ACT, int MODE>
__global__ void __launch_bounds__(kRowThreads, 1)
k_tp_reduce_rows(const uint4* __restrict__ z, const uint4* __restrict__ dz, int64_t R, int VC,
                 int RB, int64_t C, const BwdIn in, double2* __restrict__ part) {
    constexpr int VE = Vec<DT>::N;
    constexpr int B = kStatsBatch / 2;   // rows per batch (two tensors)
    const RowTile<> rt(VC, R, RB);
    float s1[VE], s2[VE];
#pragma unroll
    for (int e = 0; e < VE; ++e) s1[e] = s2[e] = 0.f;
    if (rt.count() > 0) {
        ElemBwd<MODE, ACT, DT> eb[VE];
#pragma unroll
        for (int e = 0; e < VE; ++e) eb[e].setup(in, rt.col * VE + e);
        const uint4* pz = z + rt.col;
        const uint4* pd = dz + rt.col;
        const int64_t step = rt.RPB;
        auto add = [&](const uint4& vz, const uint4& vd) {
            float fz[VE], fd[VE];
            Vec<DT>::unpack(vz, fz);
            Vec<DT>::unpack(vd, fd);
#pragma unroll
            for (int e = 0; e < VE; ++e) {
                float xh, dy;
                eb[e].eval(fz[e], fd[e], xh, dy);
                s1[e] += dy;
                s2[e] = fmaf(dy, xh, s2[e]);
            }
        };
        int64_t r = rt.r0 + rt.phase;
        for (; r + (B - 1) * step < rt.r1; r += B * step) {
            uint4 vz[B], vd[B];
#pragma unroll
            for (int k = 0; k < B; ++k) {
                vz[k] = ldg_cg(pz + (r + k * step) * VC);
                vd[k] = ldg_cg(pd + (r + k * step) * VC);
            }
#pragma unroll
            for (int k = 0; k < B; ++k) add(vz[k], vd[k]);
        }
        for (; r < rt.r1; r += step) add(ldg_cg(pz + r * VC), ldg_cg(pd + r * VC));
    }
    __shared__ float2 sm[kRowThreads];
#pragma unroll
    for (int e = 0; e < VE; ++e) {
        sm[threadIdx.x] = make_float2(s1[e], s2[e]);
        __syncthreads();
        if (rt.active && rt.phase == 0) {
            float a = 0.f, b = 0.f;
            for (int ph = 0; ph < rt.RPB; ++ph) {
                const float2 v = sm[threadIdx.x + ph * rt.W];
                a += v.x;
                b += v.y;
            }
            part[(int64_t)blockIdx.x * C + rt.col * VE + e] = make_double2(a, b);
        }
        __syncthreads();
    }
}

// ------------------------------------------------ NCHW units of small planes
// For planes of at most kUnitMaxBytes, g = 16/gcd(16, HW*s) whole planes form a
// unit that starts on a 16-byte boundary (U = g*HW*s/16 vectors); each thread
// takes one unit, loads its vectors kRowBatch at a time and accumulates the
// planes one after the other, writing each plane's partial when it ends.
constexpr int kUnitMaxBytes = 1024;

template <int DT>
__global__ void __launch_bounds__(256)
k_tp_stats_units(const uint4* __restrict__ x, int64_t units, int U, int HW,
                 double2* __restrict__ part) {
    constexpr int VE = Vec<DT>::N;
    const int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (u >= units) return;
    const uint4* src = x + u * U;
    const int64_t plane0 = u * (int64_t)U * VE / HW;
    int64_t plane = plane0;
    int rem = HW;
    float piv = 0.f, s1 = 0.f, s2 = 0.f;
    bool first = true;
    const double inv_hw = 1.0 / (double)HW;
    auto add = [&](const uint4& v) {
        float f[VE];
        Vec<DT>::unpack(v, f);
#pragma unroll
        for (int e = 0; e < VE; ++e) {
            if (first) {
                piv = f[e];
                first = false;
            }
            const float d = f[e] - piv;
            s1 += d;
            s2 = fmaf(d, d, s2);
            if (--rem == 0) {
                const double a = s1;
                part[plane] = make_double2((double)piv + a * inv_hw, (double)s2 - a * a * inv_hw);
                ++plane;
                rem = HW;
                s1 = s2 = 0.f;
                first = true;
            }
        }
    };
    int v = 0;
    for (; v + kRowBatch <= U; v += kRowBatch) {
        uint4 b[kRowBatch];
#pragma unroll
        for (int k = 0; k < kRowBatch; ++k) b[k] = __ldcs(src + v + k);
#pragma unroll
        for (int k = 0; k < kRowBatch; ++k) add(b[k]);
    }
    for (; v < U; ++v) add(__ldcs(src + v));
}

template <int DT, int ACT, int MODE>
__global__ void __launch_bounds__(256)
k_tp_reduce_units(const uint4* __restrict__ z, const uint4* __restrict__ dz, int64_t units,
                  int U, int HW, int64_t C, const BwdIn in, double2* __restrict__ part) {
    constexpr int VE = Vec<DT>::N;
    constexpr int B = kRowBatch / 2;
    const int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (u >= units) return;
    const uint4* pz = z + u * U;
    const uint4* pd = dz + u * U;
    int64_t plane = u * (int64_t)U * VE / HW;
    int rem = HW;
    float s1 = 0.f, s2 = 0.f;
    ElemBwd<MODE, ACT, DT> eb;
    eb.setup(in, plane % C);
    auto add = [&](const uint4& vz, const uint4& vd) {
        float fz[VE], fd[VE];
        Vec<DT>::unpack(vz, fz);
        Vec<DT>::unpack(vd, fd);
#pragma unroll
        for (int e = 0; e < VE; ++e) {
            float xh, dy;
            eb.eval(fz[e], fd[e], xh, dy);
            s1 += dy;
            s2 = fmaf(dy, xh, s2);
            if (--rem == 0) {
                part[plane] = make_double2(s1, s2);
                ++plane;
                rem = HW;
                s1 = s2 = 0.f;
                eb.setup(in, plane % C);
            }
        }
    };
    int v = 0;
    for (; v + B <= U; v += B) {
        uint4 bz[B], bd[B];
#pragma unroll
        for (int k = 0; k < B; ++k) {
            bz[k] = pz[v + k];
            bd[k] = pd[v + k];
        }
#pragma unroll
        for (int k = 0; k < B; ++k) add(bz[k], bd[k]);
    }
    for (; v < U; ++v) add(pz[v], pd[v]);
}

// Backward apply: block b of RB walks the rows [b*R/RB, (b+1)*R/RB) from the
// end (the reduction's blocks read their ranges' ends last, so those are the
// likeliest still in L2), the coefficients of the thread's channels in
// registers; dx written over dz.
template <int DT, int ACT, int MODE>
__global__ void __launch_bounds__(kApplyThreads)
k_tp_apply_bwd_rows(const uint4* __restrict__ z, uint4* dz, int64_t R, int VC, int RB, int64_t C,
                    const float4* __restrict__ coef, float p, float inv_p) {
    constexpr int VE = Vec<DT>::N;
    constexpr int B = kRowBatch / 2;
    const RowTile<kApplyThreads> rt(VC, R, RB);
    const int64_t n = rt.count();
    if (n == 0) return;
    float4 k0[VE], k1[VE];
#pragma unroll
    for (int e = 0; e < VE; ++e) {
        const int64_t c = rt.col * VE + e;
        k0[e] = __ldg(coef + c);
        k1[e] = MODE == kModeBwdZ ? k0[e] : __ldg(coef + C + c);
    }
    auto dx_of = [&](const uint4& vz, const uint4& vd) -> uint4 {
        float fz[VE], fd[VE];
        Vec<DT>::unpack(vz, fz);
        Vec<DT>::unpack(vd, fd);
#pragma unroll
        for (int e = 0; e < VE; ++e) {
            if (MODE == kModeBwdZ) {
                float y, dy;
                act_backward<ACT, DT>(fz[e], fd[e], p, inv_p, y, dy);
                fd[e] = fmaf(k0[e].x, dy, fmaf(k0[e].y, y, k0[e].z));
            } else {
                const float dy = act_dy_from_y<ACT, DT>(fmaf(fz[e], k0[e].x, k0[e].y), fd[e], p);
                fd[e] = fmaf(k0[e].z, dy, fmaf(k1[e].x, fz[e], k1[e].y));
            }
        }
        return Vec<DT>::pack(fd);
    };
    const uint4* pz = z + rt.col;
    uint4* pd = dz + rt.col;
    const int64_t step = rt.RPB;
    // this thread's rows, last first: r = rlast, rlast - step, ...
    int64_t r = rt.r0 + rt.phase + (n - 1) * step;
    for (; r - (B - 1) * step >= rt.r0; r -= B * step) {
        uint4 vz[B], vd[B];
#pragma unroll
        for (int k = 0; k < B; ++k) {
            vz[k] = __ldcs(pz + (r - k * step) * VC);
            vd[k] = __ldcs(pd + (r - k * step) * VC);
        }
#pragma unroll
        for (int k = 0; k < B; ++k) __stcs(pd + (r - k * step) * VC, dx_of(vz[k], vd[k]));
    }
    for (; r >= rt.r0; r -= step) __stcs(pd + r * VC, dx_of(__ldcs(pz + r * VC), __ldcs(pd + r * VC)));
}

// Channel c's parameter gradients (dbeta = S1, dgamma = S2) and the
// backward's apply coefficients from the sums over the whole batch of M
// values (see k_tp_finalize_bwd).
template <int MODE>
__device__ __forceinline__ void bwd_coef_write(int64_t c, int64_t C, double s1, double s2,
                                               double M, const BwdIn& in,
                                               float* __restrict__ dgamma,
                                               float* __restrict__ dbeta,
                                               float4* __restrict__ coef,
                                               Control* __restrict__ ctl) {
    const double g = in.gamma[c], b = in.beta[c];
    const double rstd = 1.0 / sqrt((double)in.var[c] + (double)in.eps);
    if (MODE != kModeBwdZ) {
        float xs, xb, ys, yb;
        src_affine<MODE>(in.gamma[c], in.beta[c], MODE == kModeBwdX ? in.mean[c] : 0.f,
                         in.var[c], in.eps, xs, xb, ys, yb);
        const double A = g * rstd, B = -A * s2 / M, Cc = -A * s1 / M;
        dbeta[c] = (float)s1;
        dgamma[c] = (float)s2;
        coef[c] = make_float4(ys, yb, (float)A, 0.f);
        coef[C + c] = make_float4((float)(B * (double)xs), (float)(B * (double)xb + Cc), 0.f, 0.f);
    } else if (!(fabs(g) >= 1.17549435082228750797e-38)) {   // |gamma| < FLT_MIN (or NaN)
        atomicOr(&ctl->status, kStSingular);
        dgamma[c] = __int_as_float(0x7fc00000);
        dbeta[c] = __int_as_float(0x7fc00000);
        coef[c] = make_float4(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000),
                              __int_as_float(0x7fc00000), 0.f);
    } else {
        dbeta[c] = (float)s1;
        dgamma[c] = (float)s2;
        const double A = g * rstd, B = -rstd * s2 / M;
        const double Cc = -g * rstd * s1 / M - B * b;
        coef[c] = make_float4((float)A, (float)B, (float)Cc, 0.f);
    }
}

// One warp per channel: S1 = sum dy and S2 = sum dy*xhat summed in fp64;
// dbeta = S1, dgamma = S2.  The apply coefficients:
//   in-place: dx in terms of y (the "INPLACE-ABN II" form), one record
//     dx = A*dy + B*y + Cc,  A = gamma*rstd,  B = -rstd*S2/M,
//     Cc = -gamma*rstd*S1/M - B*beta;
//   standard / checkpointing: dx = A dy + B xhat + Cc (B = -A S2/M,
//     Cc = -A S1/M) applied to the stored value a, xhat = a*xs + xb:
//     record 0 (ys, yb, A), record 1 (B xs, B xb + Cc).
template <int MODE>
__global__ void __launch_bounds__(256)
k_tp_finalize_bwd(const double2* __restrict__ part, int64_t C, int64_t K, double M,
                  const BwdIn in, float* __restrict__ dgamma, float* __restrict__ dbeta,
                  float4* __restrict__ coef, Control* __restrict__ ctl) {
    const int lane = threadIdx.x & 31;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t c = gw; c < C; c += nw) {
        double s1 = 0.0, s2 = 0.0;
        for (int64_t k = lane; k < K; k += 32) {
            const double2 pk = part[k * C + c];
            s1 += pk.x;
            s2 += pk.y;
        }
        s1 = warp_sum(s1);
        s2 = warp_sum(s2);
        if (lane == 0) bwd_coef_write<MODE>(c, C, s1, s2, M, in, dgamma, dbeta, coef, ctl);
    }
}

// dx of one element (a, dz) of channel c from the finalize's record(s).
template <int MODE, int ACT, int DT>
__device__ __forceinline__ float bwd_apply_elem(float a, float dz, const float4* __restrict__ coef,
                                                int64_t C, int64_t c, float p, float inv_p) {
    const float4 k = __ldg(coef + c);
    if (MODE == kModeBwdZ) {
        float y, dy;
        act_backward<ACT, DT>(a, dz, p, inv_p, y, dy);
        return fmaf(k.x, dy, fmaf(k.y, y, k.z));
    }
    const float4 k2 = __ldg(coef + C + c);
    const float dy = act_dy_from_y<ACT, DT>(fmaf(a, k.x, k.y), dz, p);
    return fmaf(k.z, dy, fmaf(k2.x, a, k2.y));
}

template <int DT, int ACT, int LAYOUT, int MODE>
__global__ void __launch_bounds__(256)
k_tp_apply_bwd(const typename Storage<DT>::T* __restrict__ z, typename Storage<DT>::T* dz,
               int64_t E, int64_t C, int64_t HW, const float4* __restrict__ coef, float p,
               float inv_p) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= E) return;
    ChannelWalker<LAYOUT> w;
    w.init(i, stride, C, HW);
    for (; i < E; i += stride) {
        Storage<DT>::store(dz + i, bwd_apply_elem<MODE, ACT, DT>(Storage<DT>::load(z + i),
                                                                 Storage<DT>::load(dz + i), coef,
                                                                 C, w.c, p, inv_p));
        w.advance();
    }
}

template <int DT, int ACT, int LAYOUT, int MODE>
__global__ void __launch_bounds__(256)
k_tp_apply_bwd_vec(const typename Storage<DT>::T* __restrict__ z,
                   typename Storage<DT>::T* dz, int64_t E, int64_t C, int64_t HW,
                   const float4* __restrict__ coef, float p, float inv_p) {
    constexpr int VE = Vec<DT>::N;
    const int64_t NV = E / VE;
    const int64_t nt = (int64_t)gridDim.x * blockDim.x;
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const uint4* zv = reinterpret_cast<const uint4*>(z);
    uint4* dzv = reinterpret_cast<uint4*>(dz);
    ChannelStride<LAYOUT> cs;
    cs.setup(2 * nt * VE, C, HW);
    auto apply = [&](const uint4& uz, uint4& ud, ChannelPos q) {
        float fz[VE], fd[VE];
        Vec<DT>::unpack(uz, fz);
        Vec<DT>::unpack(ud, fd);
#pragma unroll
        for (int k = 0; k < VE; ++k) {
            fd[k] = bwd_apply_elem<MODE, ACT, DT>(fz[k], fd[k], coef, C, q.c, p, inv_p);
            cs.step(q);
        }
        ud = Vec<DT>::pack(fd);
    };
    ChannelPos q0 = cs.at(t * VE), q1 = cs.at((t + nt) * VE);
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    for (int64_t v = t; v < NV; v += 2 * nt) {
        const bool two = v + nt < NV;
        const uint4 za = __ldg(zv + v);
        uint4 da = dzv[v];
        const uint4 zb = two ? __ldg(zv + v + nt) : zero;
        uint4 db = two ? dzv[v + nt] : zero;
        apply(za, da, q0);
        dzv[v] = da;
        if (two) {
            apply(zb, db, q1);
            dzv[v + nt] = db;
        }
        cs.jump(q0);
        cs.jump(q1);
    }
    const int64_t i = NV * VE + t;
    if (i < E)
        Storage<DT>::store(dz + i, bwd_apply_elem<MODE, ACT, DT>(Storage<DT>::load(z + i),
                                                                 Storage<DT>::load(dz + i), coef,
                                                                 C, cs.at(i).c, p, inv_p));
}

// ------------------------------------------------------------ running stats

__global__ void k_running_update(int64_t C, float unbias, const float* __restrict__ mean,
                                 const float* __restrict__ var, float* __restrict__ rmean,
                                 float* __restrict__ rvar, float m) {
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= C) return;
    running_step(rmean + c, rvar + c, mean[c], var[c], m, unbias);
}

// ------------------------------------------------------------ host launch

static int grid_for(int64_t work, int per_block, int cap) {
    int64_t g = (work + per_block - 1) / per_block;
    if (g < 1) g = 1;
    if (g > cap) g = cap;
    return (int)g;
}

// CTAs of `kern` (`threads` threads, no dynamic shared memory) resident on
// one SM, queried once per kernel; the grid-stride kernels are sized to one
// full wave of them (a second, partial wave would run its whole share alone).
template <typename Kern>
static int ctas_per_sm(Kern kern, int threads, std::atomic<int>& cache) {
    int nb = cache.load(std::memory_order_relaxed);
    if (nb > 0) return nb;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, threads, 0) != cudaSuccess ||
        nb < 1) {
        cudaGetLastError();
        return 4;
    }
    cache.store(nb, std::memory_order_relaxed);
    return nb;
}

// Grid of an elementwise pass: two 16-byte vectors per thread per step.
static int apply_grid(const Geom& g, int sms, int per_sm) {
    const int64_t nv = g.E / (16 / g.esize);
    return grid_for(nv, 2 * 256, sms * per_sm);
}

// NHWC rows that are a whole number of 16-byte vectors take the vector-column
// kernels.
static bool rows_vectorised(const Geom& g) {
    const int64_t rby = g.C * g.esize;
    return g.layout == kNHWC && rby % 16 == 0 && rby / 16 <= (int64_t)kRowThreads * 65535;
}

struct RowGrid {
    int RB, GY, VC;
};

// Whether the forward's apply pass walks the statistics pass's row segments
// last row first.  L2 keeps the most recently read ~80 MB of a streamed
// tensor, so a tensor larger than that is found there only in that order; a
// smaller one is found there whole, and the plain grid-stride walk is faster
// (same-box A/B: ResNet trunk 102.8 MB fwd 71.6 -> 69.6 us, the 51.4 MB
// sweep layer 50.2 -> 48.3 us, but the 6.4 MB layer 31.4 -> 35.4 us).
static bool reverse_segments(const Geom& g) {
    return rows_vectorised(g) && g.E * g.esize > ((int64_t)32 << 20);
}

// NCHW small planes: g whole planes per 16-byte aligned unit (0: not used).
static int unit_planes(const Geom& g) {
    if (g.layout != kNCHW) return 0;
    const int64_t pb = g.HW * g.esize;
    int64_t a = pb, b = 16;
    while (b) {
        const int64_t t = a % b;
        a = b;
        b = t;
    }
    const int64_t gq = 16 / a;
    if ((g.N * g.C) % gq != 0 || gq * pb > kUnitMaxBytes) return 0;
    return (int)gq;
}

// Row blocks: a multiple of the SM count (an uneven second block on some SMs
// would run alone), at most the workspace's partial slots and the rows.
static RowGrid row_grid(const Geom& g, int sms) {
    RowGrid rg;
    rg.VC = (int)(g.C * g.esize / 16);
    const int W = rg.VC < kRowThreads ? rg.VC : kRowThreads;
    rg.GY = (rg.VC + W - 1) / W;
    const int RPB = kRowThreads / W;
    // one block per SM, 16 loads in flight per thread
    int64_t rb = sms > 0 ? (int64_t)sms : 256;
    if (rb > kMaxPartialBlocks) rb = kMaxPartialBlocks;
    // a row block of fewer rows than row phases leaves threads idle
    const int64_t most = (g.R + RPB - 1) / RPB;
    if (rb > most) rb = most < 1 ? 1 : most;
    rg.RB = (int)rb;
    return rg;
}

// Row blocks of the backward apply: about `blocks` blocks in all (one wave),
// none with fewer rows than row phases.
static RowGrid apply_row_grid(const Geom& g, int blocks) {
    RowGrid rg;
    rg.VC = (int)(g.C * g.esize / 16);
    const int W = rg.VC < kApplyThreads ? rg.VC : kApplyThreads;
    rg.GY = (rg.VC + W - 1) / W;
    const int RPB = kApplyThreads / W;
    int64_t rb = blocks / rg.GY;
    const int64_t most = (g.R + RPB - 1) / RPB;
    if (rb > most) rb = most;
    if (rb > 65535) rb = 65535;
    rg.RB = (int)(rb < 1 ? 1 : rb);
    return rg;
}

// The statistics pass of x: per-block (mean, M2) partials in w.part, K per
// channel (block partition RB for the row kernels).
template <int DT>
static cudaError_t fwd_stats_launch(const Geom& g, const void* xv, const Workspace& w,
                                    cudaStream_t s, int sms, int64_t& K, int& RB) {
    using T = typename Storage<DT>::T;
    const T* x = static_cast<const T*>(xv);
    RB = 1;
    if (rows_vectorised(g)) {
        const RowGrid rg = row_grid(g, sms);
        RB = rg.RB;
        if (reverse_segments(g))
            k_tp_stats_rows<DT, true><<<dim3(rg.RB, rg.GY), kRowThreads, 0, s>>>(
                static_cast<const uint4*>(xv), g.R, rg.VC, rg.RB, g.C, w.part);
        else
            k_tp_stats_rows<DT, false><<<dim3(rg.RB, rg.GY), kRowThreads, 0, s>>>(
                static_cast<const uint4*>(xv), g.R, rg.VC, rg.RB, g.C, w.part);
        K = RB;
    } else if (g.layout == kNHWC) {
        RB = nhwc_row_blocks(g.R);
        const int W = g.C < 256 ? (int)g.C : 256;
        dim3 grid(RB, (unsigned)((g.C + W - 1) / W));
        k_tp_stats_nhwc<DT><<<grid, kTpRowThreads, 0, s>>>(x, g.R, g.C, RB, w.part);
        K = RB;
    } else if (const int gq = unit_planes(g)) {
        const int64_t units = g.N * g.C / gq;
        k_tp_stats_units<DT><<<(unsigned)((units + 255) / 256), 256, 0, s>>>(
            static_cast<const uint4*>(xv), units, (int)(gq * g.HW * g.esize / 16), (int)g.HW,
            w.part);
        K = g.N;
    } else {
        const int64_t planes = g.N * g.C;
        static std::atomic<int> occ{0};
        const int per_sm = ctas_per_sm(k_tp_stats_nchw<DT>, 256, occ);
        k_tp_stats_nchw<DT><<<grid_for(planes, 8, sms * per_sm), 256, 0, s>>>(x, planes, g.HW,
                                                                              w.part);
        K = g.N;
    }
    count_launches(1);
    return cudaGetLastError();
}

template <int DT>
static cudaError_t fwd_twophase_dt(const Geom& g, const FwdArgs& a, const Workspace& w,
                                   cudaStream_t s, int sms) {
    int64_t K = 0;
    int RB = 1;
    cudaError_t e = fwd_stats_launch<DT>(g, a.x, w, s, sms, K, RB);
    if (e != cudaSuccess) return e;
    k_tp_finalize_fwd<<<grid_for(g.C, 8, sms * 16), 256, 0, s>>>(
        w.part, g.layout, g.C, K, g.R, RB, g.HW, (double)g.M, a.gamma, a.beta, a.eps,
        a.save_mean, a.save_var, w.coef,
        RunUpd{a.running_mean, a.running_var, a.momentum,
               (float)(g.M / (double)(g.M - 1))});
    count_launches(1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // the elementwise pass with fixed channels per thread (iabn_elementwise.cu);
    // a tensor too large to stay whole in L2 is walked over the statistics
    // pass's row segments, each last row first (see reverse_segments)
    return forward_apply_pass(g, a, w.coef, s, sms, reverse_segments(g) ? RB : 0);
}

cudaError_t forward_twophase(const Geom& g, const FwdArgs& a, const Workspace& w,
                             cudaStream_t s, int sms) {
    switch (g.dtype) {
    case kF32: return fwd_twophase_dt<kF32>(g, a, w, s, sms);
    case kBF16: return fwd_twophase_dt<kBF16>(g, a, w, s, sms);
    default: return fwd_twophase_dt<kF16>(g, a, w, s, sms);
    }
}

// The reduction pass of the backward: per-block (S1, S2) partials in w.part,
// K per channel.
template <int DT, int ACT, int MODE>
static cudaError_t bwd_reduce_launch(const Geom& g, const void* src, const void* dzv,
                                     const BwdIn& in, const Workspace& w, cudaStream_t s,
                                     int sms, int64_t& K) {
    using T = typename Storage<DT>::T;
    const T* z = static_cast<const T*>(src);
    const T* dz = static_cast<const T*>(dzv);
    if (rows_vectorised(g)) {
        const RowGrid rg = row_grid(g, sms);
        k_tp_reduce_rows<DT, ACT, MODE><<<dim3(rg.RB, rg.GY), kRowThreads, 0, s>>>(
            static_cast<const uint4*>(src), static_cast<const uint4*>(dzv), g.R, rg.VC, rg.RB,
            g.C, in, w.part);
        K = rg.RB;
    } else if (g.layout == kNHWC) {
        const int RB = nhwc_row_blocks(g.R);
        const int W = g.C < 256 ? (int)g.C : 256;
        dim3 grid(RB, (unsigned)((g.C + W - 1) / W));
        k_tp_reduce_nhwc<DT, ACT, MODE><<<grid, kTpRowThreads, 0, s>>>(z, dz, g.R, g.C, RB, in,
                                                                       w.part);
        K = RB;
    } else if (const int gq = unit_planes(g)) {
        const int64_t units = g.N * g.C / gq;
        k_tp_reduce_units<DT, ACT, MODE><<<(unsigned)((units + 255) / 256), 256, 0, s>>>(
            static_cast<const uint4*>(src), static_cast<const uint4*>(dzv), units,
            (int)(gq * g.HW * g.esize / 16), (int)g.HW, g.C, in, w.part);
        K = g.N;
    } else {
        const int64_t planes = g.N * g.C;
        static std::atomic<int> occ{0};
        const int per_sm = ctas_per_sm(k_tp_reduce_nchw<DT, ACT, MODE>, 256, occ);
        k_tp_reduce_nchw<DT, ACT, MODE><<<grid_for(planes, 8, sms * per_sm), 256, 0, s>>>(
            z, dz, planes, g.C, g.HW, in, w.part);
        K = g.N;
    }
    count_launches(1);
    return cudaGetLastError();
}

// The backward's elementwise pass: dx over dz from the records in w.coef.
template <int DT, int ACT, int MODE>
static cudaError_t bwd_apply_launch(const Geom& g, const void* src, void* dzv,
                                    const Workspace& w, float p, float inv_p, cudaStream_t s,
                                    int sms) {
    using T = typename Storage<DT>::T;
    const T* z = static_cast<const T*>(src);
    T* dz = static_cast<T*>(dzv);
    if (rows_vectorised(g)) {
        auto kern = k_tp_apply_bwd_rows<DT, ACT, MODE>;
        static std::atomic<int> occ{0};
        const RowGrid ag = apply_row_grid(g, sms * ctas_per_sm(kern, kApplyThreads, occ));
        kern<<<dim3(ag.RB, ag.GY), kApplyThreads, 0, s>>>(
            static_cast<const uint4*>(src), static_cast<uint4*>(dzv), g.R, ag.VC, ag.RB, g.C,
            w.coef, p, inv_p);
    } else if (g.layout == kNHWC) {
        k_tp_apply_bwd<DT, ACT, kNHWC, MODE><<<grid_for(g.E, 256, sms * 8), 256, 0, s>>>(
            z, dz, g.E, g.C, g.HW, w.coef, p, inv_p);
    } else {
        static std::atomic<int> occ{0};
        auto kern = k_tp_apply_bwd_vec<DT, ACT, kNCHW, MODE>;
        kern<<<apply_grid(g, sms, ctas_per_sm(kern, 256, occ)), 256, 0, s>>>(
            z, dz, g.E, g.C, g.HW, w.coef, p, inv_p);
    }
    count_launches(1);
    return cudaGetLastError();
}

template <int DT, int ACT, int MODE>
static cudaError_t bwd_twophase_mode(const Geom& g, const BwdArgs& a, const Workspace& w,
                                     cudaStream_t s, int sms) {
    const float p = a.act_param;
    const float inv_p = ACT == kIdent ? 1.f : 1.f / p;
    const BwdIn in{a.gamma, a.beta, a.save_mean, a.save_var, a.eps, p, inv_p};
    int64_t K = 0;
    cudaError_t e = bwd_reduce_launch<DT, ACT, MODE>(g, a.src, a.dz, in, w, s, sms, K);
    if (e != cudaSuccess) return e;
    k_tp_finalize_bwd<MODE><<<grid_for(g.C, 8, sms * 16), 256, 0, s>>>(
        w.part, g.C, K, (double)g.M, in, a.dgamma, a.dbeta, w.coef, w.ctl);
    count_launches(1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return bwd_apply_launch<DT, ACT, MODE>(g, a.src, a.dz, w, p, inv_p, s, sms);
}

template <int DT, int ACT>
static cudaError_t bwd_twophase_act(const Geom& g, const BwdArgs& a, const Workspace& w,
                                    cudaStream_t s, int sms) {
    switch (a.mode) {
    case kModeBwdX: return bwd_twophase_mode<DT, ACT, kModeBwdX>(g, a, w, s, sms);
    case kModeBwdXhat: return bwd_twophase_mode<DT, ACT, kModeBwdXhat>(g, a, w, s, sms);
    default: return bwd_twophase_mode<DT, ACT, kModeBwdZ>(g, a, w, s, sms);
    }
}

template <int DT>
static cudaError_t bwd_twophase_dt(const Geom& g, const BwdArgs& a, const Workspace& w,
                                   cudaStream_t s, int sms) {
    switch (a.act) {
    case kLeaky: return bwd_twophase_act<DT, kLeaky>(g, a, w, s, sms);
    case kElu: return bwd_twophase_act<DT, kElu>(g, a, w, s, sms);
    default: return bwd_twophase_act<DT, kIdent>(g, a, w, s, sms);
    }
}

cudaError_t backward_twophase(const Geom& g, const BwdArgs& a, const Workspace& w,
                              cudaStream_t s, int sms) {
    switch (g.dtype) {
    case kF32: return bwd_twophase_dt<kF32>(g, a, w, s, sms);
    case kBF16: return bwd_twophase_dt<kBF16>(g, a, w, s, sms);
    default: return bwd_twophase_dt<kF16>(g, a, w, s, sms);
    }
}

// ------------------------------------------------------------ INPLACE-ABNsync
// The layer's statistics over a batch split along N across GPUs: each GPU
// reduces its shard to one record per channel, the caller gathers the
// records of all GPUs, and each GPU combines them in rank order (fp64) and
// applies the result to its shard.  Records are 3 doubles per channel:
// forward (n, mean, M2), backward (n, sum dy, sum dy*xhat).

// This GPU's forward record: the K block partials combined as
// k_tp_finalize_fwd does.
__global__ void __launch_bounds__(256)
k_sync_record_fwd(const double2* __restrict__ part, int layout, int64_t C, int64_t K,
                  int64_t R, int RB, int64_t HW, double M, double* __restrict__ rec) {
    const int lane = threadIdx.x & 31;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t c = gw; c < C; c += nw) {
        const double r = part[c].x;
        double s1 = 0.0, s2 = 0.0;
        for (int64_t k = lane; k < K; k += 32) {
            const double2 pk = part[k * C + c];
            const double d = pk.x - r;
            const double w = partial_count(layout, k, R, RB, HW) * d;
            s1 += w;
            s2 += pk.y + w * d;
        }
        s1 = warp_sum(s1);
        s2 = warp_sum(s2);
        if (lane == 0) {
            rec[c * 3] = M;
            rec[c * 3 + 1] = r + s1 / M;
            rec[c * 3 + 2] = fmax(s2 - s1 * (s1 / M), 0.0);
        }
    }
}

// The whole batch's statistics from the gathered forward records, one pass in
// rank order around rank 0's mean r:
//   Mt = sum n_k,  s1 = sum n_k (mean_k - r),  s2 = sum M2_k + n_k (mean_k - r)^2,
//   mean = r + s1/Mt,  var = (s2 - s1^2/Mt)/Mt;
// then the forward's apply coefficients.
__global__ void __launch_bounds__(256)
k_sync_finalize_fwd(const double* __restrict__ gathered, int world, int64_t C,
                    const float* __restrict__ gamma, const float* __restrict__ beta, float eps,
                    float* __restrict__ save_mean, float* __restrict__ save_var,
                    float4* __restrict__ coef, float* __restrict__ rmean,
                    float* __restrict__ rvar, float momentum) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < C; c += stride) {
        const double r = gathered[c * 3 + 1];
        double n = 0.0, s1 = 0.0, s2 = 0.0;
        for (int k = 0; k < world; ++k) {
            const double* q = gathered + ((int64_t)k * C + c) * 3;
            const double d = q[1] - r;
            n += q[0];
            s1 += q[0] * d;
            s2 += q[2] + q[0] * d * d;
        }
        const double mean = r + s1 / n;
        const double var = fmax((s2 - s1 * (s1 / n)) / n, 0.0);
        // the running statistics' count is the whole batch's
        fwd_coef_write(c, C, mean, var, gamma, beta, eps, save_mean, save_var, coef,
                       RunUpd{rmean, rvar, momentum, (float)(n / (n - 1.0))});
    }
}

// This GPU's backward record: the K block partials summed per channel.
__global__ void __launch_bounds__(256)
k_sync_record_bwd(const double2* __restrict__ part, int64_t C, int64_t K, double M,
                  double* __restrict__ rec) {
    const int lane = threadIdx.x & 31;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t c = gw; c < C; c += nw) {
        double s1 = 0.0, s2 = 0.0;
        for (int64_t k = lane; k < K; k += 32) {
            const double2 pk = part[k * C + c];
            s1 += pk.x;
            s2 += pk.y;
        }
        s1 = warp_sum(s1);
        s2 = warp_sum(s2);
        if (lane == 0) {
            rec[c * 3] = M;
            rec[c * 3 + 1] = s1;
            rec[c * 3 + 2] = s2;
        }
    }
}

// The whole batch's sums from the gathered backward records (rank order),
// then the parameter gradients and the backward's apply coefficients.
template <int MODE>
__global__ void __launch_bounds__(256)
k_sync_finalize_bwd(const double* __restrict__ gathered, int world, int64_t C, const BwdIn in,
                    float* __restrict__ dgamma, float* __restrict__ dbeta,
                    float4* __restrict__ coef, Control* __restrict__ ctl) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < C; c += stride) {
        double n = 0.0, s1 = 0.0, s2 = 0.0;
        for (int k = 0; k < world; ++k) {
            const double* q = gathered + ((int64_t)k * C + c) * 3;
            n += q[0];
            s1 += q[1];
            s2 += q[2];
        }
        bwd_coef_write<MODE>(c, C, s1, s2, n, in, dgamma, dbeta, coef, ctl);
    }
}

template <int DT>
static cudaError_t sync_fwd_stats_dt(const Geom& g, const void* x, double* rec,
                                     const Workspace& w, cudaStream_t s, int sms) {
    int64_t K = 0;
    int RB = 1;
    cudaError_t e = fwd_stats_launch<DT>(g, x, w, s, sms, K, RB);
    if (e != cudaSuccess) return e;
    k_sync_record_fwd<<<grid_for(g.C, 8, sms * 16), 256, 0, s>>>(
        w.part, g.layout, g.C, K, g.R, RB, g.HW, (double)g.M, rec);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t sync_forward_stats(const Geom& g, const void* x, double* rec, const Workspace& w,
                               cudaStream_t s, int sms) {
    switch (g.dtype) {
    case kF32: return sync_fwd_stats_dt<kF32>(g, x, rec, w, s, sms);
    case kBF16: return sync_fwd_stats_dt<kBF16>(g, x, rec, w, s, sms);
    default: return sync_fwd_stats_dt<kF16>(g, x, rec, w, s, sms);
    }
}

cudaError_t sync_forward_apply(const Geom& g, const FwdArgs& a, const double* gathered,
                               int world, const Workspace& w, cudaStream_t s, int sms) {
    k_sync_finalize_fwd<<<(unsigned)((g.C + 255) / 256), 256, 0, s>>>(
        gathered, world, g.C, a.gamma, a.beta, a.eps, a.save_mean, a.save_var, w.coef,
        a.running_mean, a.running_var, a.momentum);
    count_launches(1);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return forward_apply_pass(g, a, w.coef, s, sms,
                              reverse_segments(g) ? row_grid(g, sms).RB : 0);
}

template <int DT, int ACT>
static cudaError_t sync_bwd_act(const Geom& g, const BwdArgs& a, double* rec,
                                const double* gathered, int world, const Workspace& w,
                                cudaStream_t s, int sms) {
    const float p = a.act_param;
    const float inv_p = ACT == kIdent ? 1.f : 1.f / p;
    const BwdIn in{a.gamma, a.beta, nullptr, a.save_var, a.eps, p, inv_p};
    if (rec != nullptr) {
        int64_t K = 0;
        cudaError_t e = bwd_reduce_launch<DT, ACT, kModeBwdZ>(g, a.src, a.dz, in, w, s, sms, K);
        if (e != cudaSuccess) return e;
        k_sync_record_bwd<<<grid_for(g.C, 8, sms * 16), 256, 0, s>>>(w.part, g.C, K,
                                                                      (double)g.M, rec);
        count_launches(1);
        return cudaGetLastError();
    }
    k_sync_finalize_bwd<kModeBwdZ><<<(unsigned)((g.C + 255) / 256), 256, 0, s>>>(
        gathered, world, g.C, in, a.dgamma, a.dbeta, w.coef, w.ctl);
    count_launches(1);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return bwd_apply_launch<DT, ACT, kModeBwdZ>(g, a.src, a.dz, w, p, inv_p, s, sms);
}

template <int DT>
static cudaError_t sync_bwd_dt(const Geom& g, const BwdArgs& a, double* rec,
                               const double* gathered, int world, const Workspace& w,
                               cudaStream_t s, int sms) {
    switch (a.act) {
    case kLeaky: return sync_bwd_act<DT, kLeaky>(g, a, rec, gathered, world, w, s, sms);
    case kElu: return sync_bwd_act<DT, kElu>(g, a, rec, gathered, world, w, s, sms);
    default: return sync_bwd_act<DT, kIdent>(g, a, rec, gathered, world, w, s, sms);
    }
}

static cudaError_t sync_bwd(const Geom& g, const BwdArgs& a, double* rec,
                            const double* gathered, int world, const Workspace& w,
                            cudaStream_t s, int sms) {
    switch (g.dtype) {
    case kF32: return sync_bwd_dt<kF32>(g, a, rec, gathered, world, w, s, sms);
    case kBF16: return sync_bwd_dt<kBF16>(g, a, rec, gathered, world, w, s, sms);
    default: return sync_bwd_dt<kF16>(g, a, rec, gathered, world, w, s, sms);
    }
}

cudaError_t sync_backward_stats(const Geom& g, const BwdArgs& a, double* rec,
                                const Workspace& w, cudaStream_t s, int sms) {
    return sync_bwd(g, a, rec, nullptr, 0, w, s, sms);
}

cudaError_t sync_backward_apply(const Geom& g, const BwdArgs& a, const double* gathered,
                                int world, const Workspace& w, cudaStream_t s, int sms) {
    return sync_bwd(g, a, nullptr, gathered, world, w, s, sms);
}

cudaError_t running_update(int64_t C, int64_t count, const float* mean, const float* var,
                           float* rmean, float* rvar, float momentum, cudaStream_t s) {
    const float unbias = (float)((double)count / (double)(count - 1));
    k_running_update<<<(unsigned)((C + 255) / 256), 256, 0, s>>>(C, unbias, mean, var, rmean,
                                                                  rvar, momentum);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace iabn
