// iabn_elementwise.cu -- one-launch elementwise passes z = phi(y), y an affine
// function of the stored value per channel:
//   - evaluation mode (iabn_inference): y = gamma (x - running_mean) /
//     sqrt(running_var + eps) + beta, the coefficients computed in the same
//     launch from the running statistics ([BN] Algorithm 2, the inference
//     network);
//   - the checkpointing layer's recompute of z from the stored xhat
//     (iabn_checkpoint_recompute): y = gamma xhat + beta ([ABN] section 3,
//     "Proposed Checkpointing");
//   - the two-phase plan's forward apply, from the coefficients its finalize
//     wrote (and, for the checkpointing forward, xhat as a second output).
//
// The work is a single read of the input and a write of the output(s), so
// the bound is HBM bandwidth.  Two launch shapes:
//   rows  NHWC with rows of C*s bytes a multiple of 16: every thread owns one
//         16-byte column of a block of up to 256 columns (its 16/s channels'
//         coefficients in registers) and walks rows, four rows' loads in
//         flight before any math; blockIdx.y picks the column block.
//   flat  NCHW, and NHWC rows that are not a whole number of 16-byte vectors:
//         16-byte vectors over the flat tensor, four per thread in flight, the
//         channel of each element tracked without division; the coefficients
//         of all channels sit in shared memory when they fit (C <= 4096),
//         else they are formed per element.
// Either grid is one wave of resident blocks.
#include <atomic>

#include "iabn_bulk.cuh"
#include "iabn_device.cuh"
#include "iabn_internal.h"

namespace iabn {

namespace {

// Where a pass takes its per-channel coefficients from.
enum : int {
    kCoefGiven = 0,     // workspace records (mean, gamma*rstd, beta, beta - mean*gamma*rstd)
                        // and, second record, (rstd, ...) for the checkpointing forward
    kCoefRunning = 1,   // gamma, beta, running mean and variance, eps
    kCoefAffine = 2     // gamma, beta: y = gamma*a + beta
};

struct AffArgs {
    const unsigned char* src;   // x, or xhat for the recompute
    unsigned char* dst;         // z; checkpointing forward: xhat
    unsigned char* dst2;        // checkpointing forward: z
    int64_t E, C, HW, R;        // elements, channels, plane size, NHWC rows
    int VC;                     // rows launch: 16-byte vectors per row
    const float4* coef;         // kCoefGiven
    const float* gamma;
    const float* beta;
    const float* rmean;
    const float* rvar;
    float eps, p;
    // rows launch, second pass over x (kCoefGiven): the statistics pass's row
    // segments [b*R/nseg, (b+1)*R/nseg); 0: grid-stride walk
    int nseg;
};

// Coefficients of one channel: y = (a - m)*sc + b (fp32 storage) or
// a*sc + sh (16-bit storage); checkpointing xhat = (a - m)*rs (fp32) or
// a*rs + nmr (16-bit).
struct Coef {
    float m, sc, b, sh, rs, nmr;
};

template <int SRC, bool CKPT>
__device__ __forceinline__ Coef coef_of(const AffArgs& a, int64_t c) {
    Coef k;
    if (SRC == kCoefGiven) {
        const float4 r = a.coef[c];
        k.m = r.x;
        k.sc = r.y;
        k.b = r.z;
        k.sh = r.w;
        k.rs = CKPT ? a.coef[a.C + c].x : 1.f;
    } else if (SRC == kCoefRunning) {
        k.m = __ldg(a.rmean + c);
        k.rs = __frsqrt_rn(__ldg(a.rvar + c) + a.eps);
        k.sc = __ldg(a.gamma + c) * k.rs;
        k.b = __ldg(a.beta + c);
        k.sh = fmaf(-k.m, k.sc, k.b);
    } else {
        k.m = 0.f;
        k.rs = 1.f;
        k.sc = __ldg(a.gamma + c);
        k.b = __ldg(a.beta + c);
        k.sh = k.b;
    }
    k.nmr = -k.m * k.rs;
    return k;
}

template <int DT, int ACT, bool CKPT>
__device__ __forceinline__ void apply_elem(float v, const Coef& k, float p, float& out,
                                           float& out2) {
    const float y = DT == kF32 ? fmaf(v - k.m, k.sc, k.b) : fmaf(v, k.sc, k.sh);
    if (CKPT) {
        out = DT == kF32 ? (v - k.m) * k.rs : fmaf(v, k.rs, k.nmr);
        out2 = act_forward<ACT, DT>(y, p);
    } else {
        out = act_forward<ACT, DT>(y, p);
    }
}

constexpr int kAffThreads = 256;
constexpr int kAffUnroll = 4;

// NHWC rows: thread -> (column, row phase); its column's channels' coefficients
// in registers; kAffUnroll rows' loads in flight.
template <int DT, int ACT, int SRC, bool CKPT, bool REV>
__global__ void __launch_bounds__(kAffThreads) k_aff_rows(const AffArgs a) {
    constexpr int VE = Vec<DT>::N;   // elements per 16-byte vector
    const int W = a.VC < kAffThreads ? a.VC : kAffThreads;
    const int RPB = kAffThreads / W;
    const int t = threadIdx.x;
    const int phase = t / W;
    const int64_t col = (int64_t)blockIdx.y * W + t % W;
    if (phase >= RPB || col >= a.VC) return;
    Coef k[VE];
#pragma unroll
    for (int e = 0; e < VE; ++e) k[e] = coef_of<SRC, CKPT>(a, col * VE + e);
    const uint4* src = reinterpret_cast<const uint4*>(a.src) + col;
    uint4* dst = reinterpret_cast<uint4*>(a.dst) + col;
    uint4* dst2 = CKPT ? reinterpret_cast<uint4*>(a.dst2) + col : nullptr;
    auto one = [&](const uint4& v, int64_t r) {
        float f[VE], o[VE], o2[VE];
        Vec<DT>::unpack(v, f);
#pragma unroll
        for (int e = 0; e < VE; ++e) apply_elem<DT, ACT, CKPT>(f[e], k[e], a.p, o[e], o2[e]);
        __stcs(dst + r * a.VC, Vec<DT>::pack(o));
        if (CKPT) __stcs(dst2 + r * a.VC, Vec<DT>::pack(o2));
    };
    if (REV) {
        // The second pass over x, right after the statistics pass read it
        // segment by segment, front to back: the J blocks of segment b share
        // its rows (row phases j*RPB + phase) and walk them last first, so
        // the rows L2 still holds from that pass come first.
        const int J = (int)gridDim.x / a.nseg;
        const int b = (int)blockIdx.x / J, j = (int)blockIdx.x % J;
        const int64_t s0 = (int64_t)b * a.R / a.nseg, s1 = ((int64_t)b + 1) * a.R / a.nseg;
        const int64_t stride = (int64_t)J * RPB;
        const int64_t first = s0 + (int64_t)j * RPB + phase;
        if (first >= s1) return;
        int64_t r = first + (s1 - 1 - first) / stride * stride;   // this thread's last row
        for (; r - (kAffUnroll - 1) * stride >= first; r -= kAffUnroll * stride) {
            uint4 v[kAffUnroll];
#pragma unroll
            for (int u = 0; u < kAffUnroll; ++u) v[u] = __ldcs(src + (r - u * stride) * a.VC);
#pragma unroll
            for (int u = 0; u < kAffUnroll; ++u) one(v[u], r - u * stride);
        }
        for (; r >= first; r -= stride) one(__ldcs(src + r * a.VC), r);
        return;
    }
    const int64_t rstep = (int64_t)gridDim.x * RPB;
    for (int64_t r0 = (int64_t)blockIdx.x * RPB + phase; r0 < a.R; r0 += rstep * kAffUnroll) {
        uint4 v[kAffUnroll];
#pragma unroll
        for (int u = 0; u < kAffUnroll; ++u) {
            const int64_t r = r0 + u * rstep;
            if (r < a.R) v[u] = __ldcs(src + r * a.VC);
        }
#pragma unroll
        for (int u = 0; u < kAffUnroll; ++u) {
            const int64_t r = r0 + u * rstep;
            if (r >= a.R) continue;
            float f[VE], o[VE], o2[VE];
            Vec<DT>::unpack(v[u], f);
#pragma unroll
            for (int e = 0; e < VE; ++e) apply_elem<DT, ACT, CKPT>(f[e], k[e], a.p, o[e], o2[e]);
            __stcs(dst + r * a.VC, Vec<DT>::pack(o));
            if (CKPT) __stcs(dst2 + r * a.VC, Vec<DT>::pack(o2));
        }
    }
}

// Coefficient table entries in shared memory (flat launch), when they fit.
constexpr int kAffSmemChannels = 4096;

// Flat 16-byte vectors (NCHW, or NHWC rows that are not whole vectors).
template <int DT, int ACT, int LAYOUT, int SRC, bool CKPT>
__global__ void __launch_bounds__(kAffThreads) k_aff_flat(const AffArgs a) {
    constexpr int VE = Vec<DT>::N;
    extern __shared__ __align__(16) unsigned char aff_smem[];
    Coef* table = reinterpret_cast<Coef*>(aff_smem);
    const bool tab = a.C <= kAffSmemChannels;
    if (tab) {
        for (int64_t c = threadIdx.x; c < a.C; c += blockDim.x) table[c] = coef_of<SRC, CKPT>(a, c);
        __syncthreads();
    }
    auto coef = [&](int64_t c) -> Coef { return tab ? table[c] : coef_of<SRC, CKPT>(a, c); };
    const int64_t NV = a.E / VE;
    const int64_t nt = (int64_t)gridDim.x * blockDim.x;
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const uint4* src = reinterpret_cast<const uint4*>(a.src);
    uint4* dst = reinterpret_cast<uint4*>(a.dst);
    uint4* dst2 = reinterpret_cast<uint4*>(a.dst2);
    ChannelStride<LAYOUT> cs;
    cs.setup(kAffUnroll * nt * VE, a.C, a.HW);
    ChannelPos q[kAffUnroll];
#pragma unroll
    for (int u = 0; u < kAffUnroll; ++u) q[u] = cs.at((t + u * nt) * VE);
    for (int64_t v0 = t; v0 < NV; v0 += kAffUnroll * nt) {
        uint4 in[kAffUnroll];
#pragma unroll
        for (int u = 0; u < kAffUnroll; ++u) {
            const int64_t v = v0 + u * nt;
            if (v < NV) in[u] = __ldcs(src + v);
        }
#pragma unroll
        for (int u = 0; u < kAffUnroll; ++u) {
            const int64_t v = v0 + u * nt;
            if (v < NV) {
                float f[VE], o[VE], o2[VE];
                Vec<DT>::unpack(in[u], f);
                ChannelPos qq = q[u];
                Coef k = coef(qq.c);
                int64_t c_prev = qq.c;
#pragma unroll
                for (int e = 0; e < VE; ++e) {
                    if (qq.c != c_prev) {
                        k = coef(qq.c);
                        c_prev = qq.c;
                    }
                    apply_elem<DT, ACT, CKPT>(f[e], k, a.p, o[e], o2[e]);
                    cs.step(qq);
                }
                __stcs(dst + v, Vec<DT>::pack(o));
                if (CKPT) __stcs(dst2 + v, Vec<DT>::pack(o2));
            }
            cs.jump(q[u]);
        }
    }
    // the last E mod VE elements, one per thread of the first block
    using T = typename Storage<DT>::T;
    const int64_t i = NV * VE + t;
    if (i < a.E) {
        const Coef k = coef(cs.at(i).c);
        float o, o2;
        apply_elem<DT, ACT, CKPT>(Storage<DT>::load(reinterpret_cast<const T*>(a.src) + i), k,
                                  a.p, o, o2);
        Storage<DT>::store(reinterpret_cast<T*>(a.dst) + i, o);
        if (CKPT) Storage<DT>::store(reinterpret_cast<T*>(a.dst2) + i, o2);
    }
}

// Resident blocks of `kern` per SM (256 threads, `smem` bytes), queried once.
template <typename Kern>
int blocks_per_sm(Kern kern, size_t smem, std::atomic<int>& cache) {
    int nb = cache.load(std::memory_order_relaxed);
    if (nb > 0) return nb;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, kAffThreads, smem) !=
            cudaSuccess ||
        nb < 1) {
        cudaGetLastError();
        return 2;
    }
    cache.store(nb, std::memory_order_relaxed);
    return nb;
}

template <int DT, int ACT, int SRC, bool CKPT>
cudaError_t launch_aff(const Geom& g, AffArgs a, int sms, cudaStream_t s) {
    a.E = g.E;
    a.C = g.C;
    a.HW = g.HW;
    a.R = g.R;
    const int64_t rby = g.C * g.esize;
    if (g.layout == kNHWC && rby % 16 == 0 && rby / 16 <= (int64_t)1 << 30) {
        a.VC = (int)(rby / 16);
        // the segment walk only for a second pass over x (kCoefGiven)
        const bool rev = SRC == kCoefGiven && a.nseg > 0;
        auto kern = rev ? k_aff_rows<DT, ACT, SRC, CKPT, SRC == kCoefGiven>
                        : k_aff_rows<DT, ACT, SRC, CKPT, false>;
        static std::atomic<int> occ{0}, occ_rev{0};
        const int W = a.VC < kAffThreads ? a.VC : kAffThreads;
        const int64_t gy = (a.VC + W - 1) / W;
        if (gy > 65535) return cudaErrorNotSupported;
        const int64_t RPB = kAffThreads / W;
        const int64_t want = (int64_t)sms * blocks_per_sm(kern, 0, rev ? occ_rev : occ);
        int64_t gx = (want + gy - 1) / gy;
        const int64_t need = (g.R + RPB - 1) / RPB;
        if (gx > need) gx = need;
        if (gx < 1) gx = 1;
        if (rev) {
            // J blocks per segment, at least one
            int64_t J = gx / a.nseg;
            if (J < 1) J = 1;
            gx = J * a.nseg;
        }
        kern<<<dim3((unsigned)gx, (unsigned)gy), kAffThreads, 0, s>>>(a);
    } else {
        const size_t smem = g.C <= kAffSmemChannels ? (size_t)g.C * sizeof(Coef) : 0;
        const int64_t nv = g.E / Vec<DT>::N;
        int64_t blocks;
        cudaError_t e;
        if (g.layout == kNHWC) {
            auto kern = k_aff_flat<DT, ACT, kNHWC, SRC, CKPT>;
            static std::atomic<int> occ{0};
            if (smem > 48 * 1024 &&
                (e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)smem)) != cudaSuccess)
                return e;
            blocks = (int64_t)sms * blocks_per_sm(kern, smem, occ);
            const int64_t need = (nv + kAffThreads - 1) / kAffThreads;
            if (blocks > need) blocks = need < 1 ? 1 : need;
            kern<<<(unsigned)blocks, kAffThreads, smem, s>>>(a);
        } else {
            auto kern = k_aff_flat<DT, ACT, kNCHW, SRC, CKPT>;
            static std::atomic<int> occ{0};
            if (smem > 48 * 1024 &&
                (e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)smem)) != cudaSuccess)
                return e;
            blocks = (int64_t)sms * blocks_per_sm(kern, smem, occ);
            const int64_t need = (nv + kAffThreads - 1) / kAffThreads;
            if (blocks > need) blocks = need < 1 ? 1 : need;
            kern<<<(unsigned)blocks, kAffThreads, smem, s>>>(a);
        }
    }
    count_launches(1);
    return cudaGetLastError();
}

template <int DT, int SRC, bool CKPT>
cudaError_t launch_aff_act(const Geom& g, const AffArgs& a, int act, int sms, cudaStream_t s) {
    switch (act) {
    case kLeaky: return launch_aff<DT, kLeaky, SRC, CKPT>(g, a, sms, s);
    case kElu: return launch_aff<DT, kElu, SRC, CKPT>(g, a, sms, s);
    default: return launch_aff<DT, kIdent, SRC, CKPT>(g, a, sms, s);
    }
}

template <int SRC, bool CKPT>
cudaError_t launch_aff_dt(const Geom& g, const AffArgs& a, int act, int sms, cudaStream_t s) {
    switch (g.dtype) {
    case kF32: return launch_aff_act<kF32, SRC, CKPT>(g, a, act, sms, s);
    case kBF16: return launch_aff_act<kBF16, SRC, CKPT>(g, a, act, sms, s);
    default: return launch_aff_act<kF16, SRC, CKPT>(g, a, act, sms, s);
    }
}

}  // namespace

cudaError_t inference_pass(const Geom& g, const InfArgs& in, cudaStream_t s, int sms) {
    AffArgs a = {};
    a.src = static_cast<const unsigned char*>(in.x);
    a.dst = static_cast<unsigned char*>(in.x);
    a.gamma = in.gamma;
    a.beta = in.beta;
    a.rmean = in.running_mean;
    a.rvar = in.running_var;
    a.eps = in.eps;
    a.p = in.act_param;
    return launch_aff_dt<kCoefRunning, false>(g, a, in.act, sms, s);
}

cudaError_t recompute_pass(const Geom& g, const void* xhat, void* z, const float* gamma,
                           const float* beta, int act, float act_param, cudaStream_t s,
                           int sms) {
    AffArgs a = {};
    a.src = static_cast<const unsigned char*>(xhat);
    a.dst = static_cast<unsigned char*>(z);
    a.gamma = gamma;
    a.beta = beta;
    a.p = act_param;
    return launch_aff_dt<kCoefAffine, false>(g, a, act, sms, s);
}

cudaError_t forward_apply_pass(const Geom& g, const FwdArgs& f, const float4* coef,
                               cudaStream_t s, int sms, int nseg) {
    AffArgs a = {};
    a.src = static_cast<const unsigned char*>(f.x);
    a.dst = static_cast<unsigned char*>(f.dst);
    a.dst2 = static_cast<unsigned char*>(f.dst2);
    a.coef = coef;
    a.p = f.act_param;
    a.nseg = nseg;
    if (f.mode == kModeFwdCkpt) return launch_aff_dt<kCoefGiven, true>(g, a, f.act, sms, s);
    return launch_aff_dt<kCoefGiven, false>(g, a, f.act, sms, s);
}

}  // namespace iabn
