// iabn_resident.cuh -- the resident plan of the InPlace-ABN layer: one
// cooperative, persistent kernel per call (forward or backward), one CTA per
// SM, warp-specialised.
//
// Each CTA owns a contiguous range of "units" (NHWC: rows of C channels;
// NCHW: groups of g whole planes, g chosen so every unit starts on a 16-byte
// boundary) and streams it through shared-memory slots with the bulk-copy
// engine.  One producer warp issues every bulk load; eight consumer warps
// compute and store (fifteen in the NCHW forward); one copier warp moves
// stashed rows from the landed slots into Tensor Memory (see the TMEM stash
// below; the NCHW forward, which stashes nothing, has none).  Slots are
// handed over with mbarriers (full: data
// landed; empty: consumers done with a phase A tile; done: consumers done
// with a phase B tile, so the slot may be refilled), so no consumer waits on
// a CTA-wide barrier per tile.
//
//   phase A  tiles 0..n-1: per-thread partial statistics from shared memory.
//            Forward NHWC: sums of x - K and (x - K)^2 in fp32 around the
//            thread's own first value K of each channel, turned into (mean,
//            M2) in fp64; NCHW: exact per-plane two-pass mean and M2.
//            Backward: sum dy and sum dy*y (the "INPLACE-ABN II" form; for
//            leaky-ReLU dy*y = dz*z).
//            The last D tiles land in dedicated slots and stay resident; as
//            soon as a streamed slot frees, the producer prefetches phase B.
//   merge    NHWC: the threads of a column combine their summaries in
//            row-phase order (forward: fp64 (mean, M2) around the first
//            phase's mean); one partial per (CTA, channel).  NCHW: one partial
//            per plane.
//   barrier  grid-wide (bounded wait), a distributed fp64 finalize (one warp
//            per channel, fixed order), a second grid barrier.
//   phase B  tiles n-1..0: resident tiles first, then the streamed ones -- the
//            most recently read first: the last one of each ring slot is still
//            in the slot, the others are read back from L2 -- and then the rows
//            kept in Tensor Memory.  The consumers write their results
//            straight to global memory with 128-bit stores; the producer
//            refills each freed ring slot.
//
// Method: "In-Place Activated BatchNorm for Memory-Optimized Training of
// DNNs" (paperlayer.ai summary), section 3: "Batch Normalization Review",
// "INPLACE-ABN", "INPLACE-ABN II".  The kernel never traps: every wait is
// bounded and a timeout sets kStTimeout in the workspace status word.
#pragma once

#include <climits>

#include "iabn_bulk.cuh"
#include "iabn_device.cuh"
#include "iabn_tmem.cuh"
#include "iabn_internal.h"

namespace iabn {

constexpr int kConsumers = 256;                  // NHWC consumer threads (8 warps)
constexpr int kConsumerWarps = kConsumers / 32;
constexpr int kResThreads = kConsumers + 64;     // + one producer warp + one copier warp
// The NCHW forward keeps nothing in Tensor Memory, so it has no copier warp,
// and its plane loops fit in 128 registers a thread without spilling: 15
// consumer warps and the producer, four warps on each scheduler (each
// scheduler owns a quarter of the register file).  (The NCHW backward keeps
// the 8 + 2 layout: at 128 registers its phase B ran slower.)
constexpr int kConsumersNchwFwd = 480;
__host__ __device__ constexpr int mode_dir(int mode) {
    return mode == kModeFwd || mode == kModeFwdCkpt ? 0 : 1;
}
__host__ __device__ constexpr int res_consumers(int layout, int dir) {
    return layout == kNCHW && dir == 0 ? kConsumersNchwFwd : kConsumers;
}
__host__ __device__ constexpr int res_threads(int layout, int dir) {
    return layout == kNCHW && dir == 0 ? kConsumersNchwFwd + 32 : kResThreads;
}
constexpr int kMaxSlots = 32;
constexpr int kBarBytes = 4 * kMaxSlots * 8;     // full[], empty[], done[], cpdone[] mbarriers

struct ResPlan {
    int G;               // CTAs (at most one per SM)
    int64_t units;       // NHWC: rows; NCHW: groups of g planes
    int unit_bytes;      // bytes of one unit of one tensor (multiple of 16)
    int tile_units;      // units per tile
    int tile_bytes;      // tile_units * unit_bytes
    int half_bytes;      // tile_bytes rounded up to 128: offset of the second tensor
    int slot_bytes;      // half_bytes * tensors per tile
    int nslots;          // slots in shared memory
    int ring;            // slots cycled by the stream; the rest hold resident tiles
    int scratch_bytes;   // shared memory for the per-CTA merge (NHWC) or the phase B
                         // coefficients (NCHW), multiple of 128
    int smem_bytes;      // dynamic shared memory of the launch
    int VC, RP;          // NHWC: 16-byte columns per row; row phases (threads per column)
    int g, L;            // NCHW: planes per unit; lanes per plane
    int hints;           // 1: L2 eviction-priority hints on the bulk copies
    int stash_first;     // 1: the stash holds each thread's first rows, 0: its last
    int stash_cp;        // 1: the copy engine (tcgen05.cp) fills the stash from the
                         // landed slots (CPT 1, RP*VC = 256, first rows); 0: the
                         // consumers store their registers
    int ncoef;           // NCHW: channels of the CTA's coefficient window kept in shared
                         // memory (scratch) for phase B; 0: read from global memory
    int stash;           // NHWC: rows per consumer thread kept in TMEM from phase A
                         // to phase B (0: off); all slots then form the ring
};

struct ResArgs {
    ResPlan P;
    int64_t N, C, HW;
    double M;
    const unsigned char* src0;   // forward: x;  backward: z, x or xhat (by mode)
    const unsigned char* src1;   // backward: dz
    unsigned char* dst;          // forward: z (over x, or its own buffer), checkpointing
                                 // forward: xhat (over x); backward: dx (over dz)
    unsigned char* dst2;         // checkpointing forward: z
    const float* gamma;
    const float* beta;
    const float* mean_in;        // standard backward: saved mean
    const float* var_in;         // backward: saved biased variance
    float* out0;                 // forward: save_mean;  backward: dgamma
    float* out1;                 // forward: save_var;   backward: dbeta
    float* rmean;                // forward: running statistics to update, or null
    float* rvar;
    float momentum, unbias;      // running update: momentum, M/(M-1)
    float eps, p, inv_p;
    Control* ctl;
    double2* part;
    float4* coef;
    unsigned long long* trace;   // null, or [G][kTraceSlots] phase stamps
    unsigned long long budget_ns;
    int wait_cons;               // mbarrier wait mode of the consumers (see mbar_wait)
    int wait_prod;               // mbarrier wait mode of the producer
    int stall_cta;               // failure injection (tests): this CTA waits, for twice
                                 // the budget, on a word nothing sets before barrier 1;
                                 // -1: none
};

// Sum over aligned groups of L lanes (L a power of two); every lane of the
// warp must call it.  Fixed tree, then broadcast from the group's first lane.
__device__ __forceinline__ float group_sum(float v, int L) {
    for (int o = L >> 1; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o, L);
    return __shfl_sync(0xffffffffu, v, 0, L);
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// 16 bytes <-> float2 pairs of consecutive elements.
template <int DT> struct Pairs;
template <> struct Pairs<kF32> {
    static constexpr int NP = 2;
    static __device__ __forceinline__ void unpack(const uint4& v, float2* f) {
        f[0] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
        f[1] = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
    }
    static __device__ __forceinline__ uint4 pack(const float2* f) {
        return make_uint4(__float_as_uint(f[0].x), __float_as_uint(f[0].y),
                          __float_as_uint(f[1].x), __float_as_uint(f[1].y));
    }
};
template <> struct Pairs<kBF16> {
    static constexpr int NP = 4;
    static __device__ __forceinline__ float2 u(uint32_t w) {
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
    static __device__ __forceinline__ uint32_t p(float2 f) {
        __nv_bfloat162 h = __floats2bfloat162_rn(f.x, f.y);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    static __device__ __forceinline__ void unpack(const uint4& v, float2* f) {
        f[0] = u(v.x); f[1] = u(v.y); f[2] = u(v.z); f[3] = u(v.w);
    }
    static __device__ __forceinline__ uint4 pack(const float2* f) {
        return make_uint4(p(f[0]), p(f[1]), p(f[2]), p(f[3]));
    }
};
template <> struct Pairs<kF16> {
    static constexpr int NP = 4;
    static __device__ __forceinline__ float2 u(uint32_t w) {
        return __half22float2(*reinterpret_cast<__half2*>(&w));
    }
    static __device__ __forceinline__ uint32_t p(float2 f) {
        __half2 h = __floats2half2_rn(f.x, f.y);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    static __device__ __forceinline__ void unpack(const uint4& v, float2* f) {
        f[0] = u(v.x); f[1] = u(v.y); f[2] = u(v.z); f[3] = u(v.w);
    }
    static __device__ __forceinline__ uint4 pack(const float2* f) {
        return make_uint4(p(f[0]), p(f[1]), p(f[2]), p(f[3]));
    }
};

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

// Up to two coefficient records of one channel (phase B, NCHW).
struct Rec2 {
    float4 a, b;
};

// 16 bytes <-> the 16/s consecutive elements they hold, as floats.
template <int DT>
__device__ __forceinline__ void unpack_all(const uint4& v, float* x) {
    float2 f[Pairs<DT>::NP];
    Pairs<DT>::unpack(v, f);
#pragma unroll
    for (int q = 0; q < Pairs<DT>::NP; ++q) {
        x[2 * q] = f[q].x;
        x[2 * q + 1] = f[q].y;
    }
}

template <int DT>
__device__ __forceinline__ uint4 pack_all(const float* x) {
    float2 f[Pairs<DT>::NP];
#pragma unroll
    for (int q = 0; q < Pairs<DT>::NP; ++q) f[q] = make_float2(x[2 * q], x[2 * q + 1]);
    return Pairs<DT>::pack(f);
}

// Forward activation on a pair (leaky with slope <= 1 is max(y, a*y), with
// slope > 1 it is min(y, a*y)).
template <int ACT, int DT>
__device__ __forceinline__ float2 act_forward2(float2 y, float p, bool slope_le1) {
    if (ACT == kLeaky) {
        const float2 t = __fmul2_rn(y, f2(p, p));
        return slope_le1 ? f2(fmaxf(y.x, t.x), fmaxf(y.y, t.y))
                         : f2(fminf(y.x, t.x), fminf(y.y, t.y));
    }
    if (ACT == kElu) {
        if (DT == kF32) return f2(act_forward<kElu, DT>(y.x, p), act_forward<kElu, DT>(y.y, p));
        // 16-bit storage: e = p*(exp(min(y, 0)) - 1) is exactly 0 for y >= 0
        // (the exponential of +0 is exactly 1), so max(y, 0) + e is act_forward's
        // select, on pairs and without a comparison
        const float2 e = __fmul2_rn(f2(p, p), __fadd2_rn(f2(__expf(fminf(y.x, 0.f)),
                                                            __expf(fminf(y.y, 0.f))),
                                                         f2(-1.f, -1.f)));
        return __fadd2_rn(f2(fmaxf(y.x, 0.f), fmaxf(y.y, 0.f)), e);
    }
    return y;
}

template <int DT, int ACT, int LAYOUT, int CPT, int MODE>
__global__ void __launch_bounds__(res_threads(LAYOUT, mode_dir(MODE)), 1)
    k_resident(const ResArgs a) {
    constexpr int DIR = mode_dir(MODE);
    constexpr int NC = res_consumers(LAYOUT, DIR);   // consumer threads
    constexpr int CW = NC / 32;                      // consumer warps
    // checkpointing forward: a second output (z) besides xhat
    constexpr bool CKPT = MODE == kModeFwdCkpt;
    // backward from a stored x or xhat: y is recomputed by a scale and shift
    constexpr bool SRCV = MODE == kModeBwdX || MODE == kModeBwdXhat;
    // coefficient records per channel for phase B
    constexpr int NREC = SRCV ? 2 : 1;
    constexpr int NT = DIR == 0 ? 1 : 2;       // tensors per tile
    constexpr int NP = Pairs<DT>::NP;          // channel pairs per 16-byte vector
    constexpr int NQ = CPT * NP;               // channel pairs per thread (NHWC)
    // rows per batch in the tile loops
    constexpr int RB = 4 / CPT > 0 ? 4 / CPT : 1;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxSlots;
    uint64_t* done = empty + kMaxSlots;
    uint64_t* cpdone = done + kMaxSlots;   // TMEM copies out of a slot have finished
    __shared__ int s_fail;
    // gamma, beta (and, backward, the saved variance and, standard backward,
    // the saved mean) of the first channel each consumer half-warp finalizes,
    // fetched while phase A streams
    __shared__ float s_par[CW][2][4];

    const ResPlan& P = a.P;
    unsigned char* scratch = smem + kBarBytes;
    unsigned char* slots = scratch + P.scratch_bytes;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const bool consumer = warp < CW;
    const bool producer = warp == CW;
    const bool copier = warp == CW + 1;
    const int b = blockIdx.x;
    const int G = P.G;
    // Phase trace: 0 start, 1 phase A done, 2 merged, 3 barrier 1, 4 finalize,
    // 5 barrier 2, 6 in-CTA merge rounds done, 7 last refill issued, 8 consumer
    // warp 0 done, 14 the SM's id
    // (%globaltimer ns); 9/10/13 phase A and 11/12/15 phase B SM cycles of
    // consumer warp 0: waiting for tiles / bookkeeping / the row loops.
    auto stamp = [&](int k, bool who) {
        if (a.trace != nullptr && who) a.trace[(size_t)b * kTraceSlots + k] = global_ns();
    };
    stamp(0, tid == 0);
    if (a.trace != nullptr && tid == 0) {
        uint32_t smid;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
        a.trace[(size_t)b * kTraceSlots + 14] = smid;
    }
    // Consumer warp 0 also accounts its SM cycles: waiting for tiles vs the
    // rest of the loop, per phase (trace slots 9..12).
    const bool acct = a.trace != nullptr && tid == 0;
    long long cyc_wait = 0, cyc_work = 0, cyc_comp = 0, cyc_mark = 0;
    auto acct_start = [&]() { if (acct) cyc_mark = clock64(); };
    auto acct_wait = [&]() {
        if (acct) { const long long c = clock64(); cyc_wait += c - cyc_mark; cyc_mark = c; }
    };
    auto acct_work = [&]() {
        if (acct) { const long long c = clock64(); cyc_work += c - cyc_mark; cyc_mark = c; }
    };
    auto acct_comp = [&]() {
        if (acct) { const long long c = clock64(); cyc_comp += c - cyc_mark; cyc_mark = c; }
    };
    auto acct_flush = [&](int k) {
        if (acct) {
            a.trace[(size_t)b * kTraceSlots + k] = (unsigned long long)cyc_wait;
            a.trace[(size_t)b * kTraceSlots + k + 1] = (unsigned long long)cyc_work;
            a.trace[(size_t)b * kTraceSlots + k + 4] = (unsigned long long)cyc_comp;
            cyc_wait = cyc_work = cyc_comp = 0;
        }
    };

    // CTA b owns units [u0, u1): uq each, one more for the last ur CTAs (the
    // first CTAs also finalize the first channels, so they get the short ranges)
    const int64_t uq = P.units / G;
    const int ur = (int)(P.units - uq * G);
    const int64_t u0 = (int64_t)b * uq + max(0, b - (G - ur));
    const int64_t u1 = u0 + uq + (b >= G - ur ? 1 : 0);
    const int n = (int)((u1 - u0 + P.tile_units - 1) / P.tile_units);
    const int ring = P.ring;
    const int D = min(P.nslots - ring, n);
    const int nring = n - D;
    // TMEM stash (NHWC): every consumer thread keeps Jc of its rows in TMEM --
    // its first Jc (the CTA's first S = RP*Jc rows, the ones most likely gone
    // from L2 by phase B) or its last Jc (the CTA's last S rows).  Phase B
    // streams only the tiles [tlo, thi) that hold other rows, the j-th one
    // being tile thi-1-j.
    const bool stash = LAYOUT == kNHWC && P.stash > 0;
    const bool sfirst = stash && P.stash_first != 0;
    // copy-engine stash: tcgen05.cp moves each 4 KB piece of a stashed row
    // group (RP rows holding RP*VC = 256*CPT 16-byte chunks; per tensor) from
    // its landed slot into 8 TMEM columns, chunk L -> lane L (columns 0-3) and
    // chunk L+128 -> lane L (columns 4-7): exactly what consumer thread L,
    // resp. L+128, owns (its column k of the piece k).
    const bool scp = sfirst && P.stash_cp != 0;
    const int tpg = P.tile_units / P.RP;   // row groups per tile (NHWC)
    const int64_t nrows = u1 - u0;
    const int Jc = stash ? (int)min((int64_t)P.stash, nrows / P.RP) : 0;
    const int64_t S = (int64_t)P.RP * Jc;
    int tlo = 0, thi = nring;
    if (stash) {
        if (sfirst) {
            tlo = S >= nrows ? n : (int)(S / P.tile_units);
            thi = n;
        } else {
            thi = (int)((nrows - S + P.tile_units - 1) / P.tile_units);
        }
    }
    const int nB = thi - tlo;
    __shared__ uint32_t s_tmem;

    if (tid == 0) {
        for (int s = 0; s < P.nslots; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], CW);
            mbar_init(&done[s], CW);
            mbar_init(&cpdone[s], 1);
        }
        mbar_init_fence();
        s_fail = 0;
    }
    // grid-barrier counter base of this launch (thread 0 only; see grid_barrier)
    const uint32_t bbase = tid == 0 ? bar_base(a.ctl) : 0u;
    if (consumer && (lane & 15) == 0) {
        const int h = lane >> 4;
        const int64_t c = ((int64_t)warp * G + b) * 2 + h;
        if (c < a.C) {
            cp_async4(&s_par[warp][h][0], a.gamma + c);
            cp_async4(&s_par[warp][h][1], a.beta + c);
            if (DIR == 1) cp_async4(&s_par[warp][h][2], a.var_in + c);
            if (MODE == kModeBwdX) cp_async4(&s_par[warp][h][3], a.mean_in + c);
        }
    }
    if (stash && warp == 0) {
        __syncwarp();
        tmem_alloc_all(&s_tmem);
        tmem_fence_before_sync();
    }
    __syncthreads();
    if (stash) tmem_fence_after_sync();
    const uint32_t tmem_base = stash ? s_tmem : 0u;

    auto t_u0 = [&](int t) -> int64_t { return u0 + (int64_t)t * P.tile_units; };
    auto t_nu = [&](int t) -> int {
        const int64_t r = u1 - t_u0(t);
        return (int)(r < P.tile_units ? r : P.tile_units);
    };
    auto slotA = [&](int t) -> int { return t < nring ? t % ring : ring + (t - nring); };
    // Phase B streams tile t through ring slot t % ring too, so the last
    // phase-A tile of each ring slot is still there when phase B wants it.
    auto ring_resident = [&](int t) -> bool { return t < nring && t >= nring - ring; };
    auto slot_ptr = [&](int s) -> unsigned char* { return slots + (size_t)s * P.slot_bytes; };
    auto failed = [&]() -> bool { return *((volatile int*)&s_fail) != 0; };
    auto set_failed = [&]() { *((volatile int*)&s_fail) = 1; };

    // ================================================================ producer
    // Lane 0 of the producer warp issues every bulk copy.
    uint32_t fiss = 0;        // parity of the next load's full[] phase, per slot
    uint32_t loaded = 0;      // slots that received at least one load
    uint32_t epar = 0;        // next empty[] phase to wait for, per ring slot
    uint32_t used = 0;        // ring slots holding a phase A tile not yet released
    uint32_t cpp = 0;         // slots with a TMEM-copy commit not yet waited for
    uint32_t cppar = 0;       // next cpdone[] phase to wait for, per slot
    uint64_t pol_keep = 0, pol_stream = 0;
    const bool pl = producer && lane == 0;
    if (pl) {
        if (P.hints) {
            pol_keep = policy_evict_last();
            pol_stream = policy_evict_first();
        } else {
            pol_keep = pol_stream = policy_evict_normal();
        }
    }
    auto issue = [&](int t, int s, uint64_t pol) {
        const uint32_t bytes = (uint32_t)t_nu(t) * (uint32_t)P.unit_bytes;
        const int64_t off = t_u0(t) * P.unit_bytes;
        unsigned char* d = slot_ptr(s);
        mbar_arrive_expect_tx(&full[s], bytes * NT);
        if (P.hints) {
            bulk_load(d, a.src0 + off, bytes, &full[s], pol);
            if (NT == 2) bulk_load(d + P.half_bytes, a.src1 + off, bytes, &full[s], pol);
        } else {
            bulk_load_plain(d, a.src0 + off, bytes, &full[s]);
            if (NT == 2) bulk_load_plain(d + P.half_bytes, a.src1 + off, bytes, &full[s]);
        }
        fiss ^= 1u << s;
        loaded |= 1u << s;
    };
    // Waits until the TMEM copies out of slot s have finished reading it.
    auto wait_cp = [&](int s) -> bool {
        if (!((cpp >> s) & 1u)) return true;
        const bool ok = mbar_wait(&cpdone[s], (cppar >> s) & 1u, a.budget_ns, a.wait_prod);
        cppar ^= 1u << s;
        cpp &= ~(1u << s);
        return ok;
    };
    // Waits until the consumers released ring slot s after its phase A tile
    // (and any TMEM copy out of it finished).
    auto wait_empty = [&](int s) -> bool {
        if (!((used >> s) & 1u)) return wait_cp(s);
        const bool ok = mbar_wait(&empty[s], (epar >> s) & 1u, a.budget_ns, a.wait_prod);
        epar ^= 1u << s;
        used &= ~(1u << s);
        return ok && wait_cp(s);
    };
    if (pl) {
        for (int t = 0; t < n && !failed(); ++t) {
            const int s = slotA(t);
            if (t < nring) {
                if (!wait_empty(s)) { set_failed(); break; }
                used |= 1u << s;
            }
            // tiles read again in phase B stay in L2; stashed or resident ones need not
            const bool again = (stash ? t >= tlo && t < thi : t < nring) && !ring_resident(t);
            issue(t, s, again ? pol_keep : pol_stream);
            if (scp && t * tpg < Jc) cpp |= 1u << s;   // the copier warp copies it to TMEM
        }
        // Phase B: the j-th streamed tile is t = thi-1-j, in slot t % ring.  The
        // first one of each slot is either still there from phase A or is
        // loaded as soon as phase A releases the slot.
        const int pro = min(ring, nB);
        for (int j = 0; j < pro && !failed(); ++j) {
            const int t = thi - 1 - j;
            if (ring_resident(t)) continue;
            if (!wait_empty(t % ring)) { set_failed(); break; }
            issue(t, t % ring, pol_stream);
        }
        // every TMEM copy has finished before phase B reads TMEM
        for (int s = 0; s < ring && scp && !failed(); ++s)
            if (!wait_cp(s)) set_failed();
        if (scp) tmem_fence_before_sync();
    }

    // ================================================================ consumers
    uint32_t fpar = 0;   // consumers' next full[] phase parity, per slot
    // Warp-uniform bounded wait for slot s: lane 0 polls the barrier, the warp
    // then synchronises (ordering lane 0's acquire before the other lanes'
    // reads of the slot).
    auto cwait = [&](int s) -> bool {
        int ok = 1;
        if (lane == 0) ok = mbar_wait(&full[s], (fpar >> s) & 1u, a.budget_ns, a.wait_cons);
        __syncwarp();
        ok = __shfl_sync(0xffffffffu, ok, 0);
        fpar ^= 1u << s;
        if (!ok) set_failed();
        return ok && !__any_sync(0xffffffffu, failed() ? 1 : 0);
    };
    auto release = [&](uint64_t* bar) {
        __syncwarp();
        if (lane == 0) mbar_arrive(bar);
    };

    // NHWC mapping: consumer thread -> 16-byte column(s) and a row phase.
    int col[CPT];
    bool colok[CPT];
    int phase = 0;
    const int VC = P.VC, RP = P.RP, RBY = P.VC * 16;
    if (LAYOUT == kNHWC) {
        if (CPT == 1) {
            col[0] = tid % VC;
            phase = tid / VC;
            colok[0] = consumer && phase < RP;
        } else {
#pragma unroll
            for (int k = 0; k < CPT; ++k) {
                col[k] = tid + k * NC;
                colok[k] = consumer && col[k] < VC;
            }
        }
    } else {
#pragma unroll
        for (int k = 0; k < CPT; ++k) {
            col[k] = 0;
            colok[k] = false;
        }
    }
    const bool active = LAYOUT == kNHWC && colok[0];
    // byte offset of this thread's first 16-byte vector in a tile, and the
    // stride between its rows
    uint32_t voff[CPT];
#pragma unroll
    for (int k = 0; k < CPT; ++k) voff[k] = (uint32_t)(phase * RBY + col[k] * 16);
    const uint32_t vstep = (uint32_t)(RP * RBY);
    const uint32_t slots_sa = smem_u32(slots);
    // rows of a tile with `rows` rows that this thread handles
    auto my_rows = [&](int rows) -> int { return rows > phase ? (rows - 1 - phase) / RP + 1 : 0; };
    // Stash: js is the ordinal of this thread's first stashed row (its rows
    // are phase + RP*j of the CTA's range); stashed row js+i lives at TMEM
    // columns (i*VPR + v)*4 .. +3 (v: vector of the row) of the thread's lane
    // in the warp's quadrant, the two warps of a quadrant 256 columns apart.
    constexpr int VPR = CPT * NT;
    int js = 0;
    if (stash && !sfirst) {
        const int64_t sb0 = nrows - S;
        int64_t r = ((int64_t)phase - sb0) % RP;
        if (r < 0) r += RP;
        js = (int)((sb0 + r - phase) / RP);
    }
    const uint32_t tm_thread =
        tmem_base + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(256 * ((warp >> 2) & 1));
    const int tile_ord = P.tile_units / RP;   // row ordinals per tile and thread (NHWC)
    // NCHW mapping: groups of L lanes per plane.
    const int L = P.L;
    const int GP = NC / L;
    const int grp = tid / L, glane = tid % L;
    const int HW = (int)a.HW;
    const int pbytes = HW * (int)sizeof(typename Storage<DT>::T);
    const float inv_hw = 1.f / (float)HW;
    const double inv_hw_d = 1.0 / (double)HW;
    const float p = a.p, inv_p = a.inv_p;
    const bool le1 = p <= 1.f;

    // NHWC accumulators: forward (sum d, sum d^2 with d = x - K); backward
    // (sum dy, sum dy*y).
    float2 acc0[NQ], acc1[NQ], piv[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        acc0[q] = f2(0.f, 0.f);
        acc1[q] = f2(0.f, 0.f);
        piv[q] = f2(0.f, 0.f);
    }
    // rows of the CTA's range this thread accumulates (NHWC): phase, phase +
    // RP, ...
    // (a CTA owns fewer than 2^31 units; the host plan checks it)
    const int nrows32 = (int)nrows;
    const int rq = nrows32 / RP, rr = nrows32 - rq * RP;   // rows per phase: rq or rq + 1
    const int my_n = LAYOUT == kNHWC ? rq + (phase < rr ? 1 : 0) : 0;
    if (DIR == 0 && LAYOUT == kNHWC && active && my_n > 0) {
        // pivot K (kept negated): the thread's own first value of each of its
        // channels, so its fp32 sums stay as small as the channel's spread
        // allows whatever the data's offset (a pivot shared by the whole grid
        // loses accuracy when that one value is far from the mean)
        const uint4* row = reinterpret_cast<const uint4*>(a.src0 + (u0 + phase) * (int64_t)RBY);
#pragma unroll
        for (int k = 0; k < CPT; ++k)
            if (colok[k]) {
                float2 f[NP];
                Pairs<DT>::unpack(__ldg(row + col[k]), f);
#pragma unroll
                for (int q = 0; q < NP; ++q) piv[k * NP + q] = f2(-f[q].x, -f[q].y);
            }
    }

    // standard / checkpointing backward (NHWC): the constants with which this
    // thread recovers xhat and y from the stored values of its channels
    float2 pxs[NQ], pxb[NQ], pys[NQ], pyb[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        pxs[q] = f2(1.f, 1.f);
        pxb[q] = pys[q] = pyb[q] = f2(0.f, 0.f);
    }
    if (SRCV && LAYOUT == kNHWC && active) {
#pragma unroll
        for (int k = 0; k < CPT; ++k)
            if (colok[k])
#pragma unroll
                for (int q = 0; q < NP; ++q) {
                    const int j = k * NP + q;
                    const int64_t ch = (int64_t)(col[k] * NP + q) * 2;
                    float v[2][4];
#pragma unroll
                    for (int e = 0; e < 2; ++e)
                        src_affine<MODE>(__ldg(a.gamma + ch + e), __ldg(a.beta + ch + e),
                                         MODE == kModeBwdX ? __ldg(a.mean_in + ch + e) : 0.f,
                                         MODE == kModeBwdX ? __ldg(a.var_in + ch + e) : 1.f,
                                         a.eps, v[e][0], v[e][1], v[e][2], v[e][3]);
                    pxs[j] = f2(v[0][0], v[1][0]);
                    pxb[j] = f2(v[0][1], v[1][1]);
                    pys[j] = f2(v[0][2], v[1][2]);
                    pyb[j] = f2(v[0][3], v[1][3]);
                }
    }

    if (copier && lane == 0 && scp) {
        // Each stashed tile, once landed: its row groups into TMEM (fwd: 8
        // columns per group; bwd: z then dz, 16 columns per group), then a
        // commit to cpdone[] that the producer waits for before refilling.
        // The k-th tile of a slot completes full[] phase k; the producer does
        // not reload the slot before this commit, so the parity cannot alias.
        for (int t = 0; t < nring && t * tpg < Jc && !failed(); ++t) {
            const int s = slotA(t);
            if (!mbar_wait(&full[s], (uint32_t)((t / ring) & 1), a.budget_ns, a.wait_prod)) {
                set_failed();
                break;
            }
            const uint32_t sbase = slots_sa + (uint32_t)s * (uint32_t)P.slot_bytes;
            for (int gi = 0; gi < tpg && t * tpg + gi < Jc; ++gi) {
                const int i = t * tpg + gi;
#pragma unroll
                for (int kc = 0; kc < CPT; ++kc)
#pragma unroll
                    for (int k = 0; k < NT; ++k) {
                        const uint32_t src = sbase + (uint32_t)(k * P.half_bytes) +
                                             (uint32_t)(gi * CPT + kc) * 4096u;
                        tmem_cp_128x256b(tmem_base + (uint32_t)(8 * (NT * (i * CPT + kc) + k)),
                                         smem_desc_plain(src, 2048u, 128u));
                    }
            }
            tmem_commit(&cpdone[s]);
        }
    }
    if (consumer) {
        acct_start();
        for (int t = 0; t < n; ++t) {
            const int s = slotA(t);
            if (!cwait(s)) break;
            acct_wait();
            const unsigned char* base = slot_ptr(s);
            if (LAYOUT == kNHWC) {
                const int rows = t_nu(t);
                if (active) {
                    const int m = my_rows(rows);
                    const uint32_t sb = slots_sa + (uint32_t)s * (uint32_t)P.slot_bytes;
                    acct_work();
                    // rows in batches of RB: all loads of a batch first, then the math
                    for (int i0 = 0; i0 < m; i0 += RB) {
                        uint4 vz[RB][CPT], vd[RB][CPT];
#pragma unroll
                        for (int u = 0; u < RB; ++u)
#pragma unroll
                            for (int k = 0; k < CPT; ++k) {
                                if (i0 + u >= m || (CPT > 1 && !colok[k])) continue;
                                const uint32_t o = sb + voff[k] + (uint32_t)(i0 + u) * vstep;
                                vz[u][k] = lds128(o);
                                if (DIR == 1) vd[u][k] = lds128(o + (uint32_t)P.half_bytes);
                            }
                        if (stash && !scp) {
                            // rows from ordinal js on also go to TMEM (warp-uniform:
                            // a warp's lanes share the row phase): a whole batch as
                            // one 16/32-column store, else vector by vector
                            const int ib = t * tile_ord + i0 - js;
                            const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
                            if (ib >= 0 && ib + RB <= Jc && i0 + RB <= m) {
                                uint4 w[RB * VPR];
#pragma unroll
                                for (int u = 0; u < RB; ++u)
#pragma unroll
                                    for (int k = 0; k < CPT; ++k) {
                                        const bool ok = CPT == 1 || colok[k];
                                        w[(u * CPT + k) * NT] = ok ? vz[u][k] : z4;
                                        if (DIR == 1) w[(u * CPT + k) * NT + 1] = ok ? vd[u][k] : z4;
                                    }
                                const uint32_t ta = tm_thread + (uint32_t)(ib * VPR * 4);
                                if (NT == 1) tmem_st16(ta, w);
                                else tmem_st32(ta, w);
                            } else {
#pragma unroll
                                for (int u = 0; u < RB; ++u) {
                                    const int i = ib + u;
                                    if (i0 + u < m && i >= 0 && i < Jc) {
#pragma unroll
                                        for (int k = 0; k < CPT; ++k) {
                                            const uint32_t ta = tm_thread + (uint32_t)((i * VPR + k * NT) * 4);
                                            const bool ok = CPT == 1 || colok[k];
                                            tmem_st4(ta, ok ? vz[u][k] : z4);
                                            if (DIR == 1) tmem_st4(ta + 4, ok ? vd[u][k] : z4);
                                        }
                                    }
                                }
                            }
                        }
#pragma unroll
                        for (int u = 0; u < RB; ++u)
#pragma unroll
                            for (int k = 0; k < CPT; ++k) {
                                if (i0 + u >= m || (CPT > 1 && !colok[k])) continue;
                                if (DIR == 0) {
                                    float2 f[NP];
                                    Pairs<DT>::unpack(vz[u][k], f);
#pragma unroll
                                    for (int q = 0; q < NP; ++q) {
                                        const int j = k * NP + q;
                                        const float2 d = __fadd2_rn(f[q], piv[j]);
                                        acc0[j] = __fadd2_rn(acc0[j], d);
                                        acc1[j] = __ffma2_rn(d, d, acc1[j]);
                                    }
                                } else if (SRCV) {
                                    // standard / checkpointing: xhat and y from the
                                    // stored value, dy from y
                                    float2 fa[NP], fd[NP];
                                    Pairs<DT>::unpack(vz[u][k], fa);
                                    Pairs<DT>::unpack(vd[u][k], fd);
#pragma unroll
                                    for (int q = 0; q < NP; ++q) {
                                        const int j = k * NP + q;
                                        const float2 xh = MODE == kModeBwdX
                                                              ? __ffma2_rn(fa[q], pxs[j], pxb[j])
                                                              : fa[q];
                                        const float2 y = __ffma2_rn(fa[q], pys[j], pyb[j]);
                                        const float2 dy =
                                            f2(act_dy_from_y<ACT, DT>(y.x, fd[q].x, p),
                                               act_dy_from_y<ACT, DT>(y.y, fd[q].y, p));
                                        acc0[j] = __fadd2_rn(acc0[j], dy);
                                        acc1[j] = __ffma2_rn(dy, xh, acc1[j]);
                                    }
                                } else {
                                    float2 fz[NP], fd[NP];
                                    Pairs<DT>::unpack(vz[u][k], fz);
                                    Pairs<DT>::unpack(vd[u][k], fd);
#pragma unroll
                                    for (int q = 0; q < NP; ++q) {
                                        const int j = k * NP + q;
                                        if (ACT == kLeaky) {
                                            // dy*y = dz*z on both branches
                                            acc1[j] = __ffma2_rn(fd[q], fz[q], acc1[j]);
                                            const float2 ad = __fmul2_rn(fd[q], f2(p, p));
                                            const float2 dy = f2(fz[q].x > 0.f ? fd[q].x : ad.x,
                                                                 fz[q].y > 0.f ? fd[q].y : ad.y);
                                            acc0[j] = __fadd2_rn(acc0[j], dy);
                                        } else if (ACT == kIdent) {
                                            acc1[j] = __ffma2_rn(fd[q], fz[q], acc1[j]);
                                            acc0[j] = __fadd2_rn(acc0[j], fd[q]);
                                        } else {
                                            float y0, y1, d0, d1;
                                            act_backward<ACT, DT>(fz[q].x, fd[q].x, p, inv_p, y0,
                                                                  d0);
                                            act_backward<ACT, DT>(fz[q].y, fd[q].y, p, inv_p, y1,
                                                                  d1);
                                            acc0[j] = __fadd2_rn(acc0[j], f2(d0, d1));
                                            acc1[j] = __ffma2_rn(f2(d0, d1), f2(y0, y1), acc1[j]);
                                        }
                                    }
                                }
                            }
                    }
                    acct_comp();
                }
            } else {
                // NCHW: one partial per plane
                const int np = t_nu(t) * P.g;
                const int64_t plane0 = t_u0(t) * P.g;
                for (int bp = 0; bp < np; bp += GP) {
                    const int pp = bp + grp;
                    const bool valid = pp < np;
                    const unsigned char* pz = base + (size_t)pp * pbytes;
                    // Elements i = glane + L*j of the plane, in chunks of PC: the
                    // chunk's loads first, then its math into two accumulator
                    // chains (even / odd k), then the remainder into chain 0.
                    constexpr int PC = 8;
                    auto lim = [&]() { return HW - (PC - 1) * L; };   // chunk start bound
                    if (DIR == 0 && DT == kF32) {
                        // fp32 storage: exact two passes, mean then M2
                        float sa = 0.f, sb = 0.f;
                        if (valid) {
                            int i = glane;
                            for (; i < lim(); i += PC * L) {
                                float x[PC];
#pragma unroll
                                for (int k = 0; k < PC; ++k) x[k] = Elem<DT>::ld(pz, i + k * L);
#pragma unroll
                                for (int k = 0; k < PC; k += 2) {
                                    sa += x[k];
                                    sb += x[k + 1];
                                }
                            }
                            for (; i < HW; i += L) sa += Elem<DT>::ld(pz, i);
                        }
                        const float mean = group_sum(sa + sb, L) * inv_hw;
                        float qa = 0.f, qb = 0.f;
                        if (valid) {
                            int i = glane;
                            for (; i < lim(); i += PC * L) {
                                float x[PC];
#pragma unroll
                                for (int k = 0; k < PC; ++k) x[k] = Elem<DT>::ld(pz, i + k * L) - mean;
#pragma unroll
                                for (int k = 0; k < PC; k += 2) {
                                    qa = fmaf(x[k], x[k], qa);
                                    qb = fmaf(x[k + 1], x[k + 1], qb);
                                }
                            }
                            for (; i < HW; i += L) {
                                const float d = Elem<DT>::ld(pz, i) - mean;
                                qa = fmaf(d, d, qa);
                            }
                        }
                        const float sq = group_sum(qa + qb, L);
                        if (valid && glane == 0) a.part[plane0 + pp] = make_double2(mean, sq);
                    } else if (DIR == 0) {
                        // 16-bit storage: one pass around the plane's first element
                        // k: mean = k + S1/HW, M2 = S2 - S1^2/HW
                        float s1a = 0.f, s2a = 0.f, s1b = 0.f, s2b = 0.f, piv = 0.f;
                        if (valid) {
                            piv = Elem<DT>::ld(pz, 0);
                            int i = glane;
                            for (; i < lim(); i += PC * L) {
                                float x[PC];
#pragma unroll
                                for (int k = 0; k < PC; ++k) x[k] = Elem<DT>::ld(pz, i + k * L) - piv;
#pragma unroll
                                for (int k = 0; k < PC; k += 2) {
                                    s1a += x[k];
                                    s2a = fmaf(x[k], x[k], s2a);
                                    s1b += x[k + 1];
                                    s2b = fmaf(x[k + 1], x[k + 1], s2b);
                                }
                            }
                            for (; i < HW; i += L) {
                                const float d = Elem<DT>::ld(pz, i) - piv;
                                s1a += d;
                                s2a = fmaf(d, d, s2a);
                            }
                        }
                        const float s1 = group_sum(s1a + s1b, L);
                        const float s2 = group_sum(s2a + s2b, L);
                        if (valid && glane == 0) {
                            const double d1 = s1;
                            a.part[plane0 + pp] =
                                make_double2((double)piv + d1 * (double)inv_hw_d,
                                             (double)s2 - d1 * d1 * (double)inv_hw_d);
                        }
                    } else if (SRCV) {
                        // standard / checkpointing: xhat and y from the stored
                        // value with the plane's channel constants
                        float s1a = 0.f, sya = 0.f, s1b = 0.f, syb = 0.f;
                        if (valid) {
                            const int64_t c = (plane0 + pp) % a.C;
                            float xs, xb, ys, yb;
                            src_affine<MODE>(__ldg(a.gamma + c), __ldg(a.beta + c),
                                             MODE == kModeBwdX ? __ldg(a.mean_in + c) : 0.f,
                                             MODE == kModeBwdX ? __ldg(a.var_in + c) : 1.f,
                                             a.eps, xs, xb, ys, yb);
                            auto add = [&](float av, float dv, float& s1, float& sy) {
                                const float xh = MODE == kModeBwdX ? fmaf(av, xs, xb) : av;
                                const float dy = act_dy_from_y<ACT, DT>(fmaf(av, ys, yb), dv, p);
                                s1 += dy;
                                sy = fmaf(dy, xh, sy);
                            };
                            const unsigned char* pd = pz + P.half_bytes;
                            int i = glane;
                            for (; i < lim(); i += PC * L) {
                                float av[PC], dv[PC];
#pragma unroll
                                for (int k = 0; k < PC; ++k) {
                                    av[k] = Elem<DT>::ld(pz, i + k * L);
                                    dv[k] = Elem<DT>::ld(pd, i + k * L);
                                }
#pragma unroll
                                for (int k = 0; k < PC; k += 2) {
                                    add(av[k], dv[k], s1a, sya);
                                    add(av[k + 1], dv[k + 1], s1b, syb);
                                }
                            }
                            for (; i < HW; i += L)
                                add(Elem<DT>::ld(pz, i), Elem<DT>::ld(pd, i), s1a, sya);
                        }
                        const float s1 = group_sum(s1a + s1b, L);
                        const float sy = group_sum(sya + syb, L);
                        if (valid && glane == 0) a.part[plane0 + pp] = make_double2(s1, sy);
                    } else {
                        float s1a = 0.f, sya = 0.f, s1b = 0.f, syb = 0.f;
                        if (valid) {
                            const unsigned char* pd = pz + P.half_bytes;
                            int i = glane;
                            for (; i < lim(); i += PC * L) {
                                float zv[PC], dv[PC];
#pragma unroll
                                for (int k = 0; k < PC; ++k) {
                                    zv[k] = Elem<DT>::ld(pz, i + k * L);
                                    dv[k] = Elem<DT>::ld(pd, i + k * L);
                                }
#pragma unroll
                                for (int k = 0; k < PC; k += 2) {
                                    float ya, dya, yb, dyb;
                                    act_backward<ACT, DT>(zv[k], dv[k], p, inv_p, ya, dya);
                                    act_backward<ACT, DT>(zv[k + 1], dv[k + 1], p, inv_p, yb, dyb);
                                    s1a += dya;
                                    sya = fmaf(dya, ya, sya);
                                    s1b += dyb;
                                    syb = fmaf(dyb, yb, syb);
                                }
                            }
                            for (; i < HW; i += L) {
                                float ya, dya;
                                act_backward<ACT, DT>(Elem<DT>::ld(pz, i), Elem<DT>::ld(pd, i), p,
                                                      inv_p, ya, dya);
                                s1a += dya;
                                sya = fmaf(dya, ya, sya);
                            }
                        }
                        const float s1 = group_sum(s1a + s1b, L);
                        const float sy = group_sum(sya + syb, L);
                        if (valid && glane == 0) a.part[plane0 + pp] = make_double2(s1, sy);
                    }
                }
            }
            if (t < nring) release(&empty[s]);
            acct_work();
        }
        acct_flush(9);
        if (stash && !scp) tmem_wait_st();   // this thread's stores land before its loads
    }
    __syncthreads();
    if (scp) tmem_fence_after_sync();   // the producer saw every TMEM copy complete
    stamp(1, tid == 0);

    // ------------------------------------------- per-CTA merge (NHWC)
    if (!failed() && LAYOUT == kNHWC && DIR == 0) {
        // Forward: each thread's sums around its pivot K become (mean, M2) in
        // fp64: mean = K + S1/n, M2 = S2 - S1^2/n.  Row phases 1..RP-1 publish
        // them ([phase-1][pair][mean | M2][column] double2s); phase 0 adds them
        // around its own mean R in phase order:
        //   s1 = sum n_p (mean_p - R),  s2 = sum M2_p + n_p (mean_p - R)^2,
        // giving the CTA's (R + s1/n, s2 - s1^2/n) over its nrows rows.
        const double inv_n = my_n > 0 ? 1.0 / (double)my_n : 0.0;
        auto summary = [&](int i, double2& mean, double2& m2) {
            const double s1x = acc0[i].x, s1y = acc0[i].y;
            mean = make_double2(s1x * inv_n - (double)piv[i].x, s1y * inv_n - (double)piv[i].y);
            m2 = make_double2((double)acc1[i].x - s1x * s1x * inv_n,
                              (double)acc1[i].y - s1y * s1y * inv_n);
        };
        if (CPT == 1 && RP > 1) {
            double2* scr = reinterpret_cast<double2*>(scratch);
            if (colok[0] && phase > 0 && my_n > 0) {
#pragma unroll
                for (int q = 0; q < NP; ++q) {
                    double2 mean, m2;
                    summary(q, mean, m2);
                    scr[(((phase - 1) * NP + q) * 2) * VC + col[0]] = mean;
                    scr[(((phase - 1) * NP + q) * 2 + 1) * VC + col[0]] = m2;
                }
            }
            __syncthreads();
            if (colok[0] && phase == 0) {
                const double inv_rows = 1.0 / (double)nrows;
                double2 R[NP], s1[NP], s2[NP];
#pragma unroll
                for (int q = 0; q < NP; ++q) {
                    summary(q, R[q], s2[q]);
                    s1[q] = make_double2(0.0, 0.0);
                }
                for (int ph = 1; ph < RP && ph < nrows32; ++ph) {
                    const double np = (double)(rq + (ph < rr ? 1 : 0));
#pragma unroll
                    for (int q = 0; q < NP; ++q) {
                        const double2 m = scr[(((ph - 1) * NP + q) * 2) * VC + col[0]];
                        const double2 v = scr[(((ph - 1) * NP + q) * 2 + 1) * VC + col[0]];
                        const double dx = m.x - R[q].x, dy = m.y - R[q].y;
                        s1[q].x += np * dx;
                        s1[q].y += np * dy;
                        s2[q].x += v.x + np * dx * dx;
                        s2[q].y += v.y + np * dy * dy;
                    }
                }
#pragma unroll
                for (int q = 0; q < NP; ++q) {
                    const int64_t ch = (int64_t)(col[0] * NP + q) * 2;
                    double2* dstp = a.part + ch * G + b;   // channel-major
                    dstp[0] = make_double2(R[q].x + s1[q].x * inv_rows,
                                           s2[q].x - s1[q].x * s1[q].x * inv_rows);
                    dstp[G] = make_double2(R[q].y + s1[q].y * inv_rows,
                                           s2[q].y - s1[q].y * s1[q].y * inv_rows);
                }
            }
        } else if (active && phase == 0) {
            // one thread per column: its summary is the CTA's
#pragma unroll
            for (int k = 0; k < CPT; ++k)
                if (colok[k])
#pragma unroll
                    for (int q = 0; q < NP; ++q) {
                        double2 mean, m2;
                        summary(k * NP + q, mean, m2);
                        const int64_t ch = (int64_t)(col[k] * NP + q) * 2;
                        double2* dstp = a.part + ch * G + b;   // channel-major
                        dstp[0] = make_double2(mean.x, m2.x);
                        dstp[G] = make_double2(mean.y, m2.y);
                    }
        }
        stamp(6, tid == 0);
    }
    if (!failed() && LAYOUT == kNHWC && DIR == 1) {
        if (CPT == 1 && RP > 1) {
            // Row phases 1..RP-1 publish their sums ([phase-1][pair][column]
            // float4s, so a warp's stores and loads are contiguous); phase 0
            // adds them in phase order.
            float4* scr = reinterpret_cast<float4*>(scratch);
            if (colok[0] && phase > 0) {
#pragma unroll
                for (int q = 0; q < NP; ++q)
                    scr[((phase - 1) * NP + q) * VC + col[0]] =
                        make_float4(acc0[q].x, acc0[q].y, acc1[q].x, acc1[q].y);
            }
            __syncthreads();
            if (colok[0] && phase == 0) {
                for (int ph = 1; ph < RP; ++ph) {
                    float4 v[NP];
#pragma unroll
                    for (int q = 0; q < NP; ++q) v[q] = scr[((ph - 1) * NP + q) * VC + col[0]];
#pragma unroll
                    for (int q = 0; q < NP; ++q) {
                        acc0[q] = __fadd2_rn(acc0[q], f2(v[q].x, v[q].y));
                        acc1[q] = __fadd2_rn(acc1[q], f2(v[q].z, v[q].w));
                    }
                }
            }
        }
        stamp(6, tid == 0);
        if (active && phase == 0) {
            // (sum dy, sum dy*y)
#pragma unroll
            for (int k = 0; k < CPT; ++k)
                if (colok[k])
#pragma unroll
                    for (int q = 0; q < NP; ++q) {
                        const int64_t ch = (int64_t)(col[k] * NP + q) * 2;
                        const int i = k * NP + q;
                        double2* dstp = a.part + ch * G + b;   // channel-major
                        dstp[0] = make_double2(acc0[i].x, acc1[i].x);
                        dstp[G] = make_double2(acc0[i].y, acc1[i].y);
                    }
        }
    }
    stamp(2, tid == 0);

    // ------------------------------------------------- barriers and finalize
    if (b == a.stall_cta && tid == 0) {
        // injected failure: a wait on a flag nothing sets runs out (bounded)
        const unsigned long long t0 = global_ns();
        while (ld_acquire_gpu(&a.ctl->never_set) == 0u && global_ns() - t0 < 2 * a.budget_ns) {
        }
        atomicOr(&a.ctl->status, kStTimeout);
        set_failed();
    }
    // Finalize (below): one consumer half-warp per channel pair, each lane
    // caching up to KC partials k = lane%16 + 16 i.  The forward weighs them by
    // the values behind them: NHWC, the rows of CTA k; NCHW, one plane.  Their
    // counts are known before the partials are.
    constexpr int KC = 10;   // partials cached per lane when K <= 160
    const int64_t K = LAYOUT == kNHWC ? (int64_t)G : a.N;
    // partial k of channel c: NHWC channel-major (a half-warp's loads of one
    // channel are contiguous), NCHW per plane (n, c) in plane order
    auto part_at = [&](int64_t k, int64_t c) -> double2 {
        return LAYOUT == kNHWC ? a.part[c * K + k] : a.part[k * a.C + c];
    };
    const bool cached = K <= 16 * KC;
    auto count_of = [&](int64_t k) -> double {
        if (LAYOUT == kNCHW) return (double)a.HW;
        return (double)(uq + (k >= G - ur ? 1 : 0));
    };
    double wk[KC];
#pragma unroll
    for (int i = 0; i < KC; ++i) {
        const int64_t k = (lane & 15) + 16 * i;
        wk[i] = DIR == 0 && consumer && cached && k < K ? count_of(k) : 0.0;
    }
    grid_barrier(a.ctl, bbase + (uint32_t)G, a.budget_ns, &s_fail);
    stamp(3, tid == 0);
    if (consumer && (lane & 15) == 0) cp_async_wait_all();   // s_par (issued at launch)
    if (!failed() && consumer) {
        // one consumer half-warp per channel over the whole grid, fp64, fixed
        // order; a warp takes the channels 2cp and 2cp+1 (the loop is
        // warp-uniform; a half without a channel computes on a stand-in).
        // Channel pairs go to warp 0 of every CTA first, then warp 1, ...: the
        // scattered partial loads spread over as many SMs as there are pairs.
        const int hl = lane & 15, half = lane >> 4;
        const int64_t nw = (int64_t)G * CW;
        bool first = true;
        for (int64_t cpair = (int64_t)warp * G + b; cpair * 2 < a.C;
             cpair += nw, first = false) {
            const int64_t cw = cpair * 2 + half;
            const bool cv = cw < a.C;
            const int64_t c = cv ? cw : a.C - 1;
            double2 pk[KC];
#pragma unroll
            for (int i = 0; i < KC; ++i) {
                const int64_t k = hl + 16 * i;
                pk[i] = cached && k < K ? part_at(k, c) : make_double2(0.0, 0.0);
            }
            // per-channel parameters (lane 0 of the half uses them)
            float gmf = 0.f, btf = 0.f, vif = 0.f, mnf = 0.f;
            if (hl == 0) {
                if (first) {
                    gmf = s_par[warp][half][0];
                    btf = s_par[warp][half][1];
                    vif = s_par[warp][half][2];
                    mnf = s_par[warp][half][3];
                } else {
                    gmf = a.gamma[c];
                    btf = a.beta[c];
                    if (DIR == 1) vif = a.var_in[c];
                    if (MODE == kModeBwdX) mnf = a.mean_in[c];
                }
            }
            if (DIR == 0) {
                // Partials are (mean_k, M2_k) over n_k values (NHWC: CTA k's
                // rows; NCHW: plane k).  One pass around r, the first
                // partial's mean:
                //   s1 = sum n_k (mean_k - r),  s2 = sum M2_k + n_k (mean_k - r)^2,
                //   mean = r + s1/M,  M2 = s2 - s1^2/M.
                const double r = __shfl_sync(0xffffffffu, cached ? pk[0].x : part_at(0, c).x, 0, 16);
                double s1 = 0.0, s2 = 0.0;
                if (cached) {
#pragma unroll
                    for (int i = 0; i < KC; ++i) {
                        const double w = wk[i] * (pk[i].x - r);
                        s1 += w;
                        s2 += pk[i].y + w * (pk[i].x - r);
                    }
                } else {
                    for (int64_t k = hl; k < K; k += 16) {
                        const double2 v = part_at(k, c);
                        const double w = count_of(k) * (v.x - r);
                        s1 += w;
                        s2 += v.y + w * (v.x - r);
                    }
                }
                s1 = half_warp_sum(s1);
                s2 = half_warp_sum(s2);
                if (hl == 0 && cv) {
                    const double mean = r + s1 / a.M;
                    const double var = fmax((s2 - s1 * (s1 / a.M)) / a.M, 0.0);
                    a.out0[c] = (float)mean;
                    a.out1[c] = (float)var;
                    if (a.rmean != nullptr)
                        running_step(a.rmean + c, a.rvar + c, (float)mean, (float)var,
                                     a.momentum, a.unbias);
                    const double rstd = 1.0 / sqrt(var + (double)a.eps);
                    const double sc = (double)gmf * rstd;
                    if (CKPT) {
                        // xhat = (x - mean)*rstd (fp32 storage) or x*rstd - mean*rstd;
                        // y = gamma*xhat + beta
                        a.coef[c] = make_float4(DT == kF32 ? (float)-mean : (float)(-mean * rstd),
                                                (float)rstd, gmf, btf);
                    } else {
                        // (mean, scale, beta, beta - mean*scale)
                        a.coef[c] = make_float4((float)mean, (float)sc, btf,
                                                (float)((double)btf - mean * sc));
                    }
                }
            } else {
                double s1 = 0.0, sy = 0.0;
                if (cached) {
#pragma unroll
                    for (int i = 0; i < KC; ++i) {
                        s1 += pk[i].x;
                        sy += pk[i].y;
                    }
                } else {
                    for (int64_t k = hl; k < K; k += 16) {
                        const double2 v = part_at(k, c);
                        s1 += v.x;
                        sy += v.y;
                    }
                }
                s1 = half_warp_sum(s1);
                sy = half_warp_sum(sy);
                if (SRCV && hl == 0 && cv) {
                    // standard / checkpointing: dbeta = sum dy, dgamma = sum dy*xhat;
                    // dx = A dy + B xhat + Cc with A = gamma rstd, B = -A dgamma/M,
                    // Cc = -A dbeta/M, applied to the stored value a through
                    // xhat = a*xs + xb:  dx = A dy + (B xs) a + (B xb + Cc)
                    float xs, xb, ys, yb;
                    src_affine<MODE>(gmf, btf, mnf, vif, a.eps, xs, xb, ys, yb);
                    const double rstd = 1.0 / sqrt((double)vif + (double)a.eps);
                    const double A = (double)gmf * rstd;
                    const double B = -A * sy / a.M, Cc = -A * s1 / a.M;
                    a.out0[c] = (float)sy;
                    a.out1[c] = (float)s1;
                    a.coef[c] = make_float4(ys, yb, (float)A, 0.f);
                    a.coef[a.C + c] = make_float4((float)(B * (double)xs),
                                                  (float)(B * (double)xb + Cc), 0.f, 0.f);
                }
                if (!SRCV && hl == 0 && cv) {
                    const double gm = gmf, bt = btf;
                    const double rstd = 1.0 / sqrt((double)vif + (double)a.eps);
                    if (!(fabs(gm) >= 1.17549435082228750797e-38)) {   // |gamma| < FLT_MIN
                        atomicOr(&a.ctl->status, kStSingular);
                        const float qnan = __int_as_float(0x7fc00000);
                        a.out0[c] = qnan;
                        a.out1[c] = qnan;
                        a.coef[c] = make_float4(qnan, qnan, qnan, 0.f);
                    } else {
                        // dbeta = sum dy; dgamma = sum dy*xhat = (sum dy*y - beta sum dy)/gamma
                        const double dg = (sy - bt * s1) / gm;
                        a.out0[c] = (float)dg;
                        a.out1[c] = (float)s1;
                        // dx = A dy + B y + Cc
                        const double A = gm * rstd, B = -rstd * dg / a.M;
                        const double Cc = -gm * rstd * s1 / a.M - B * bt;
                        a.coef[c] = make_float4((float)A, (float)B, (float)Cc, 0.f);
                    }
                }
            }
        }
    }
    stamp(4, tid == 0);
    grid_barrier(a.ctl, bbase + 2u * (uint32_t)G, a.budget_ns, &s_fail);
    if (b == 0 && tid == 0) bar_pad(a.ctl, (uint32_t)G, 2u);
    // NCHW: the coefficients of the CTA's channel window, (u0*g + i) mod C for
    // i < ncoef, into shared memory (every thread reaches the barrier)
    const int64_t ch0 = LAYOUT == kNCHW ? (u0 * P.g) % a.C : 0;
    float4* scoef = reinterpret_cast<float4*>(scratch);
    if (LAYOUT == kNCHW && P.ncoef > 0) {
        if (consumer && !failed())
            for (int i = tid; i < P.ncoef; i += NC) {
                const int64_t c = ch0 + i;
                const int64_t cm = c >= a.C ? c - a.C : c;
                scoef[i] = a.coef[cm];
                if (NREC == 2) scoef[P.ncoef + i] = a.coef[a.C + cm];
            }
        __syncthreads();
    }
    stamp(5, tid == 0);

    // ================================================================ phase B
    if (producer) {
        if (pl && !failed()) {
            // The consumers write their results to global memory themselves;
            // the producer loads streamed tile t into slot t % ring once they
            // are done with the slot's previous phase-B tile, t + ring.
            uint32_t dpar = 0;
            bool ok = true;
            for (int j = ring; j < nB && ok; ++j) {
                const int t = thi - 1 - j;
                const int s = t % ring;
                ok = mbar_wait(&done[s], (dpar >> s) & 1u, a.budget_ns, a.wait_prod);
                dpar ^= 1u << s;
                if (!ok) break;
                issue(t, s, pol_stream);
            }
            if (!ok) set_failed();
            stamp(7, true);
        }
    } else if (consumer && !failed()) {
        // results go straight to global memory (16-byte stores)
        auto put = [&](void* g, const uint4& v) { stg128(g, v); };
        // coefficients of this thread's channels (NHWC)
        // c3/c4 are kept per channel only when a thread owns one column;
        // otherwise the backward forms them on the fly (register budget).
        constexpr int NQ34 = CPT == 1 ? NQ : 1;
        float2 c0[NQ], c1[NQ], c2[NQ], c3[NQ34], c4[NQ34];
#pragma unroll
        for (int k = 0; k < CPT; ++k)
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                const int i = k * NP + q;
                float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0, w0 = v0, w1 = v0;
                if (colok[k]) {
                    v0 = a.coef[(col[k] * NP + q) * 2];
                    v1 = a.coef[(col[k] * NP + q) * 2 + 1];
                    if (NREC == 2) {
                        w0 = a.coef[a.C + (col[k] * NP + q) * 2];
                        w1 = a.coef[a.C + (col[k] * NP + q) * 2 + 1];
                    }
                }
                if (CKPT) {
                    // the checkpointing layer runs with one column per thread
                    c0[i] = f2(v0.x, v1.x);                   // -mean or -mean*rstd
                    c1[i] = f2(v0.y, v1.y);                   // rstd
                    c2[i] = f2(v0.z, v1.z);                   // gamma
                    c3[i < NQ34 ? i : 0] = f2(v0.w, v1.w);    // beta
                } else if (SRCV) {
                    // y = a*ys + yb; dx = A dy + B' a + C' (one column per thread)
                    c0[i] = f2(v0.x, v1.x);                   // ys
                    c1[i] = f2(v0.y, v1.y);                   // yb
                    c2[i] = f2(v0.z, v1.z);                   // A
                    c3[i < NQ34 ? i : 0] = f2(w0.x, w1.x);    // B'
                    c4[i < NQ34 ? i : 0] = f2(w0.y, w1.y);    // C'
                } else if (DIR == 0) {
                    c0[i] = f2(-v0.x, -v1.x);    // -mean
                    c1[i] = f2(v0.y, v1.y);      // scale
                    c2[i] = f2(v0.w, v1.w);      // beta - mean*scale (16-bit storage)
                    if (DT == kF32) c2[i] = f2(v0.z, v1.z);   // beta (fp32 storage)
                } else {
                    c0[i] = f2(v0.x, v1.x);                   // A
                    c1[i] = f2(v0.y, v1.y);                   // B
                    c2[i] = f2(v0.z, v1.z);                   // Cc
                    if (CPT == 1) {
                        c3[i] = f2(v0.x * p, v1.x * p);           // A*a (leaky, z <= 0)
                        c4[i] = f2(v0.y * inv_p, v1.y * inv_p);   // B/a (leaky, z <= 0)
                    }
                }
            }
        // Rewrites the tile in slot s in place (forward: x -> z; backward: dz -> dx).
        // Rewrites one row's CPT vectors: forward x -> z in vz, backward
        // dz -> dx in vd (z in vz).
        // (checkpointing forward: xhat into vz, z into vo.)
        auto rewrite = [&](uint4* vz, uint4* vd, uint4* vo) {
#pragma unroll
            for (int k = 0; k < CPT; ++k) {
                if (CPT > 1 && !colok[k]) continue;
                if (CKPT) {
                    float2 f[NP], o[NP];
                    Pairs<DT>::unpack(vz[k], f);
#pragma unroll
                    for (int q = 0; q < NP; ++q) {
                        const int j = k * NP + q;
                        const float2 xh = DT == kF32 ? __fmul2_rn(__fadd2_rn(f[q], c0[j]), c1[j])
                                                     : __ffma2_rn(f[q], c1[j], c0[j]);
                        o[q] = act_forward2<ACT, DT>(__ffma2_rn(xh, c2[j], c3[j < NQ34 ? j : 0]),
                                                     p, le1);
                        f[q] = xh;
                    }
                    vz[k] = Pairs<DT>::pack(f);
                    vo[k] = Pairs<DT>::pack(o);
                } else if (SRCV) {
                    float2 fa[NP], fd[NP];
                    Pairs<DT>::unpack(vz[k], fa);
                    Pairs<DT>::unpack(vd[k], fd);
#pragma unroll
                    for (int q = 0; q < NP; ++q) {
                        const int j = k * NP + q;
                        const int jj = j < NQ34 ? j : 0;
                        const float2 y = __ffma2_rn(fa[q], c0[j], c1[j]);
                        const float2 dy = f2(act_dy_from_y<ACT, DT>(y.x, fd[q].x, p),
                                             act_dy_from_y<ACT, DT>(y.y, fd[q].y, p));
                        fd[q] = __ffma2_rn(c2[j], dy, __ffma2_rn(c3[jj], fa[q], c4[jj]));
                    }
                    vd[k] = Pairs<DT>::pack(fd);
                } else if (DIR == 0) {
                    float2 f[NP];
                    Pairs<DT>::unpack(vz[k], f);
#pragma unroll
                    for (int q = 0; q < NP; ++q) {
                        const int j = k * NP + q;
                        // 16-bit storage: y = x*scale + (beta - mean*scale); its
                        // rounding error is far below one storage ulp.  fp32:
                        // y = (x - mean)*scale + beta.
                        const float2 y = DT == kF32 ? __ffma2_rn(__fadd2_rn(f[q], c0[j]), c1[j], c2[j])
                                                    : __ffma2_rn(f[q], c1[j], c2[j]);
                        f[q] = act_forward2<ACT, DT>(y, p, le1);
                    }
                    vz[k] = Pairs<DT>::pack(f);
                } else {
                    float2 fz[NP], fd[NP];
                    Pairs<DT>::unpack(vz[k], fz);
                    Pairs<DT>::unpack(vd[k], fd);
#pragma unroll
                    for (int q = 0; q < NP; ++q) {
                        const int j = k * NP + q;
                        if (ACT == kLeaky) {
                            // dx = A dy + B y + Cc with (dy, y) = (dz, z) for z > 0
                            // and (a dz, z/a) otherwise
                            const bool px = fz[q].x > 0.f, py = fz[q].y > 0.f;
                            const float2 a3 = CPT == 1 ? c3[j < NQ34 ? j : 0]
                                                       : __fmul2_rn(c0[j], f2(p, p));
                            const float2 a4 = CPT == 1 ? c4[j < NQ34 ? j : 0]
                                                       : __fmul2_rn(c1[j], f2(inv_p, inv_p));
                            const float2 Ak = f2(px ? c0[j].x : a3.x, py ? c0[j].y : a3.y);
                            const float2 Bk = f2(px ? c1[j].x : a4.x, py ? c1[j].y : a4.y);
                            fd[q] = __ffma2_rn(Ak, fd[q], __ffma2_rn(Bk, fz[q], c2[j]));
                        } else if (ACT == kIdent) {
                            fd[q] = __ffma2_rn(c0[j], fd[q], __ffma2_rn(c1[j], fz[q], c2[j]));
                        } else {
                            float y0, y1, d0, d1;
                            act_backward<ACT, DT>(fz[q].x, fd[q].x, p, inv_p, y0, d0);
                            act_backward<ACT, DT>(fz[q].y, fd[q].y, p, inv_p, y1, d1);
                            fd[q] = __ffma2_rn(c0[j], f2(d0, d1), __ffma2_rn(c1[j], f2(y0, y1), c2[j]));
                        }
                    }
                    vd[k] = Pairs<DT>::pack(fd);
                }
            }
        };
        // Rewrites the tile in slot s -- this thread's rows q in [qlo, qhi) of
        // it -- and writes the results to global memory.
        auto apply_tile = [&](int t, int s, int qlo, int qhi) {
            unsigned char* base = slot_ptr(s);
            if (LAYOUT == kNHWC) {
                const int rows = t_nu(t);
                if (!active) return;
                const int m = min(my_rows(rows), qhi);
                const uint32_t sb = slots_sa + (uint32_t)s * (uint32_t)P.slot_bytes;
                const uint32_t hb = DIR == 0 ? 0u : (uint32_t)P.half_bytes;
                unsigned char* gtile = a.dst + t_u0(t) * P.unit_bytes;
                unsigned char* gtile2 = CKPT ? a.dst2 + t_u0(t) * P.unit_bytes : nullptr;
                // The backward with one column per thread takes its rows one at
                // a time here: batches of 2 or 4 rows measured 2-4 us slower on
                // the large layers.
                constexpr int RBB = DIR == 1 && CPT == 1 ? 1 : RB;
                // rows in batches of RBB: loads, then math, then stores
                for (int i0 = max(qlo, 0); i0 < m; i0 += RBB) {
                    uint4 vz[RBB][CPT], vd[RBB][CPT], vo[RBB][CPT];
#pragma unroll
                    for (int u = 0; u < RBB; ++u)
#pragma unroll
                        for (int k = 0; k < CPT; ++k) {
                            if (i0 + u >= m || (CPT > 1 && !colok[k])) continue;
                            const uint32_t o = sb + voff[k] + (uint32_t)(i0 + u) * vstep;
                            vz[u][k] = lds128(o);
                            if (DIR == 1) vd[u][k] = lds128(o + hb);
                        }
#pragma unroll
                    for (int u = 0; u < RBB; ++u)
                        if (i0 + u < m) rewrite(vz[u], vd[u], vo[u]);
                    // results go straight to their place in global memory
#pragma unroll
                    for (int u = 0; u < RBB; ++u)
#pragma unroll
                        for (int k = 0; k < CPT; ++k) {
                            if (i0 + u >= m || (CPT > 1 && !colok[k])) continue;
                            const size_t o = voff[k] + (size_t)(i0 + u) * vstep;
                            put(gtile + o, DIR == 0 ? vz[u][k] : vd[u][k]);
                            if (CKPT) put(gtile2 + o, vo[u][k]);
                        }
                }
            } else {
                // NCHW: 16-byte vectors of the tile.  An element's plane (and so
                // its channel) follows from its index in the tile; the
                // coefficients switch at plane boundaries.  128-bit global stores.
                constexpr int EPV = 16 / (int)sizeof(typename Storage<DT>::T);
                const int nvec = t_nu(t) * (P.unit_bytes / 16);
                const uint32_t C32 = (uint32_t)a.C, hw = (uint32_t)HW;
                // window index of the tile's first plane (channel = ch0 + index mod C)
                const uint32_t ibase = (uint32_t)(((t_u0(t) - u0) * P.g) % a.C);
                const uint32_t sbv = slots_sa + (uint32_t)s * (uint32_t)P.slot_bytes;
                // coefficient record(s) of window index i (second record: the
                // standard / checkpointing backward's B' and C')
                auto coef_at = [&](uint32_t i) -> Rec2 {
                    Rec2 r;
                    if (P.ncoef > 0) {
                        r.a = scoef[i];
                        r.b = NREC == 2 ? scoef[P.ncoef + i] : r.a;
                    } else {
                        const int64_t c = ch0 + i;
                        const int64_t cm = c >= a.C ? c - a.C : c;
                        r.a = a.coef[cm];
                        r.b = NREC == 2 ? a.coef[a.C + cm] : r.a;
                    }
                    return r;
                };
                unsigned char* gt = a.dst + t_u0(t) * P.unit_bytes;
                unsigned char* gt2 = CKPT ? a.dst2 + t_u0(t) * P.unit_bytes : nullptr;
                // This thread's vectors v = tid + NC*j start ES elements
                // apart: its plane offset `off` and window index `c` advance by
                // fixed steps (dq planes + dr elements), no division per vector.
                constexpr uint32_t ES = (uint32_t)NC * EPV;
                const uint32_t dq = ES / hw, dr = ES - dq * hw, dqc = dq % C32;
                uint32_t c, off;
                {
                    const uint32_t e0 = (uint32_t)tid * EPV;
                    // e0 / HW: e0 < 2^24, so the float quotient is off by at most one
                    uint32_t pl = (uint32_t)((float)e0 * inv_hw);
                    if (pl * hw > e0) --pl;
                    if ((pl + 1u) * hw <= e0) ++pl;
                    off = e0 - pl * hw;
                    c = (ibase + pl) % C32;
                }
                // One vector: its elements rewritten with their channels'
                // coefficients, then c and off advanced to this thread's next
                // vector.
                auto vec_work = [&](const uint4& vz, const uint4& vd, uint4& out, uint4& out2) {
                    uint32_t rem = hw - off;   // elements of plane c from this vector on
                    uint32_t cc = c;
                    float xz[EPV], xd[EPV], xo[EPV];
                    unpack_all<DT>(vz, xz);
                    if (DIR == 1) unpack_all<DT>(vd, xd);
                    // one element with coefficients q: forward (16-bit) y = x*scale +
                    // (beta - mean*scale), (fp32) y = (x - mean)*scale + beta;
                    // backward dx = A dy + B y + Cc; checkpointing forward xhat and
                    // z = phi(gamma*xhat + beta); standard / checkpointing backward
                    // y = a*ys + yb, dx = A dy + B' a + C'
                    auto rewrite_elem = [&](int k, const Rec2& r) {
                        const float4& q = r.a;
                        if (CKPT) {
                            const float xh = DT == kF32 ? (xz[k] + q.x) * q.y : fmaf(xz[k], q.y, q.x);
                            xo[k] = act_forward<ACT, DT>(fmaf(xh, q.z, q.w), p);
                            xz[k] = xh;
                        } else if (SRCV) {
                            const float dy = act_dy_from_y<ACT, DT>(fmaf(xz[k], q.x, q.y), xd[k], p);
                            xz[k] = fmaf(q.z, dy, fmaf(r.b.x, xz[k], r.b.y));
                        } else if (DIR == 0) {
                            const float y = DT == kF32 ? fmaf(xz[k] - q.x, q.y, q.z)
                                                       : fmaf(xz[k], q.y, q.w);
                            xz[k] = act_forward<ACT, DT>(y, p);
                        } else {
                            float y, dy;
                            act_backward<ACT, DT>(xz[k], xd[k], p, inv_p, y, dy);
                            xz[k] = fmaf(q.x, dy, fmaf(q.y, y, q.z));
                        }
                    };
                    if (hw >= (uint32_t)EPV) {
                        // planes at least a vector long: two coefficient sets at
                        // most, chosen per element without branches
                        const Rec2 q0 = coef_at(cc), q1 = coef_at(cc + 1u == C32 ? 0u : cc + 1u);
                        if (DIR == 0 && !CKPT) {
                            // the forward: both channels' affine results on
                            // pairs, then one select per element (not one per
                            // coefficient) and the activation on pairs
                            const float4 &a0 = q0.a, &a1 = q1.a;
#pragma unroll
                            for (int k = 0; k < EPV; k += 2) {
                                const float2 x = f2(xz[k], xz[k + 1]);
                                const float2 y0 =
                                    DT == kF32 ? __ffma2_rn(__fadd2_rn(x, f2(-a0.x, -a0.x)),
                                                            f2(a0.y, a0.y), f2(a0.z, a0.z))
                                               : __ffma2_rn(x, f2(a0.y, a0.y), f2(a0.w, a0.w));
                                const float2 y1 =
                                    DT == kF32 ? __ffma2_rn(__fadd2_rn(x, f2(-a1.x, -a1.x)),
                                                            f2(a1.y, a1.y), f2(a1.z, a1.z))
                                               : __ffma2_rn(x, f2(a1.y, a1.y), f2(a1.w, a1.w));
                                const float2 y = f2((uint32_t)k < rem ? y0.x : y1.x,
                                                    (uint32_t)k + 1u < rem ? y0.y : y1.y);
                                const float2 z = act_forward2<ACT, DT>(y, p, le1);
                                xz[k] = z.x;
                                xz[k + 1] = z.y;
                            }
                        } else if (DIR == 1 && !SRCV) {
                            // the in-place backward: dx with both channels'
                            // coefficients on pairs, then one select per element
                            const float4 &a0 = q0.a, &a1 = q1.a;
#pragma unroll
                            for (int k = 0; k < EPV; k += 2) {
                                float y0, d0, y1, d1;
                                act_backward<ACT, DT>(xz[k], xd[k], p, inv_p, y0, d0);
                                act_backward<ACT, DT>(xz[k + 1], xd[k + 1], p, inv_p, y1, d1);
                                const float2 y = f2(y0, y1), dy = f2(d0, d1);
                                const float2 r0 = __ffma2_rn(f2(a0.x, a0.x), dy,
                                                             __ffma2_rn(f2(a0.y, a0.y), y,
                                                                        f2(a0.z, a0.z)));
                                const float2 r1 = __ffma2_rn(f2(a1.x, a1.x), dy,
                                                             __ffma2_rn(f2(a1.y, a1.y), y,
                                                                        f2(a1.z, a1.z)));
                                xz[k] = (uint32_t)k < rem ? r0.x : r1.x;
                                xz[k + 1] = (uint32_t)k + 1u < rem ? r0.y : r1.y;
                            }
                        } else {
#pragma unroll
                            for (int k = 0; k < EPV; ++k) {
                                const bool first = (uint32_t)k < rem;
                                rewrite_elem(k, first ? q0 : q1);
                            }
                        }
                    } else {
                        Rec2 q = coef_at(cc);
#pragma unroll
                        for (int k = 0; k < EPV; ++k) {
                            if (rem == 0u) {
                                cc = cc + 1u == C32 ? 0u : cc + 1u;
                                q = coef_at(cc);
                                rem = hw;
                            }
                            --rem;
                            rewrite_elem(k, q);
                        }
                    }
                    off += dr;
                    c += dqc;
                    if (off >= hw) {
                        off -= hw;
                        ++c;
                    }
                    if (c >= C32) c -= C32;
                    out = pack_all<DT>(xz);
                    if (CKPT) out2 = pack_all<DT>(xo);
                };
                // one vector at a time (a two-vector interleave measured slower:
                // many-channel 40.5 / 60.3 us against 36.9 / 55.3)
                for (int v = tid; v < nvec; v += NC) {
                    const uint4 vz = lds128(sbv + (uint32_t)v * 16u);
                    const uint4 vd =
                        DIR == 1 ? lds128(sbv + (uint32_t)P.half_bytes + (uint32_t)v * 16u) : vz;
                    uint4 o, o2;
                    vec_work(vz, vd, o, o2);
                    put(gt + (size_t)v * 16, o);
                    if (CKPT) put(gt2 + (size_t)v * 16, o2);
                }
            }
        };
        acct_start();
        for (int t = n - 1; t >= nring; --t) {
            const int s = ring + (t - nring);
            apply_tile(t, s, 0, INT_MAX);
            release(&done[s]);
        }
        acct_work();
        for (int j = 0; j < nB; ++j) {
            const int t = thi - 1 - j;
            const int s = t % ring;
            // a tile still in its slot from phase A needs no wait
            if (!ring_resident(t) && !cwait(s)) break;
            acct_wait();
            // skip the stashed rows: ordinals [js, js + Jc)
            const int qlo = stash && sfirst ? Jc - t * tile_ord : 0;
            const int qhi = stash && !sfirst ? js - t * tile_ord : INT_MAX;
            apply_tile(t, s, qlo, qhi);
            acct_comp();
            release(&done[s]);
            acct_work();
        }
        // the stashed rows last: their results are written after every read
        // of phase B, so their new L2 lines evict nothing phase B still reads
        if (scp) {
            // the stashed row groups, RB at a time (four vectors per
            // tensor): this thread's column k of group i is at TMEM column
            // 8*(NT*(i*CPT + k) + tensor) + 4*(warp/4)
            unsigned char* grow = a.dst + u0 * P.unit_bytes;
            unsigned char* grow2 = CKPT ? a.dst2 + u0 * P.unit_bytes : nullptr;
            const uint32_t ta = tmem_base + ((uint32_t)(32 * (warp & 3)) << 16) +
                                (uint32_t)(4 * ((warp >> 2) & 1));
            for (int i0 = 0; i0 < Jc; i0 += RB) {
                uint4 bz[RB * CPT], bd[RB * CPT], bo[RB * CPT];
                const uint32_t f0 = (uint32_t)(i0 * CPT);
                tmem_ld4x4(ta + 8u * NT * f0, 8u * NT, bz);
                if (NT == 2) tmem_ld4x4(ta + 8u * NT * f0 + 8u, 8u * NT, bd);
#pragma unroll
                for (int u = 0; u < RB; ++u) {
                    if (i0 + u >= Jc) continue;
                    uint4* vz = bz + u * CPT;
                    uint4* vd = NT == 2 ? bd + u * CPT : bz + u * CPT;
                    rewrite(vz, vd, bo + u * CPT);
#pragma unroll
                    for (int k = 0; k < CPT; ++k) {
                        const size_t o = voff[k] + (size_t)(i0 + u) * vstep;
                        put(grow + o, DIR == 0 ? vz[k] : vd[k]);
                        if (CKPT) put(grow2 + o, bo[u * CPT + k]);
                    }
                }
            }
        } else if (stash && active) {
            // the stashed rows (no wait for any tile)
            unsigned char* grow = a.dst + u0 * P.unit_bytes;
            unsigned char* grow2 = CKPT ? a.dst2 + u0 * P.unit_bytes : nullptr;
            for (int i0 = 0; i0 < Jc; i0 += RB) {
                uint4 buf[RB * VPR];   // RB*CPT = 4 vectors per tensor
                if (NT == 1) tmem_ld16(tm_thread + (uint32_t)(i0 * VPR * 4), buf);
                else tmem_ld32(tm_thread + (uint32_t)(i0 * VPR * 4), buf);
#pragma unroll
                for (int u = 0; u < RB; ++u) {
                    if (i0 + u >= Jc) continue;
                    uint4 vz[CPT], vd[CPT], vo[CPT];
#pragma unroll
                    for (int k = 0; k < CPT; ++k) {
                        vz[k] = buf[(u * CPT + k) * NT];
                        vd[k] = buf[(u * CPT + k) * NT + (NT - 1)];
                    }
                    rewrite(vz, vd, vo);
                    const size_t j = (size_t)(js + i0 + u);
#pragma unroll
                    for (int k = 0; k < CPT; ++k) {
                        if (CPT > 1 && !colok[k]) continue;
                        put(grow + voff[k] + j * vstep, DIR == 0 ? vz[k] : vd[k]);
                        if (CKPT) put(grow2 + voff[k] + j * vstep, vo[k]);
                    }
                }
            }
        }
        acct_work();
        acct_flush(11);
    }

    // ----------------------------------------------------------- exit
    if (pl) {
        if (failed()) {
            atomicOr(&a.ctl->status, kStTimeout);
            // Wait for the last load into every slot before the CTA exits;
            // completed ones return at once.  The budget is the fixed default,
            // whatever the configured one: loads of valid memory always land.
            for (int s = 0; s < P.nslots; ++s)
                if ((loaded >> s) & 1u)
                    mbar_wait(&full[s], ((fiss >> s) & 1u) ^ 1u, kWaitBudgetNs);
        }
    }
    stamp(8, tid == 0);
    if (stash) {
        // every TMEM load of the CTA has completed (each waits in place)
        tmem_fence_before_sync();
        __syncthreads();
        tmem_fence_after_sync();
        if (warp == 0) {
            __syncwarp();
            tmem_free_all(tmem_base);
        }
    }
}

}  // namespace iabn
#include <atomic>

namespace iabn {

// Launches one instantiation cooperatively (all CTAs co-resident, which the
// grid barrier relies on).
template <int DT, int ACT, int LAYOUT, int CPT, int MODE>
cudaError_t launch_resident_one(const ResArgs& a, int smem_optin, cudaStream_t s) {
    auto kern = k_resident<DT, ACT, LAYOUT, CPT, MODE>;
    static std::atomic<uint64_t> configured{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load(std::memory_order_acquire) & bit)) {
        // leave 1 KiB of the opt-in limit for the kernel's static shared memory
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem_optin - 1024);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_release);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)a.P.G);
    cfg.blockDim = dim3(res_threads(LAYOUT, mode_dir(MODE)));
    cfg.dynamicSmemBytes = (size_t)a.P.smem_bytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, a);
    if (e == cudaSuccess) count_launches(1);
    return e;
}

template <int DT, int LAYOUT, int CPT, int MODE>
cudaError_t launch_resident_act(const ResArgs& a, int act, int smem_optin, cudaStream_t s) {
    switch (act) {
    case kLeaky: return launch_resident_one<DT, kLeaky, LAYOUT, CPT, MODE>(a, smem_optin, s);
    case kElu: return launch_resident_one<DT, kElu, LAYOUT, CPT, MODE>(a, smem_optin, s);
    default: return launch_resident_one<DT, kIdent, LAYOUT, CPT, MODE>(a, smem_optin, s);
    }
}

// The in-place layer's modes take every resident shape; the standard
// backward and the checkpointing modes only one 16-byte column per thread
// (make_plan declines the rest).
template <int DT, int MODE>
cudaError_t launch_resident_mode(const ResArgs& a, int layout, int cpt, int act, int smem_optin,
                                 cudaStream_t s) {
    if (layout == kNCHW) return launch_resident_act<DT, kNCHW, 1, MODE>(a, act, smem_optin, s);
    if (cpt == 1) return launch_resident_act<DT, kNHWC, 1, MODE>(a, act, smem_optin, s);
    if constexpr (MODE == kModeFwd || MODE == kModeBwdZ) {
        if (cpt == 2) return launch_resident_act<DT, kNHWC, 2, MODE>(a, act, smem_optin, s);
        return launch_resident_act<DT, kNHWC, 4, MODE>(a, act, smem_optin, s);
    } else {
        return cudaErrorNotSupported;
    }
}

// Defined in iabn_resident_{f32,bf16,f16}_{fwd,bwd}.cu (forward modes /
// backward modes).
#define IABN_RESIDENT_DECL(NAME)                                                              \
    cudaError_t NAME(const ResArgs& a, int layout, int cpt, int act, int mode, int smem_optin, \
                     cudaStream_t s);
IABN_RESIDENT_DECL(launch_resident_f32_fwd)
IABN_RESIDENT_DECL(launch_resident_f32_bwd)
IABN_RESIDENT_DECL(launch_resident_bf16_fwd)
IABN_RESIDENT_DECL(launch_resident_bf16_bwd)
IABN_RESIDENT_DECL(launch_resident_f16_fwd)
IABN_RESIDENT_DECL(launch_resident_f16_bwd)
#undef IABN_RESIDENT_DECL

}  // namespace iabn
