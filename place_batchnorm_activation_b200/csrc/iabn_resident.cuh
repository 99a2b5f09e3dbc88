// iabn_resident.cuh -- the resident plan of the InPlace-ABN layer: one
// cooperative, persistent kernel per call (forward or backward), one CTA per
// SM.
//
// Each CTA owns a contiguous range of "units" (NHWC: rows of C channels;
// NCHW: groups of g whole planes, g chosen so every unit starts on a 16-byte
// boundary) and streams it through shared memory in tiles with the bulk-copy
// engine (cp.async.bulk + mbarrier):
//
//   phase A  tiles 0..n-1: per-thread statistics (forward: Welford count,
//            mean, M2; backward: sum dy and sum dy*xhat) from shared memory.
//            The last D tiles land in dedicated slots and stay resident.
//   merge    NHWC: the threads of a column merge in a fixed tree, one partial
//            per (CTA, channel); NCHW: one partial per plane.
//   barrier  grid-wide (bounded wait), then a distributed fp64 finalize (one
//            warp per channel, fixed order), then a second grid barrier.
//   phase B  tiles n-1..0 (reverse order): resident tiles are rewritten in
//            place in shared memory; the others are fetched again -- the most
//            recently read first, while they are still in L2 -- and written
//            back with bulk stores.
//
// Method: "In-Place Activated BatchNorm for Memory-Optimized Training of
// DNNs" (paperlayer.ai summary), section 3: "Batch Normalization Review",
// "INPLACE-ABN", "INPLACE-ABN II".  The kernel never traps: every wait is
// bounded and a timeout sets kStTimeout in the workspace status word.
#pragma once

#include "iabn_bulk.cuh"
#include "iabn_device.cuh"
#include "iabn_internal.h"

namespace iabn {

constexpr int kResThreads = 512;
constexpr int kResWarps = kResThreads / 32;
constexpr int kMaxSlots = 30;
constexpr int kBarBytes = 256;   // mbarrier area at the start of dynamic shared memory

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
    int smem_bytes;      // dynamic shared memory of the launch
    int VC, RP;          // NHWC: 16-byte columns per row; row phases (threads per column)
    int g, L;            // NCHW: planes per unit; lanes per plane
    int hints;           // 1: L2 eviction-priority hints on the bulk copies
};

struct ResArgs {
    ResPlan P;
    int64_t N, C, HW;
    double M;
    const unsigned char* src0;   // forward: x;            backward: z
    const unsigned char* src1;   // backward: dz
    unsigned char* dst;          // forward: x (z over it); backward: dz (dx over it)
    const float* gamma;
    const float* beta;
    const float* var_in;         // backward: saved biased variance
    float* out0;                 // forward: save_mean;  backward: dgamma
    float* out1;                 // forward: save_var;   backward: dbeta
    float eps, p, inv_p;
    Control* ctl;
    double2* part;
    float4* coef;
    unsigned long long budget_ns;
};

// Sum over aligned groups of L lanes (L a power of two); every lane of the
// warp must call it.  Fixed tree, then broadcast from the group's first lane.
__device__ __forceinline__ float group_sum(float v, int L) {
    for (int o = L >> 1; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o, L);
    return __shfl_sync(0xffffffffu, v, 0, L);
}

template <int DT, int ACT, int LAYOUT, int CPT, int DIR>
__global__ void __launch_bounds__(kResThreads, 1) k_resident(const ResArgs a) {
    constexpr int NT = DIR == 0 ? 1 : 2;       // tensors per tile
    constexpr int V = Vec<DT>::N;              // elements per 16-byte vector
    constexpr int NV = CPT * V;                // channels per thread (NHWC)
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    unsigned char* slots = smem + kBarBytes;

    const ResPlan& P = a.P;
    const int tid = threadIdx.x;
    const int b = blockIdx.x;
    const int G = P.G;
    const int64_t u0 = (int64_t)b * P.units / G;
    const int64_t u1 = (int64_t)(b + 1) * P.units / G;
    const int n = (int)((u1 - u0 + P.tile_units - 1) / P.tile_units);
    const int ring = P.ring;
    const int D = min(P.nslots - ring, n);
    const int nring = n - D;

    if (tid == 0) {
        for (int s = 0; s < P.nslots; ++s) mbar_init(&bars[s], 1);
        mbar_init_fence();
    }
    __syncthreads();

    uint64_t pol_keep, pol_stream;
    if (P.hints) {
        pol_keep = policy_evict_last();
        pol_stream = policy_evict_first();
    } else {
        pol_keep = pol_stream = policy_evict_normal();
    }

    uint32_t parity = 0;    // per-slot mbarrier phase (identical in every thread)
    uint32_t pending = 0;   // slots with a load in flight (identical in every thread)

    auto t_u0 = [&](int t) -> int64_t { return u0 + (int64_t)t * P.tile_units; };
    auto t_nu = [&](int t) -> int {
        const int64_t r = u1 - t_u0(t);
        return (int)(r < P.tile_units ? r : P.tile_units);
    };
    auto slotA = [&](int t) -> int { return t < nring ? t % ring : ring + (t - nring); };
    auto slot_ptr = [&](int s) -> unsigned char* { return slots + (size_t)s * P.slot_bytes; };
    // Thread 0 issues; every thread records the slot as pending.
    auto issue = [&](int t, int s, uint64_t pol) {
        if (tid == 0) {
            const uint32_t bytes = (uint32_t)t_nu(t) * (uint32_t)P.unit_bytes;
            const int64_t off = t_u0(t) * P.unit_bytes;
            unsigned char* d = slot_ptr(s);
            mbar_arrive_expect_tx(&bars[s], bytes * NT);
            bulk_load(d, a.src0 + off, bytes, &bars[s], pol);
            if (NT == 2) bulk_load(d + P.half_bytes, a.src1 + off, bytes, &bars[s], pol);
        }
        pending |= 1u << s;
    };
    auto wait = [&](int s) -> bool {
        const bool ok = mbar_wait(&bars[s], (parity >> s) & 1u, a.budget_ns);
        parity ^= 1u << s;
        pending &= ~(1u << s);
        return ok;
    };

    // ---------------------------------------------------------- mapping
    // NHWC: thread -> 16-byte column(s) and a row phase.
    int col[CPT];
    bool colok[CPT];
    int phase = 0;
    const int VC = P.VC, RP = P.RP, RBY = P.VC * 16;
    if (LAYOUT == kNHWC) {
        if (CPT == 1) {
            col[0] = tid % VC;
            phase = tid / VC;
            colok[0] = phase < RP;
        } else {
#pragma unroll
            for (int k = 0; k < CPT; ++k) {
                col[k] = tid + k * kResThreads;
                colok[k] = col[k] < VC;
            }
        }
    }
    // NCHW: groups of L lanes per plane.
    const int L = P.L;
    const int GP = kResThreads / L;
    const int grp = tid / L, glane = tid % L;
    const int HW = (int)a.HW;
    const int pbytes = HW * (int)sizeof(typename Storage<DT>::T);
    const float inv_hw = 1.f / (float)HW;

    // per-thread accumulators (NHWC): forward (cnt, mean, m2); backward (s1, s2)
    float cnt = 0.f;
    float acc0[NV], acc1[NV];
    float kx[NV], ky[NV];   // backward: 1/gamma and -beta/gamma per channel
#pragma unroll
    for (int j = 0; j < NV; ++j) { acc0[j] = 0.f; acc1[j] = 0.f; kx[j] = 0.f; ky[j] = 0.f; }
    if (LAYOUT == kNHWC && DIR == 1) {
#pragma unroll
        for (int k = 0; k < CPT; ++k)
            if (colok[k])
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    const int ch = col[k] * V + j;
                    const float ig = 1.f / a.gamma[ch];
                    kx[k * V + j] = ig;
                    ky[k * V + j] = -a.beta[ch] * ig;
                }
    }

    bool fail = false;

    // ---------------------------------------------------------- phase A
    {
        const int pro = min(ring - 1, n);
        for (int t = 0; t < pro; ++t) issue(t, slotA(t), t < nring ? pol_keep : pol_stream);
        for (int t = 0; t < n; ++t) {
            const int tn = t + ring - 1;
            if (tn < n) issue(tn, slotA(tn), tn < nring ? pol_keep : pol_stream);
            const int s = slotA(t);
            const bool ok = wait(s);
            if (ok) {
                const unsigned char* base = slot_ptr(s);
                if (LAYOUT == kNHWC) {
                    const int rows = t_nu(t);
                    if (CPT == 2 || colok[0]) {
                        for (int r = phase; r < rows; r += RP) {
                            if (DIR == 0) {
                                cnt += 1.f;
                                const float inv = __fdividef(1.f, cnt);
#pragma unroll
                                for (int k = 0; k < CPT; ++k) {
                                    if (!colok[k]) continue;
                                    const uint4 v = *reinterpret_cast<const uint4*>(
                                        base + (size_t)r * RBY + col[k] * 16);
                                    float f[V];
                                    Vec<DT>::unpack(v, f);
#pragma unroll
                                    for (int j = 0; j < V; ++j) {
                                        float& mu = acc0[k * V + j];
                                        const float d = f[j] - mu;
                                        mu = fmaf(d, inv, mu);
                                        acc1[k * V + j] = fmaf(d, f[j] - mu, acc1[k * V + j]);
                                    }
                                }
                            } else {
#pragma unroll
                                for (int k = 0; k < CPT; ++k) {
                                    if (!colok[k]) continue;
                                    const size_t o = (size_t)r * RBY + col[k] * 16;
                                    const uint4 vz = *reinterpret_cast<const uint4*>(base + o);
                                    const uint4 vd =
                                        *reinterpret_cast<const uint4*>(base + P.half_bytes + o);
                                    float fz[V], fd[V];
                                    Vec<DT>::unpack(vz, fz);
                                    Vec<DT>::unpack(vd, fd);
#pragma unroll
                                    for (int j = 0; j < V; ++j) {
                                        float y, dy;
                                        act_backward<ACT, DT>(fz[j], fd[j], a.p, a.inv_p, y, dy);
                                        const int q = k * V + j;
                                        acc0[q] += dy;
                                        acc1[q] = fmaf(dy, fmaf(y, kx[q], ky[q]), acc1[q]);
                                    }
                                }
                            }
                        }
                    }
                } else {
                    // NCHW: one partial per plane
                    const int np = t_nu(t) * P.g;
                    const int64_t plane0 = t_u0(t) * P.g;
                    for (int bp = 0; bp < np; bp += GP) {
                        const int pp = bp + grp;
                        const bool valid = pp < np;
                        const unsigned char* pz = base + (size_t)pp * pbytes;
                        if (DIR == 0) {
                            float sum = 0.f;
                            if (valid)
                                for (int i = glane; i < HW; i += L) sum += Elem<DT>::ld(pz, i);
                            const float mean = group_sum(sum, L) * inv_hw;
                            float sq = 0.f;
                            if (valid)
                                for (int i = glane; i < HW; i += L) {
                                    const float d = Elem<DT>::ld(pz, i) - mean;
                                    sq = fmaf(d, d, sq);
                                }
                            sq = group_sum(sq, L);
                            if (valid && glane == 0) a.part[plane0 + pp] = make_double2(mean, sq);
                        } else {
                            float s1 = 0.f, s2 = 0.f;
                            if (valid) {
                                const int c = (int)((uint64_t)(plane0 + pp) % (uint64_t)a.C);
                                const float ig = 1.f / __ldg(a.gamma + c);
                                const float nb = -__ldg(a.beta + c) * ig;
                                const unsigned char* pd = pz + P.half_bytes;
                                for (int i = glane; i < HW; i += L) {
                                    float y, dy;
                                    act_backward<ACT, DT>(Elem<DT>::ld(pz, i), Elem<DT>::ld(pd, i),
                                                          a.p, a.inv_p, y, dy);
                                    s1 += dy;
                                    s2 = fmaf(dy, fmaf(y, ig, nb), s2);
                                }
                            }
                            s1 = group_sum(s1, L);
                            s2 = group_sum(s2, L);
                            if (valid && glane == 0) a.part[plane0 + pp] = make_double2(s1, s2);
                        }
                    }
                }
            }
            if (__syncthreads_or(!ok)) {
                fail = true;
                break;
            }
        }
    }

    // ------------------------------------------- per-CTA merge (NHWC)
    if (!fail && LAYOUT == kNHWC) {
        if (CPT == 1 && RP > 1) {
            // Scratch in the ring slots (no load is in flight there now).
            float2* scr = reinterpret_cast<float2*>(slots);          // [RP][VC][V]
            float* scnt = reinterpret_cast<float*>(slots + (size_t)kResThreads * V * 8);
            if (colok[0]) {
#pragma unroll
                for (int j = 0; j < V; ++j)
                    scr[((size_t)phase * VC + col[0]) * V + j] = make_float2(acc0[j], acc1[j]);
                if (col[0] == 0) scnt[phase] = cnt;
            }
            for (int st = 1; st < RP; st <<= 1) {
                __syncthreads();
                const bool act = colok[0] && (phase % (2 * st)) == 0 && phase + st < RP;
                if (act) {
                    const int o = phase + st;
                    if (DIR == 0) {
                        const float na = cnt, nb = scnt[o], nt = na + nb;
                        if (nb > 0.f) {
                            const float f = na > 0.f ? nb / nt : 1.f;
#pragma unroll
                            for (int j = 0; j < V; ++j) {
                                const float2 q = scr[((size_t)o * VC + col[0]) * V + j];
                                const float d = q.x - acc0[j];
                                acc0[j] = fmaf(d, f, acc0[j]);
                                acc1[j] = acc1[j] + q.y + d * d * na * f;
                            }
                            cnt = nt;
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < V; ++j) {
                            const float2 q = scr[((size_t)o * VC + col[0]) * V + j];
                            acc0[j] += q.x;
                            acc1[j] += q.y;
                        }
                    }
                }
                __syncthreads();
                if (act) {
#pragma unroll
                    for (int j = 0; j < V; ++j)
                        scr[((size_t)phase * VC + col[0]) * V + j] = make_float2(acc0[j], acc1[j]);
                    if (col[0] == 0) scnt[phase] = cnt;
                }
            }
            __syncthreads();
        }
        if (phase == 0) {
#pragma unroll
            for (int k = 0; k < CPT; ++k)
                if (colok[k])
#pragma unroll
                    for (int j = 0; j < V; ++j)
                        a.part[(int64_t)b * a.C + col[k] * V + j] =
                            make_double2(acc0[k * V + j], acc1[k * V + j]);
        }
        __syncthreads();   // scratch reads done before the ring slots are reloaded
    }

    // ------------------------------------- prefetch phase B, then barriers
    // Phase B order: resident tiles n-1..nring, then ring tiles nring-1..0;
    // the j-th ring tile of phase B (tile nring-1-j) uses ring slot j % ring.
    const int depthB = max(1, ring - 2);
    if (!fail) {
        const int pro = min(depthB, nring);
        for (int j = 0; j < pro; ++j) issue(nring - 1 - j, j % ring, pol_stream);
    }
    if (!fail && !grid_barrier(a.ctl, a.budget_ns)) fail = true;

    // finalize: one warp per channel over the whole grid, fp64, fixed order
    if (!fail) {
        const int wid = tid >> 5, lane = tid & 31;
        const int64_t nw = (int64_t)G * kResWarps;
        const int64_t K = LAYOUT == kNHWC ? (int64_t)G : a.N;
        for (int64_t c = (int64_t)b * kResWarps + wid; c < a.C; c += nw) {
            if (DIR == 0) {
                double s = 0.0;
                for (int64_t k = lane; k < K; k += 32) {
                    const double cntk = LAYOUT == kNHWC
                                            ? (double)((k + 1) * P.units / G - k * P.units / G)
                                            : (double)a.HW;
                    s += cntk * a.part[k * a.C + c].x;
                }
                const double mean = warp_sum(s) / a.M;
                double q = 0.0;
                for (int64_t k = lane; k < K; k += 32) {
                    const double cntk = LAYOUT == kNHWC
                                            ? (double)((k + 1) * P.units / G - k * P.units / G)
                                            : (double)a.HW;
                    const double2 pk = a.part[k * a.C + c];
                    const double d = pk.x - mean;
                    q += pk.y + cntk * d * d;
                }
                const double var = warp_sum(q) / a.M;
                if (lane == 0) {
                    a.out0[c] = (float)mean;
                    a.out1[c] = (float)var;
                    const double rstd = 1.0 / sqrt(var + (double)a.eps);
                    a.coef[c] = make_float4((float)mean, (float)((double)a.gamma[c] * rstd),
                                            a.beta[c], 0.f);
                }
            } else {
                double s1 = 0.0, s2 = 0.0;
                for (int64_t k = lane; k < K; k += 32) {
                    const double2 pk = a.part[k * a.C + c];
                    s1 += pk.x;
                    s2 += pk.y;
                }
                s1 = warp_sum(s1);
                s2 = warp_sum(s2);
                if (lane == 0) {
                    const double gm = a.gamma[c], bt = a.beta[c];
                    const double rstd = 1.0 / sqrt((double)a.var_in[c] + (double)a.eps);
                    if (!(fabs(gm) >= 1.17549435082228750797e-38)) {   // |gamma| < FLT_MIN
                        atomicOr(&a.ctl->status, kStSingular);
                        const float qnan = __int_as_float(0x7fc00000);
                        a.out0[c] = qnan;
                        a.out1[c] = qnan;
                        a.coef[c] = make_float4(qnan, qnan, qnan, 0.f);
                    } else {
                        a.out0[c] = (float)s2;
                        a.out1[c] = (float)s1;
                        const double A = gm * rstd, B = -rstd * s2 / a.M;
                        const double Cc = -gm * rstd * s1 / a.M - B * bt;
                        a.coef[c] = make_float4((float)A, (float)B, (float)Cc, 0.f);
                    }
                }
            }
        }
    }
    if (!fail && !grid_barrier(a.ctl, a.budget_ns)) fail = true;

    // ---------------------------------------------------------- phase B
    if (!fail) {
        float c0[NV], c1[NV], c2[NV];
        if (LAYOUT == kNHWC) {
#pragma unroll
            for (int k = 0; k < CPT; ++k)
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (colok[k]) q = a.coef[col[k] * V + j];
                    c0[k * V + j] = q.x;
                    c1[k * V + j] = q.y;
                    c2[k * V + j] = q.z;
                }
        }
        // Rewrites the tile in slot s in place (forward: x -> z; backward: dz -> dx).
        auto apply_tile = [&](int t, int s) {
            unsigned char* base = slot_ptr(s);
            if (LAYOUT == kNHWC) {
                const int rows = t_nu(t);
                if (CPT == 2 || colok[0]) {
                    for (int r = phase; r < rows; r += RP) {
#pragma unroll
                        for (int k = 0; k < CPT; ++k) {
                            if (!colok[k]) continue;
                            const size_t o = (size_t)r * RBY + col[k] * 16;
                            if (DIR == 0) {
                                uint4* pv = reinterpret_cast<uint4*>(base + o);
                                float f[V];
                                Vec<DT>::unpack(*pv, f);
#pragma unroll
                                for (int j = 0; j < V; ++j) {
                                    const int q = k * V + j;
                                    f[j] = act_forward<ACT, DT>(fmaf(f[j] - c0[q], c1[q], c2[q]),
                                                                a.p);
                                }
                                *pv = Vec<DT>::pack(f);
                            } else {
                                const uint4 vz = *reinterpret_cast<const uint4*>(base + o);
                                uint4* pd = reinterpret_cast<uint4*>(base + P.half_bytes + o);
                                float fz[V], fd[V];
                                Vec<DT>::unpack(vz, fz);
                                Vec<DT>::unpack(*pd, fd);
#pragma unroll
                                for (int j = 0; j < V; ++j) {
                                    const int q = k * V + j;
                                    float y, dy;
                                    act_backward<ACT, DT>(fz[j], fd[j], a.p, a.inv_p, y, dy);
                                    fd[j] = fmaf(c0[q], dy, fmaf(c1[q], y, c2[q]));
                                }
                                *pd = Vec<DT>::pack(fd);
                            }
                        }
                    }
                }
            } else {
                const int np = t_nu(t) * P.g;
                const int64_t plane0 = t_u0(t) * P.g;
                const uint32_t cbase = (uint32_t)((uint64_t)plane0 % (uint64_t)a.C);
                for (int pp = grp; pp < np; pp += GP) {
                    const uint32_t c = (cbase + (uint32_t)pp) % (uint32_t)a.C;
                    const float4 q = __ldg(a.coef + c);
                    unsigned char* pz = base + (size_t)pp * pbytes;
                    if (DIR == 0) {
                        for (int i = glane; i < HW; i += L)
                            Elem<DT>::st(pz, i, act_forward<ACT, DT>(
                                                    fmaf(Elem<DT>::ld(pz, i) - q.x, q.y, q.z), a.p));
                    } else {
                        unsigned char* pd = pz + P.half_bytes;
                        for (int i = glane; i < HW; i += L) {
                            float y, dy;
                            act_backward<ACT, DT>(Elem<DT>::ld(pz, i), Elem<DT>::ld(pd, i), a.p,
                                                  a.inv_p, y, dy);
                            Elem<DT>::st(pd, i, fmaf(q.x, dy, fmaf(q.y, y, q.z)));
                        }
                    }
                }
            }
        };
        // Thread 0 stores the rewritten tile (after every thread's writes are
        // ordered before the bulk copy's reads).
        auto store_tile = [&](int t, int s) {
            fence_proxy_async_smem();
            __syncthreads();
            if (tid == 0) {
                const uint32_t bytes = (uint32_t)t_nu(t) * (uint32_t)P.unit_bytes;
                const int64_t off = t_u0(t) * P.unit_bytes;
                bulk_store(a.dst + off, slot_ptr(s) + (DIR == 0 ? 0 : P.half_bytes), bytes,
                           pol_stream);
                bulk_commit();
            }
        };
        for (int t = n - 1; t >= nring; --t) {
            const int s = ring + (t - nring);
            apply_tile(t, s);
            store_tile(t, s);
        }
        for (int j = 0; j < nring; ++j) {
            const int jn = j + depthB;
            if (jn < nring) {
                // the slot of ring tile jn last held ring tile jn - ring, stored
                // at least two iterations ago
                if (tid == 0) bulk_wait_read<1>();
                issue(nring - 1 - jn, jn % ring, pol_stream);
            }
            const int s = j % ring;
            const bool ok = wait(s);
            if (ok) apply_tile(nring - 1 - j, s);
            if (__syncthreads_or(!ok)) {
                fail = true;
                break;
            }
            store_tile(nring - 1 - j, s);
        }
    }

    // ----------------------------------------------------------- exit
    if (fail && tid == 0) {
        atomicOr(&a.ctl->status, kStTimeout);
        for (int s = 0; s < P.nslots; ++s)
            if (pending & (1u << s)) mbar_wait(&bars[s], (parity >> s) & 1u, a.budget_ns);
    }
    if (tid == 0) bulk_wait_all();
}

}  // namespace iabn

#include <atomic>

namespace iabn {

// Launches one instantiation cooperatively (all CTAs co-resident, which the
// grid barrier relies on).
template <int DT, int ACT, int LAYOUT, int CPT, int DIR>
cudaError_t launch_resident_one(const ResArgs& a, int smem_optin, cudaStream_t s) {
    auto kern = k_resident<DT, ACT, LAYOUT, CPT, DIR>;
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
    cfg.blockDim = dim3(kResThreads);
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

template <int DT, int LAYOUT, int CPT, int DIR>
cudaError_t launch_resident_act(const ResArgs& a, int act, int smem_optin, cudaStream_t s) {
    switch (act) {
    case kLeaky: return launch_resident_one<DT, kLeaky, LAYOUT, CPT, DIR>(a, smem_optin, s);
    case kElu: return launch_resident_one<DT, kElu, LAYOUT, CPT, DIR>(a, smem_optin, s);
    default: return launch_resident_one<DT, kIdent, LAYOUT, CPT, DIR>(a, smem_optin, s);
    }
}

template <int DT, int DIR>
cudaError_t launch_resident_dir(const ResArgs& a, int layout, int cpt, int act, int smem_optin,
                                cudaStream_t s) {
    if (layout == kNCHW) return launch_resident_act<DT, kNCHW, 1, DIR>(a, act, smem_optin, s);
    if (cpt == 1) return launch_resident_act<DT, kNHWC, 1, DIR>(a, act, smem_optin, s);
    return launch_resident_act<DT, kNHWC, 2, DIR>(a, act, smem_optin, s);
}

// Defined in iabn_resident_{f32,bf16,f16}.cu.
cudaError_t launch_resident_f32(const ResArgs& a, int layout, int cpt, int act, int dir,
                                int smem_optin, cudaStream_t s);
cudaError_t launch_resident_bf16(const ResArgs& a, int layout, int cpt, int act, int dir,
                                 int smem_optin, cudaStream_t s);
cudaError_t launch_resident_f16(const ResArgs& a, int layout, int cpt, int act, int dir,
                                int smem_optin, cudaStream_t s);

}  // namespace iabn
