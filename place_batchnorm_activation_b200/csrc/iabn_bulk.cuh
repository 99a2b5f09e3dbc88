// iabn_bulk.cuh -- thin wrappers over the sm_90+/sm_100 bulk-copy engine
// (cp.async.bulk, non-tensor form), shared-memory mbarriers with bounded
// waits, and L2 eviction-priority policies.
//
// Rules these wrappers rely on: source and destination addresses and the
// byte count of every bulk copy are multiples of 16; the expected transaction
// bytes of one mbarrier phase stay below 2^20; no copy uses cluster
// multicast.
#pragma once

#include <stdint.h>

#include "iabn_device.cuh"

namespace iabn {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

// Makes the barrier initialisation visible to the bulk-copy (async) proxy.
__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking test for completion of the phase with the given parity.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait with an explicit suspend-time hint (ns).
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity,
                                                   uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity to complete, at most budget_ns.
// mode 0: mbarrier.try_wait (the hardware may suspend the thread between
// checks); mode 1: spin on the non-blocking test_wait; mode 2: try_wait with
// a 32 ns suspend-time hint.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          unsigned long long budget_ns, int mode = 0) {
    auto probe = [&]() -> bool {
        if (mode == 1) return mbar_test_wait(bar, parity);
        if (mode == 2) return mbar_try_wait_hint(bar, parity, 32u);
        return mbar_try_wait(bar, parity);
    };
    if (probe()) return true;
    const unsigned long long t0 = global_ns();
    for (unsigned int k = 1;; ++k) {
        if (probe()) return true;
        // read the timer only every 64 polls
        if ((k & 63u) == 0 && global_ns() - t0 > budget_ns) return false;
    }
}

// 16-byte global store.
__device__ __forceinline__ void stg128(void* p, const uint4& v) {
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// 16-byte shared-memory load / store at a 32-bit shared address.
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

// (No "memory" clobber: ordering against the mbarrier arrive and the async
// proxy fence that follow comes from those volatile asm statements, and a
// clobber here would serialise every row of the tile loops.)
__device__ __forceinline__ void sts128(uint32_t addr, const uint4& v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w));
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t policy_evict_normal() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Global -> shared bulk copy completing on `bar` (transaction bytes).
__device__ __forceinline__ void bulk_load(void* dst_smem, const void* src_gmem, uint32_t bytes,
                                          uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// The same without an L2 cache hint.
__device__ __forceinline__ void bulk_load_plain(void* dst_smem, const void* src_gmem,
                                                uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void bulk_store_plain(void* dst_gmem, const void* src_smem,
                                                 uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 ::"l"(dst_gmem), "r"(smem_u32(src_smem)), "r"(bytes)
                 : "memory");
}

// Shared -> global bulk copy, tracked by the issuing thread's bulk groups.
__device__ __forceinline__ void bulk_store(void* dst_gmem, const void* src_smem, uint32_t bytes,
                                           uint64_t policy) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group.L2::cache_hint [%0], [%1], %2, %3;"
                 ::"l"(dst_gmem), "r"(smem_u32(src_smem)), "r"(bytes), "l"(policy)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Asynchronous 4-byte global -> shared copy (no register staging, so the
// issuing thread does not stall on the load); cp_async_wait_all() makes the
// issuing thread's copies visible to it.
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src)
                 : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// Waits until at most N committed store groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Waits until all committed store groups have completed.
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later
// bulk-copy (async-proxy) reads of the same bytes.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------ 16-byte vector packing

template <int DT> struct Vec;
template <> struct Vec<kF32> {
    static constexpr int N = 4;
    static __device__ __forceinline__ void unpack(const uint4& v, float* f) {
        f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
    }
    static __device__ __forceinline__ uint4 pack(const float* f) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                          __float_as_uint(f[3]));
    }
};
template <> struct Vec<kBF16> {
    static constexpr int N = 8;
    static __device__ __forceinline__ void unpack2(uint32_t w, float& lo, float& hi) {
        lo = __uint_as_float(w << 16);
        hi = __uint_as_float(w & 0xffff0000u);
    }
    static __device__ __forceinline__ void unpack(const uint4& v, float* f) {
        unpack2(v.x, f[0], f[1]); unpack2(v.y, f[2], f[3]);
        unpack2(v.z, f[4], f[5]); unpack2(v.w, f[6], f[7]);
    }
    static __device__ __forceinline__ uint32_t pack2(float lo, float hi) {
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    static __device__ __forceinline__ uint4 pack(const float* f) {
        return make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]),
                          pack2(f[6], f[7]));
    }
};
template <> struct Vec<kF16> {
    static constexpr int N = 8;
    static __device__ __forceinline__ void unpack2(uint32_t w, float& lo, float& hi) {
        __half2 h = *reinterpret_cast<__half2*>(&w);
        float2 f = __half22float2(h);
        lo = f.x;
        hi = f.y;
    }
    static __device__ __forceinline__ void unpack(const uint4& v, float* f) {
        unpack2(v.x, f[0], f[1]); unpack2(v.y, f[2], f[3]);
        unpack2(v.z, f[4], f[5]); unpack2(v.w, f[6], f[7]);
    }
    static __device__ __forceinline__ uint32_t pack2(float lo, float hi) {
        __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    static __device__ __forceinline__ uint4 pack(const float* f) {
        return make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]),
                          pack2(f[6], f[7]));
    }
};

// Scalar shared-memory element access (NCHW planes need not be 4-byte aligned).
template <int DT> struct Elem;
template <> struct Elem<kF32> {
    static __device__ __forceinline__ float ld(const unsigned char* base, int i) {
        return reinterpret_cast<const float*>(base)[i];
    }
    static __device__ __forceinline__ void st(unsigned char* base, int i, float v) {
        reinterpret_cast<float*>(base)[i] = v;
    }
};
template <> struct Elem<kBF16> {
    static __device__ __forceinline__ float ld(const unsigned char* base, int i) {
        return __uint_as_float((uint32_t)reinterpret_cast<const unsigned short*>(base)[i] << 16);
    }
    static __device__ __forceinline__ void st(unsigned char* base, int i, float v) {
        reinterpret_cast<unsigned short*>(base)[i] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
};
template <> struct Elem<kF16> {
    static __device__ __forceinline__ float ld(const unsigned char* base, int i) {
        return __half2float(__ushort_as_half(reinterpret_cast<const unsigned short*>(base)[i]));
    }
    static __device__ __forceinline__ void st(unsigned char* base, int i, float v) {
        reinterpret_cast<unsigned short*>(base)[i] = __half_as_ushort(__float2half_rn(v));
    }
};

}  // namespace iabn
