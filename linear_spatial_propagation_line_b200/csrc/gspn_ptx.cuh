// Thin wrappers over the sm_90+/sm_100a PTX used by the fused kernel:
// mbarriers, TMA tensor loads, DSMEM stores with transaction completion,
// cluster barriers, L2 cache policies, vector reductions and the global timer.
// Every wait here is bounded by the caller (see wait_parity_bounded).
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace gspn {
namespace ptx {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---- cluster ---------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Address of the same shared variable in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void st_cluster_s32(uint32_t addr, int v) {
    asm volatile("st.shared::cluster.s32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
// 4-byte DSMEM store that completes 4 transaction bytes on the remote mbarrier.
__device__ __forceinline__ void st_async_f32(uint32_t remote_addr, float v, uint32_t remote_bar) {
    asm volatile(
        "st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(
            remote_addr),
        "r"(__float_as_uint(v)), "r"(remote_bar)
        : "memory");
}

// ---- mbarrier ----------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Waits for phase `parity` of `bar`; gives up after `limit_ns` and returns false.
__device__ __forceinline__ bool wait_parity_bounded(uint32_t bar, uint32_t parity,
                                                    uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (global_timer_ns() - t0 > limit_ns) return false;
    }
}

// ---- L2 cache policies ---------------------------------------------------------
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

// ---- TMA -------------------------------------------------------------------------
// 3-D tiled tensor load into this CTA's shared memory; completion is counted in
// bytes on `bar`.  No multicast.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, uint32_t bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar), "l"(policy)
        : "memory");
}
__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---- global reductions / stores with cache hints -----------------------------------
__device__ __forceinline__ void red_add_f32(float* addr, float v, uint64_t policy) {
    asm volatile("red.relaxed.gpu.global.add.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(addr), "f"(v),
                 "l"(policy)
                 : "memory");
}
__device__ __forceinline__ void red_add_v4_f32(float* addr, float a, float b, float c, float d) {
    asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a),
                 "f"(b), "f"(c), "f"(d)
                 : "memory");
}
__device__ __forceinline__ int atom_add_acq_rel_gpu(int* addr, int v) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(v)
                 : "memory");
    return old;
}
__device__ __forceinline__ int ld_acquire_gpu(const int* addr) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(addr) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_gpu(int* addr, int v) {
    asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(addr), "r"(v) : "memory");
}

// 8-byte DSMEM store (two floats) completing 8 transaction bytes remotely.
__device__ __forceinline__ void st_async_f32x2(uint32_t remote_addr, float a, float b,
                                               uint32_t remote_bar) {
    asm volatile(
        "st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(
            remote_addr),
        "f"(a), "f"(b), "r"(remote_bar)
        : "memory");
}
__device__ __forceinline__ void red_add_v2_f32(float* addr, float a, float b, uint64_t policy) {
    asm volatile("red.relaxed.gpu.global.add.L2::cache_hint.v2.f32 [%0], {%1, %2}, %3;" ::"l"(addr),
                 "f"(a), "f"(b), "l"(policy)
                 : "memory");
}
__device__ __forceinline__ void red_add_v4_f32_hint(float* addr, float a, float b, float c,
                                                    float d, uint64_t policy) {
    asm volatile(
        "red.relaxed.gpu.global.add.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(addr),
        "f"(a), "f"(b), "f"(c), "f"(d), "l"(policy)
        : "memory");
}
// Predicated forms: the instruction is skipped (no branch) when `on` is 0.
__device__ __forceinline__ void red_add_v2_f32_if(bool on, float* addr, float a, float b,
                                                  uint64_t policy) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %0, 0;\n\t"
        "@p red.relaxed.gpu.global.add.L2::cache_hint.v2.f32 [%1], {%2, %3}, %4;\n\t}" ::"r"(
            (uint32_t)on),
        "l"(addr), "f"(a), "f"(b), "l"(policy)
        : "memory");
}
__device__ __forceinline__ void red_add_v4_f32_if(bool on, float* addr, float a, float b, float c,
                                                  float d, uint64_t policy) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %0, 0;\n\t"
        "@p red.relaxed.gpu.global.add.L2::cache_hint.v4.f32 [%1], {%2, %3, %4, %5}, %6;\n\t}" ::"r"(
            (uint32_t)on),
        "l"(addr), "f"(a), "f"(b), "f"(c), "f"(d), "l"(policy)
        : "memory");
}
__device__ __forceinline__ void sts_f32_if(bool on, uint32_t a, float v) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %0, 0;\n\t@p st.shared.f32 [%1], %2;\n\t}" ::"r"(
            (uint32_t)on),
        "r"(a), "f"(v)
        : "memory");
}
// Plain arrive (count 1) on a CTA-local mbarrier, release semantics.
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// Waits (CTA scope) for phase `parity`; gives up after `limit_ns`.
__device__ __forceinline__ bool mbar_try_wait_cta(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool wait_parity_cta_bounded(uint32_t bar, uint32_t parity,
                                                        uint64_t limit_ns) {
    if (mbar_try_wait_cta(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait_cta(bar, parity)) return true;
        if (global_timer_ns() - t0 > limit_ns) return false;
    }
}
// 3-D tiled tensor load with the default (evict_normal) L2 policy.
__device__ __forceinline__ void tma_load_3d_normal(uint32_t dst, const CUtensorMap* map, int c0,
                                                   int c1, int c2, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
        : "memory");
}
// Explicit shared-memory accesses (32-bit shared addresses).  Volatile so they
// stay ordered with the barriers around them.
__device__ __forceinline__ float lds_f32(uint32_t a) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t lds_u16(uint32_t a) {
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ uint4 lds_v4(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(a)
                 : "memory");
    return v;
}
__device__ __forceinline__ uint2 lds_v2(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ void sts_v2_f32(uint32_t a, float x, float y) {
    asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(a), "f"(x), "f"(y) : "memory");
}
__device__ __forceinline__ void sts_f32(uint32_t a, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}
// 16-byte shared store of four floats.
__device__ __forceinline__ void sts_v4_f32(uint32_t a, float x, float y, float z, float w) {
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(x), "f"(y), "f"(z),
                 "f"(w)
                 : "memory");
}
// Predicated 8-byte shared store (skipped, no branch, when `on` is 0).
__device__ __forceinline__ void sts_v2_f32_if(bool on, uint32_t a, float x, float y) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %0, 0;\n\t"
        "@p st.shared.v2.f32 [%1], {%2, %3};\n\t}" ::"r"((uint32_t)on),
        "r"(a), "f"(x), "f"(y)
        : "memory");
}
// Predicated 16-byte shared store (skipped, no branch, when `on` is 0).
__device__ __forceinline__ void sts_v4_f32_if(bool on, uint32_t a, float x, float y, float z,
                                              float w) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %0, 0;\n\t"
        "@p st.shared.v4.f32 [%1], {%2, %3, %4, %5};\n\t}" ::"r"((uint32_t)on),
        "r"(a), "f"(x), "f"(y), "f"(z), "f"(w)
        : "memory");
}
// Named barrier over the first `count` threads of the CTA (count % 32 == 0).
__device__ __forceinline__ void named_barrier(uint32_t id, uint32_t count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ---- packed fp32 pairs (sm_100 f32x2 arithmetic) -------------------------------
// a if c else b, without a branch.
__device__ __forceinline__ unsigned long long sel64(bool c, unsigned long long a,
                                                    unsigned long long b) {
    unsigned long long r;
    asm("{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %3, 0;\n\tselp.b64 %0, %1, %2, p;\n\t}"
        : "=l"(r)
        : "l"(a), "l"(b), "r"((uint32_t)c));
    return r;
}
// A pair holds position A in the low half and position B in the high half.
typedef unsigned long long f2;
__device__ __forceinline__ f2 pk(float a, float b) {
    f2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void upk(f2 v, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c) {
    f2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ f2 mul2(f2 a, f2 b) {
    f2 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f2 add2(f2 a, f2 b) {
    f2 d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

}  // namespace ptx
}  // namespace gspn
