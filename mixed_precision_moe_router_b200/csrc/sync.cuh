// mbarrier, bulk-copy and bounded-wait helpers (sm_100a inline PTX).
//
// Every wait here is bounded: after `limit` SM clock cycles it gives up and
// returns false, and the caller records MOE_STATUS_TIMEOUT and stops, so a
// lost signal ends the kernel with an error instead of hanging the GPU.
#pragma once
#include "common.cuh"

namespace moe {

constexpr long long kWaitLimitCycles = 2000000000LL;  // ~1 s at the B200 SM clock

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// try_wait with a suspend-time hint: the waiting thread sleeps in hardware
// until the phase completes or about 1 ms passes, instead of spinning and
// taking issue slots from the warps doing the work.
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(1000000u)
        : "memory");
    return ok != 0;
}

// try_wait with a caller-chosen suspend-time hint in nanoseconds.
__device__ __forceinline__ bool mbar_try_wait_ns(uint64_t *bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity; false once *abort is set (by
// another warp of the CTA giving up) or after `limit` SM clock cycles.
__device__ __forceinline__ bool mbar_wait_abortable(uint64_t *bar, uint32_t parity, const volatile int *abort,
                                                    long long limit) {
    if (mbar_try_wait_ns(bar, parity, 20000u)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait_ns(bar, parity, 20000u)) {
        if (*abort || clock64() - t0 > limit) return false;
    }
    return true;
}

// Warp-wide wait for the phase with the given parity: lane 0 polls (with the
// abort flag and the cycle limit of mbar_wait_abortable), then every lane
// confirms with one try_wait of its own (which acquires the phase; it cannot
// have moved on, since advancing it takes an action of this warp).  Returns the
// same result in every lane.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t *bar, uint32_t parity, const volatile int *abort,
                                               long long limit) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait_abortable(bar, parity, abort, limit);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok) mbar_try_wait_ns(bar, parity, 0u);
    return ok;
}

// Wait for the phase with the given parity; false after `limit` cycles.
__device__ __forceinline__ bool mbar_wait_limit(uint64_t *bar, uint32_t parity, long long limit) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > limit) return false;
    }
    return true;
}

// Wait until the phase with the given parity has completed; false on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > kWaitLimitCycles) return false;
    }
    return true;
}

// 1-D bulk copy global -> shared, completing `bytes` of transaction on `bar`.
// dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Asynchronous global -> shared copies of 4 and 16 bytes (cp.async), waited
// for with cp_async_wait_all.
__device__ __forceinline__ void cp_async_4b(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_16b(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Bulk prefetch of [src, src + bytes) into L2 (16-byte aligned, multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void *src, uint32_t bytes) {
    if (bytes) asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Spin until *ctr >= target (acquire), sleeping 32 ns, 64 ns, ... up to 1 us
// between polls; false on timeout.
__device__ __forceinline__ bool wait_geq_backoff(const int *ctr, int target) {
    if (ld_acquire(ctr) >= target) return true;
    const long long t0 = clock64();
    unsigned ns = 32;
    while (ld_acquire(ctr) < target) {
        if (clock64() - t0 > kWaitLimitCycles) return false;
        __nanosleep(ns);
        if (ns < 1024) ns *= 2;
    }
    return true;
}

// Spin until *ctr >= target (acquire); false once *abort is set or after
// `limit` cycles.  The polling thread has nothing else to do, so it polls at
// the L2 round-trip rate with a short pause: a longer backoff would add its
// own length to the dependency it waits for.
__device__ __forceinline__ bool wait_geq_abortable(const int *ctr, int target, const volatile int *abort,
                                                   long long limit) {
    if (ld_acquire(ctr) >= target) return true;
    const long long t0 = clock64();
    while (ld_acquire(ctr) < target) {
        if (*abort || clock64() - t0 > limit) return false;
        __nanosleep(32);
    }
    return true;
}

// Grid-wide barrier, called by thread 0 of every CTA with the CTA synchronised
// before and after.  `bar` counts arrivals over the launch (zero at launch,
// never reset), so barrier number n (0, 1, ...) is passed once it reaches
// (n + 1) * grid.  The arrival is a release add, which orders the writes the
// CTA made before the barrier; the wait polls with acquire loads, bounded and
// abortable.  Returns false when the wait gave up.
__device__ __forceinline__ bool grid_barrier(int *bar, int n, const volatile int *abort, long long limit) {
    const int target = (n + 1) * static_cast<int>(gridDim.x * gridDim.y * gridDim.z);
    asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(bar) : "memory");
    if (ld_acquire(bar) >= target) return true;
    const long long t0 = clock64();
    while (ld_acquire(bar) < target)
        if (*abort || clock64() - t0 > limit) return false;
    return true;
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

}  // namespace moe
