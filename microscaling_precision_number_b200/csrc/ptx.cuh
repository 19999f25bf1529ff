// ptx.cuh -- thin inline-PTX wrappers for sm_100a: mbarriers, TMA bulk-tensor loads,
// fences, and a wall-clock-bounded barrier wait (the watchdog).
#pragma once
#include <cstdint>

namespace mxk {

// Bounded waits give up after this many nanoseconds of %globaltimer time, record a
// code in the watchdog flag and let the kernel unwind.  No wait in this library can
// spin forever.
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s

// Watchdog codes (what timed out).
enum : int { WD_DUAL_FULL = 1, WD_GEMM_FULL = 2, WD_GEMM_EMPTY = 3, WD_GEMM_ACC = 4, WD_GEMM_DRAIN = 5,
             WD_STREAM_FULL = 6, WD_STREAM_EMPTY = 7, WD_DUAL_EMPTY = 8, WD_SELFTEST = 9 };

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar_addr, uint32_t phase) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar_addr), "r"(phase)
        : "memory");
    return done != 0;
}

// Wait until the barrier's phase with parity `phase` has completed.  Returns false (and
// records `code` in *watchdog) if that does not happen within `limit_ns`.  While waiting
// it also polls the watchdog flag: once any CTA has given up, every other waiter returns
// false at once instead of spending its own full limit.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t phase, int *watchdog, int code,
                                                  uint64_t limit_ns = kWaitLimitNs) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, phase)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; i++) {
        if (mbar_try_wait(a, phase)) return true;
        if ((i & 255u) == 0u) {
            if (watchdog && *reinterpret_cast<volatile int *>(watchdog) != 0) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                if (watchdog) atomicExch(watchdog, code);
                return false;
            }
        }
    }
}

// ---- warp-uniform issue ---------------------------------------------------------------------
// The issuing warps of the matmuls (and the dual quantiser's producer) run their loops with all 32 lanes converged and let one
// elected lane issue each group of tcgen05 / TMA instructions.  Measured on B200: a
// tcgen05.mma stream issued this way sustains one M = 256 x N = 256 x K = 32 pair MMA per
// 128 cycles (the tensor pipe's rate), whereas the same loop run by lane 0 alone inside a
// divergent branch issued one per ~560 cycles.
__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}" : "=r"(pred));
    return pred != 0;
}
// Bounded wait by a whole warp; true only if every lane saw the phase complete.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t phase, int *watchdog, int code) {
    const bool ok = mbar_wait_bounded(bar, phase, watchdog, code);
    return __all_sync(0xffffffffu, ok);
}
// A shared failure flag read uniformly by a warp.
__device__ __forceinline__ bool warp_failed(volatile int *flag) { return __any_sync(0xffffffffu, *flag != 0); }

// Short limit for error-path drains of a CTA's own in-flight copies.
constexpr uint64_t kDrainLimitNs = 20000000ull;   // 20 ms

// 2-D tiled TMA load of a box at element coordinates (x = innermost, y) into shared
// memory, completing `bytes` on the barrier (armed separately with expect_tx).
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const void *tmap, int32_t x, int32_t y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Plain (untiled) bulk copy global -> shared of `bytes` (multiple of 16, both 16-byte aligned).
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gsrc, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(smem_dst)), "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const void *tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

}  // namespace mxk
