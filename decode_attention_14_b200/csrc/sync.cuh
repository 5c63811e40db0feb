// sync.cuh -- shared-memory barriers with bounded waits, used by the kernels
// whose warps hand work to one another through mbarriers.
#pragma once

#include <stdint.h>

#ifndef RQ_WAIT_NS
#define RQ_WAIT_NS 1000000000ull
#endif
#ifndef RQ_POLLS_PER_CHECK
#define RQ_POLLS_PER_CHECK 4
#endif

namespace rq {

constexpr unsigned long long kWaitNs = RQ_WAIT_NS;   // limit of one wait (1 s by default)

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
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
// Non-blocking test of an mbarrier phase.
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
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
__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Bounded wait on an mbarrier phase; gives up after kWaitNs or as soon as
// another warp of the CTA has given up.  SLEEP_NS > 0 backs off between
// polls (for waits whose latency does not matter).  The abort flag and the
// clock are checked once per RQ_POLLS_PER_CHECK polls: a poll is two
// instructions, the checks several more, and waiting warps share the
// schedulers with working ones.
template <unsigned SLEEP_NS = 0>
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (;;) {
#pragma unroll
        for (int i = 0; i < RQ_POLLS_PER_CHECK; i++) {
            if (SLEEP_NS) __nanosleep(SLEEP_NS);
            if (mbar_try_wait(bar, parity)) return true;
        }
        if (*abort_flag) return false;
        if (global_ns() - t0 > kWaitNs) return false;
    }
}

}  // namespace rq
