// bulk.cuh -- bulk copies (the TMA engine, no tensor map) between global
// memory and this CTA's shared memory, and the mbarrier that tracks them.
//
// A load arms the barrier with the bytes it will deliver (expect_tx) and the
// copy completes that phase when they have landed. Every wait is bounded: it
// polls the barrier against %globaltimer and gives up after `limit_ns`
// (2 s unless the caller says otherwise), so a copy that never completes ends
// in a status the caller reports, never in a hung GPU. Addresses and sizes
// are multiples of 16 bytes. tests/mbar_timeout.cu runs these helpers: a copy
// that completes, and a phase armed for bytes that never arrive.
#pragma once

#include <cstdint>

namespace epb {

constexpr uint64_t kWaitLimitNs = 2000000000ull; // a bounded wait gives up after 2 s

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// a barrier with one expected arrival per phase
__device__ __forceinline__ void mbar_init(uint64_t *bar) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(bar)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// arrive on the barrier and arm its current phase for `bytes` of copies
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// arm the barrier for `bytes` and start the load of global [src, src+bytes)
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    mbar_expect_tx(bar, bytes);
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok)
                 : "r"(smem_u32(bar)), "r"(parity)
                 : "memory");
    return ok != 0;
}

// wait for phase `parity` of the barrier to complete, for at most limit_ns;
// false if it gave up
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_test(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_test(bar, parity))
        if (global_ns() - t0 > limit_ns) return false;
    return true;
}

// an L2 policy that marks lines evict-first (streamed output, as st.global.cs)
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void bulk_store(void *dst, const void *src, uint32_t bytes, uint64_t pol) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group.L2::cache_hint [%0], [%1], %2, %3;" ::"l"(dst),
                 "r"(smem_u32(src)), "r"(bytes), "l"(pol)
                 : "memory");
}

// every bulk store issued so far has finished reading shared memory
__device__ __forceinline__ void bulk_stores_read() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

} // namespace epb
