// stream.cuh -- asynchronous-copy plumbing shared by the kernels: mbarriers
// with bounded waits, TMA bulk copies global -> shared, contiguous unit
// ranges and the acquire-release publish of finished units.
//
// Every wait is bounded; a wait that runs out sets this file's error flag
// (read by dflash2_device_errors) and the kernel returns after a bounded wait
// for its own copies in flight.
#pragma once

#include <mutex>

#include "common.cuh"

namespace dfl {

// One flag word per translation unit (internal linkage), read on the host by
// that file's dfl_errors_* helper.
static __device__ unsigned int g_dev_err;

enum : unsigned {
    ERR_PRODUCER = 1u,
    ERR_MMA = 2u,
    ERR_EPILOGUE = 4u,
    ERR_DRAIN = 8u,
    ERR_STREAM = 16u,
    ERR_INPUT = 32u  // a token id outside [0, V): treated as described at the call, no load
};

constexpr uint64_t WAIT_NS = 1000000000ull;  // bound on any single wait: 1 s

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// Wait for the phase with the given parity to complete; false after WAIT_NS.
// Each try_wait carries a suspend-time hint, so a waiting warp sleeps in the
// barrier until the phase completes (or the hint runs out) instead of
// spinning through issue slots the computing warps need; the clock is read
// once per try.
constexpr uint32_t SUSPEND_NS = 20000;
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity), "r"(SUSPEND_NS)
        : "memory");
    return done != 0;
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    if (mbar_try(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        if (mbar_try(bar, parity)) return true;
        if (global_ns() - t0 > WAIT_NS) return false;
    }
}
// The same wait without the suspend hint: test_wait (which never suspends)
// polled with a short sleep, for a copy issued just before the wait (there
// the hint's suspension can outlast the copy by far); false after WAIT_NS.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}
__device__ __forceinline__ bool mbar_wait_poll(uint32_t bar, uint32_t parity) {
    if (mbar_test(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        __nanosleep(64);
        if (mbar_test(bar, parity)) return true;
        if (global_ns() - t0 > WAIT_NS) return false;
    }
}

// Bulk copy of `bytes` (a multiple of 16; both addresses 16-byte aligned)
// from global to shared memory, completing on `bar` (which expects them).
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
    mbar_expect_tx(bar, bytes);
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// The same copy on a barrier whose transaction count the caller already
// raised (one expect_tx covering several copies).
__device__ __forceinline__ void bulk_g2s_nx(uint32_t dst, const void* src, uint32_t bytes,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Contiguous share [lo, hi) of `units` for this CTA (consecutive units of a
// row / sequence mostly stay on one CTA, so it publishes them together).
__device__ __forceinline__ void cta_range(int64_t units, int64_t& lo, int64_t& hi) {
    lo = units * (int64_t)blockIdx.x / gridDim.x;
    hi = units * (int64_t)(blockIdx.x + 1) / gridDim.x;
}

// Prefetch the line holding p into L2, to be kept over streamed data.
__device__ __forceinline__ void prefetch_l2_last(const void* p) {
    asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(p));
}

// Acquire load / release store of a flag word (gpu scope).
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(unsigned* p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned ld_relaxed(const unsigned* p) {
    unsigned v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// Wait until *p is non-zero and return it (read once more with acquire
// semantics); 0 after WAIT_NS.  The poll is a relaxed load (cheap for the
// SM's caches) that backs off from 64 to 256 ns.
__device__ __forceinline__ unsigned wait_nonzero(const unsigned* p) {
    unsigned v = ld_acquire(p);
    if (v) return v;
    const uint64_t t0 = global_ns();
    unsigned ns = 64;
    while (true) {
        __nanosleep(ns);
        if (ns < 256) ns <<= 1;
        if (ld_relaxed(p)) return ld_acquire(p);
        if (global_ns() - t0 > WAIT_NS) return 0u;
    }
}

// Publish `count` units of group g whose partials this thread (thread 0) has
// already stored, with one acquire-release add: the release orders those
// stores before the count, the acquire lets the last publisher read every
// other CTA's partials.  Returns true on the publisher that completes the
// group (expected units in all).
__device__ __forceinline__ bool publish(unsigned* counter, unsigned count, unsigned expected) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;"
                 : "=r"(old)
                 : "l"(counter), "r"(count)
                 : "memory");
    return old + count == expected;
}

}  // namespace dfl
