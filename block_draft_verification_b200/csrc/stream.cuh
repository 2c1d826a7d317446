// stream.cuh -- asynchronous-copy plumbing shared by the kernels: mbarriers
// with bounded waits, TMA bulk copies global -> shared, and the chunk views
// the streaming kernels reduce from.
//
// Streaming kernels are persistent: a CTA walks its units u = blockIdx.x,
// blockIdx.x + gridDim.x, ...; one thread issues the bulk copy of the next
// unit's chunk into the other half of a two-slot shared-memory ring before
// the block reduces the current one, so HBM keeps streaming while the block
// merges and sorts.  Every wait is bounded; a wait that runs out sets this
// file's error flag (read by dflash2_device_errors) and the kernel returns
// after a bounded wait for its own copies in flight.
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
    ERR_STREAM = 16u
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
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = global_ns();
    while (true) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(bar), "r"(parity)
            : "memory");
        if (done) return true;
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

// ---------------------------------------------------------------------------
// Chunk views.  A thread's share of a chunk is NV 16-byte vectors, vector i at
// element v0 + (i * NT + t) * VW (see Row in common.cuh).  Elements at or past
// vend read as -inf.
template <bool BF16>
struct SmemChunk {  // the chunk sits in shared memory (TMA ring slot); its
                    // length is a whole number of 16-byte vectors
    using R = Row<BF16>;
    const uint8_t* buf;
    int64_t v0;
    int nvec;  // valid vectors in the chunk
    __device__ __forceinline__ SmemChunk(const uint8_t* b, int64_t v0_, int64_t vend_)
        : buf(b), v0(v0_), nvec((int)((vend_ - v0_) / R::VW)) {}
    __device__ __forceinline__ uint4 vec(int i) const {
        const int idx = i * NT + (int)threadIdx.x;
        if (idx < nvec) return *(const uint4*)(buf + idx * 16);
        return make_uint4(R::NEG_INF_WORD, R::NEG_INF_WORD, R::NEG_INF_WORD, R::NEG_INF_WORD);
    }
    __device__ __forceinline__ int64_t index_of(int i, int e) const {
        return v0 + (int64_t)(i * NT + (int)threadIdx.x) * R::VW + e;
    }
};
template <bool BF16>
struct RegChunk {  // the chunk is read element by element into registers
    using R = Row<BF16>;
    uint4 r[R::NV];
    int64_t v0, vend;
    __device__ __forceinline__ void load(const void* row, int64_t v0_, int64_t vend_) {
        v0 = v0_;
        vend = vend_;
        R::template load<false>(row, v0, vend, r);
    }
    __device__ __forceinline__ uint4 vec(int i) const { return r[i]; }
    __device__ __forceinline__ int64_t index_of(int i, int e) const {
        return v0 + (int64_t)(i * NT + (int)threadIdx.x) * R::VW + e;
    }
};

// Thread max and sum-exp over a chunk view (two passes; pairwise per vector).
template <bool BF16, class C>
__device__ __forceinline__ Lse view_lse(const C& ch, float c) {
    using R = Row<BF16>;
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < R::NV; ++i) {
        const uint4 v = ch.vec(i);
#pragma unroll
        for (int e = 0; e < R::VW; ++e) m = fmaxf(m, R::elem(v, e));
    }
    if (m == -INFINITY) return {m, 0.0f};
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < R::NV; ++i) {
        const uint4 v = ch.vec(i);
        float tt[R::VW];
#pragma unroll
        for (int e = 0; e < R::VW; ++e) tt[e] = ex2((R::elem(v, e) - m) * c);
#pragma unroll
        for (int w = R::VW / 2; w > 0; w >>= 1)
#pragma unroll
            for (int e = 0; e < w; ++e) tt[e] += tt[e + w];
        s += tt[0];
    }
    return {m, s};
}
// Same, with an fp64 running sum of the per-vector sums.
template <bool BF16, class C>
__device__ __forceinline__ LseD view_lse_d(const C& ch, float c) {
    using R = Row<BF16>;
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < R::NV; ++i) {
        const uint4 v = ch.vec(i);
#pragma unroll
        for (int e = 0; e < R::VW; ++e) m = fmaxf(m, R::elem(v, e));
    }
    if (m == -INFINITY) return {m, 0.0f, 0.0};
    double s = 0.0;
#pragma unroll
    for (int i = 0; i < R::NV; ++i) {
        const uint4 v = ch.vec(i);
        float tt[R::VW];
#pragma unroll
        for (int e = 0; e < R::VW; ++e) tt[e] = ex2((R::elem(v, e) - m) * c);
#pragma unroll
        for (int w = R::VW / 2; w > 0; w >>= 1)
#pragma unroll
            for (int e = 0; e < w; ++e) tt[e] += tt[e + w];
        s += (double)tt[0];
    }
    return {m, 0.0f, s};
}
// Thread max of a chunk view.
template <bool BF16, class C>
__device__ __forceinline__ float view_max(const C& ch) {
    using R = Row<BF16>;
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < R::NV; ++i) m = fmaxf(m, vec_max<BF16>(ch.vec(i)));
    return m;
}
// Lowest index of this thread's elements equal to x (0xFFFFFFFF if none).
template <bool BF16, class C>
__device__ __forceinline__ uint32_t view_first(const C& ch, float x) {
    using R = Row<BF16>;
    uint32_t first = 0xFFFFFFFFu;
#pragma unroll
    for (int i = R::NV - 1; i >= 0; --i) {
        const uint4 v = ch.vec(i);
#pragma unroll
        for (int e = R::VW - 1; e >= 0; --e)
            if (R::elem(v, e) == x) first = (uint32_t)ch.index_of(i, e);
    }
    return first;
}

// Contiguous share [lo, hi) of `units` for this CTA (consecutive units of a
// row / sequence mostly stay on one CTA, so it publishes them together).
__device__ __forceinline__ void cta_range(int64_t units, int64_t& lo, int64_t& hi) {
    lo = units * (int64_t)blockIdx.x / gridDim.x;
    hi = units * (int64_t)(blockIdx.x + 1) / gridDim.x;
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

// Persistent grid size for a kernel: resident CTAs per SM x SMs, at most
// units.  The occupancy query runs once per (kernel, device, smem) and is
// cached.
template <class Kernel>
inline int persistent_grid(Kernel k, int threads, size_t dyn_smem, int64_t units) {
    struct Entry {
        const void* fn;
        int dev;
        size_t smem;
        int ctas;
    };
    static Entry cache[64];
    static int n_cache = 0;
    static std::mutex mu;
    int dev = 0;
    cudaGetDevice(&dev);
    int ctas = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < n_cache; ++i)
            if (cache[i].fn == (const void*)k && cache[i].dev == dev && cache[i].smem == dyn_smem)
                ctas = cache[i].ctas;
        if (ctas == 0) {
            int sms = 148, per_sm = 1;
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, threads, dyn_smem) !=
                    cudaSuccess ||
                per_sm < 1)
                per_sm = 1;
            ctas = sms * per_sm;
            if (n_cache < 64) cache[n_cache++] = Entry{(const void*)k, dev, dyn_smem, ctas};
        }
    }
    return (int)(units < ctas ? units : ctas);
}

}  // namespace dfl
