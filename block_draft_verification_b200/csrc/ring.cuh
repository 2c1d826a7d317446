// ring.cuh -- persistent streaming of vocabulary rows: every warp keeps its
// own two-slot ring of TMA bulk copies in flight and reduces whole chunks on
// its own.
//
// A unit is one chunk of a row: SLOT_BYTES of logits (4096 bf16 or 2048 fp32
// elements; the last chunk of a row is shorter).  The chunk length depends on
// the dtype only, never on the batch, the grid or the device, and every chunk
// is reduced by one warp in a fixed order, so a chunk's partial result is the
// same bits whatever batch its row sits in.
//
// One CTA per SM takes a contiguous range of units, and each of its NCW
// warps a contiguous part of that range (consecutive chunks of a row mostly
// stay with one warp).  A warp owns two ring slots and brings its own units
// in: its lane 0 issues the bulk copy of unit k + 2 into the slot unit k
// leaves, so the next unit is in flight while the warp reduces the current
// one, and a warp that stops to merge a finished row delays nobody else.
// No block-wide barrier is taken after the set-up, and every wait is bounded
// (stream.cuh).
#pragma once

#include "stream.cuh"

namespace dfl {

constexpr int SLOT_BYTES = 8192;                   // one chunk
constexpr int NCW = 12;                            // warps per CTA
constexpr int RING_THREADS = 32 * NCW;
constexpr int RING_BYTES = 2 * NCW * SLOT_BYTES;   // 192 KB of dynamic shared memory
constexpr int NVL = SLOT_BYTES / 16 / 32;          // 16-byte vectors per lane of a chunk: 16

// Chunk length in elements for an element size, and chunks per row.
__host__ __device__ constexpr int chunk_len(int es) { return SLOT_BYTES / es; }
__host__ __device__ inline int64_t row_chunks(int64_t V, int es) {
    return (V + chunk_len(es) - 1) / chunk_len(es);
}

// This warp's contiguous share [lo, hi) of the CTA's units.
__device__ __forceinline__ void warp_range(int64_t units, int64_t& lo, int64_t& hi) {
    int64_t clo, chi;
    cta_range(units, clo, chi);
    const int64_t n = chi - clo;
    const int w = threadIdx.x >> 5;
    lo = clo + n * w / NCW;
    hi = clo + n * (w + 1) / NCW;
}

// Position of a unit in (group, row of the group, chunk of the row), with R
// rows of S chunks per group; the divisions happen once, in init, and the
// units of a range are then walked with next().
struct UnitCursor {
    int64_t g;  // group (a sequence, or a row when R = 1)
    int r;      // row within the group
    int c;      // chunk within the row
    int S, R;
    __device__ __forceinline__ void init(int64_t u, int S_, int R_) {
        S = S_;
        R = R_;
        const int64_t per = (int64_t)S * R;
        g = u / per;
        const int rem = (int)(u - g * per);
        r = rem / S;
        c = rem - r * S;
    }
    __device__ __forceinline__ void next() {
        if (++c == S) {
            c = 0;
            if (++r == R) {
                r = 0;
                ++g;
            }
        }
    }
    __device__ __forceinline__ bool last_of_row() const { return c == S - 1; }
    __device__ __forceinline__ bool last_of_group() const { return c == S - 1 && r == R - 1; }
};

// A warp's two slots and their full barriers.  Unit k of the warp's range
// lands in slot k & 1; its barrier completes phase k >> 1.
struct WarpRing {
    uint8_t* buf;   // slot 0; slot 1 follows
    uint32_t bar;   // full barrier of slot 0; slot 1's is 8 bytes on
    __device__ __forceinline__ uint8_t* slot(int k) const { return buf + (k & 1) * SLOT_BYTES; }
    // lane 0: bring a unit in
    __device__ __forceinline__ void issue(int k, const void* src, uint32_t bytes) const {
        bulk_g2s(smem_u32(slot(k)), src, bytes, bar + 8 * (k & 1));
    }
    // all lanes: unit k has landed (false after the bound)
    __device__ __forceinline__ bool wait(int k) const {
        return mbar_wait(bar + 8 * (k & 1), (uint32_t)((k >> 1) & 1));
    }
    // the same for a unit issued just before (polled, never suspended)
    __device__ __forceinline__ bool wait_fresh(int k) const {
        return mbar_wait_poll(bar + 8 * (k & 1), (uint32_t)((k >> 1) & 1));
    }
    // every lane is done reading unit k's slot: lane 0 may refill it
    __device__ __forceinline__ void done(int k) const {
        __syncwarp();
        if ((threadIdx.x & 31) == 0)  // generic-proxy reads before the async-proxy refill
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
};

// Bring unit k in: `bytes` from p (lane 0 issues the copy); a short chunk's
// slot is filled past its end with `fill` words (-inf), so every chunk in
// shared memory is a full slot and the reductions need no bounds checks.
__device__ __forceinline__ void warp_ring_load(const WarpRing& r, int k, const char* p,
                                               uint32_t bytes, uint32_t fill) {
    if (bytes < (uint32_t)SLOT_BYTES) {
        uint4* t = (uint4*)r.slot(k);
        for (int q = (int)(bytes / 16) + (threadIdx.x & 31); q < SLOT_BYTES / 16; q += 32)
            t[q] = make_uint4(fill, fill, fill, fill);
        __syncwarp();  // the fill is seen by every lane that later reads the slot
    }
    if ((threadIdx.x & 31) == 0) r.issue(k, p, bytes);
}
template <class Src>
__device__ __forceinline__ void warp_ring_issue(const WarpRing& r, int k, const UnitCursor& ic,
                                                uint32_t fill, Src src) {
    const char* p;
    uint32_t bytes;
    src(ic, p, bytes);
    warp_ring_load(r, k, p, bytes, fill);
}

// Set up the calling warp's ring (barriers in `bars`, two per warp) and
// issue its first two units.  `ic` is the issue cursor, at the warp's first
// unit; src(ic, p, bytes) gives that unit's address and size; ic ends two
// units on.
template <class Src>
__device__ __forceinline__ WarpRing warp_ring_start(uint8_t* ring, uint64_t* bars, int n,
                                                    UnitCursor& ic, uint32_t fill, Src src) {
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    WarpRing r{ring + 2 * w * SLOT_BYTES, smem_u32(&bars[2 * w])};
    if (lane == 0) {
        mbar_init(r.bar, 1);
        mbar_init(r.bar + 8, 1);
        mbar_fence_init();
    }
    for (int k = 0; k < 2 && k < n; ++k) {
        warp_ring_issue(r, k, ic, fill, src);
        ic.next();
    }
    __syncwarp();
    return r;
}
// After unit k: refill its slot with unit k + 2 (if any; the issue cursor
// is there).
template <class Src>
__device__ __forceinline__ void warp_ring_next(const WarpRing& r, int k, int n, UnitCursor& ic,
                                               uint32_t fill, Src src) {
    r.done(k);
    if (k + 2 < n) {
        warp_ring_issue(r, k + 2, ic, fill, src);
        ic.next();
    }
}
// On a failed wait: let the copies this warp still has in flight land
// (bounded) before the CTA may exit.
__device__ __forceinline__ void warp_ring_abort(const WarpRing& r, int k, int n) {
    if ((threadIdx.x & 31) == 0) {
        atomicOr(&g_dev_err, ERR_STREAM);
        for (int j = k; j < k + 2 && j < n; ++j) mbar_wait(r.bar + 8 * (j & 1), (uint32_t)((j >> 1) & 1));
    }
}

// ---------------------------------------------------------------------------
// A chunk as seen by one warp: 16-byte vectors q = 0 .. nvec-1, element
// v0 + q * VW + e.  Lane l takes vectors l, l + 32, ...  SMEM: the chunk sits
// in a ring slot.  Global: read element by element from the row (any
// alignment).  Either way elements at or past n read as -inf.
template <bool BF16>
struct ChunkT {
    static constexpr int ES = BF16 ? 2 : 4;
    static constexpr int VW = 16 / ES;
    static constexpr int LEN = SLOT_BYTES / ES;
    static constexpr uint32_t NEG_INF_WORD = BF16 ? 0xFF80FF80u : 0xFF800000u;
    __device__ static __forceinline__ uint32_t word(const uint4& r, int i) {
        return i == 0 ? r.x : i == 1 ? r.y : i == 2 ? r.z : r.w;
    }
    // Element e of a vector widened to fp32 (exact).
    __device__ static __forceinline__ float elem(const uint4& r, int e) {
        if (BF16) {
            const uint32_t w = word(r, e >> 1);
            return __uint_as_float((e & 1) ? (w & 0xFFFF0000u) : (w << 16));
        }
        return __uint_as_float(word(r, e));
    }
    // The same for an index known only at run time (selects, no local memory).
    __device__ static __forceinline__ float elem_at(const uint4& r, int e) {
        const int wi = BF16 ? (e >> 1) : e;
        const uint32_t wd = (wi & 2) ? ((wi & 1) ? r.w : r.z) : ((wi & 1) ? r.y : r.x);
        if (BF16) return __uint_as_float((e & 1) ? (wd & 0xFFFF0000u) : (wd << 16));
        return __uint_as_float(wd);
    }
};

// The slot always holds SLOT_BYTES: past the chunk's n elements it is filled
// with -inf, so vectors are read without bounds checks (n still bounds the
// indices a result may name).
template <bool BF16>
struct SmemView {
    using C = ChunkT<BF16>;
    const uint8_t* buf;
    int64_t v0;
    int n;
    __device__ __forceinline__ int nvec() const { return SLOT_BYTES / 16; }
    __device__ __forceinline__ uint4 vec(int q) const { return *(const uint4*)(buf + 16 * q); }
    __device__ __forceinline__ uint4 vec_or(int q) const { return vec(q); }
    __device__ __forceinline__ int64_t index(int q, int e) const { return v0 + (int64_t)q * C::VW + e; }
};

template <bool BF16>
struct GlobalView {
    using C = ChunkT<BF16>;
    const uint8_t* row;  // the row's element 0
    int64_t v0;
    int n;
    __device__ __forceinline__ int nvec() const { return (n + C::VW - 1) / C::VW; }
    __device__ __forceinline__ uint4 vec(int q) const {
        uint32_t w[4] = {C::NEG_INF_WORD, C::NEG_INF_WORD, C::NEG_INF_WORD, C::NEG_INF_WORD};
#pragma unroll
        for (int e = 0; e < C::VW; ++e) {
            const int off = q * C::VW + e;
            if (off < n) {
                if (BF16) {
                    const uint32_t b = __ldg((const unsigned short*)row + v0 + off);
                    w[e >> 1] = (e & 1) ? ((w[e >> 1] & 0x0000FFFFu) | (b << 16))
                                        : ((w[e >> 1] & 0xFFFF0000u) | b);
                } else {
                    w[e] = __ldg((const unsigned int*)row + v0 + off);
                }
            }
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
    __device__ __forceinline__ uint4 vec_or(int q) const { return vec(q); }
    __device__ __forceinline__ int64_t index(int q, int e) const { return v0 + (int64_t)q * C::VW + e; }
};

// Packed maximum of a vector's elements: bf16 as a bf16x2 pair (values are
// finite; -0 and +0 may come back either way, every later compare treats them
// as equal), fp32 as one float's bits; unpack_max widens either to fp32.
template <bool BF16>
__device__ __forceinline__ uint32_t vmax_packed(const uint4& v) {
    if (BF16) {
        auto b2 = [](uint32_t w) { return *reinterpret_cast<const __nv_bfloat162*>(&w); };
        const __nv_bfloat162 m = __hmax2(__hmax2(b2(v.x), b2(v.y)), __hmax2(b2(v.z), b2(v.w)));
        return *reinterpret_cast<const uint32_t*>(&m);
    }
    return __float_as_uint(fmaxf(fmaxf(__uint_as_float(v.x), __uint_as_float(v.y)),
                                 fmaxf(__uint_as_float(v.z), __uint_as_float(v.w))));
}
template <bool BF16>
__device__ __forceinline__ uint32_t pmax(uint32_t a, uint32_t b) {
    if (BF16) {
        const __nv_bfloat162 m = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&a),
                                         *reinterpret_cast<const __nv_bfloat162*>(&b));
        return *reinterpret_cast<const uint32_t*>(&m);
    }
    return __float_as_uint(fmaxf(__uint_as_float(a), __uint_as_float(b)));
}
template <bool BF16>
__device__ __forceinline__ float unpack_max(uint32_t m) {
    if (BF16) return fmaxf(__uint_as_float(m << 16), __uint_as_float(m & 0xFFFF0000u));
    return __uint_as_float(m);
}
// True if some element of the packed maximum is >= t (t2: t packed likewise).
template <bool BF16>
__device__ __forceinline__ bool any_ge(uint32_t m, uint32_t t2) {
    if (BF16)
        return !__hblt2(*reinterpret_cast<const __nv_bfloat162*>(&m),
                        *reinterpret_cast<const __nv_bfloat162*>(&t2));
    return __uint_as_float(m) >= __uint_as_float(t2);
}
// A value known to be exactly representable in the element type, packed.
template <bool BF16>
__device__ __forceinline__ uint32_t pack_value(float t) {
    if (BF16) {
        const uint32_t h = __float_as_uint(t) >> 16;
        return h | (h << 16);
    }
    return __float_as_uint(t);
}

// Pass 1 over a chunk: the packed maximum of each of this lane's NVL vectors
// (vector i of lane l is q = 32 i + l; -inf past the chunk) and the lane
// maximum (-inf if the lane has no element).  All NVL loads are independent.
template <bool BF16, class View>
__device__ __forceinline__ float chunk_pass1(const View& v, uint32_t (&vm)[NVL]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int i = 0; i < NVL; ++i) vm[i] = vmax_packed<BF16>(v.vec_or(32 * i + lane));
    uint32_t t[NVL / 2];
#pragma unroll
    for (int i = 0; i < NVL / 2; ++i) t[i] = pmax<BF16>(vm[2 * i], vm[2 * i + 1]);
#pragma unroll
    for (int h = NVL / 4; h > 0; h >>= 1)
#pragma unroll
        for (int i = 0; i < h; ++i) t[i] = pmax<BF16>(t[i], t[i + h]);
    return unpack_max<BF16>(t[0]);
}

__device__ __forceinline__ float warp_max(float m) {
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, j));
    return m;
}
__device__ __forceinline__ double warp_sum(double s) {
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) s += __shfl_xor_sync(FULL, s, j);
    return s;
}

// sum over the vector's elements of exp2(x c2 - mc): fp32 pairwise within the
// vector (index order), one FMA per exponent.  The FMAs and the first two
// levels of the sum run on element pairs (fma / add .f32x2), each half
// rounded as the scalar instruction rounds it.
template <bool BF16>
__device__ __forceinline__ float vec_expsum(const uint4& w, float c2, float nmc) {
    using C = ChunkT<BF16>;
    const uint64_t cc = f2_pack(c2, c2), nn = f2_pack(nmc, nmc);
    uint64_t p[C::VW / 2];  // exponentials of elements (2i, 2i + 1)
#pragma unroll
    for (int i = 0; i < C::VW / 2; ++i) {
        const uint64_t a = f2_fma(f2_pack(C::elem(w, 2 * i), C::elem(w, 2 * i + 1)), cc, nn);
        p[i] = f2_pack(ex2(f2_lo(a)), ex2(f2_hi(a)));
    }
    if (BF16) {
        // a = (t0 + t4, t1 + t5), b = (t2 + t6, t3 + t7); then a + b, lo + hi
        const uint64_t q = f2_add(f2_add(p[0], p[C::VW / 4]), f2_add(p[1], p[C::VW / 4 + 1]));
        return f2_lo(q) + f2_hi(q);
    }
    // (t0 + t2, t1 + t3)
    const uint64_t q = f2_add(p[0], p[1]);
    return f2_lo(q) + f2_hi(q);
}

// Pass 2: the chunk's sum of exp2(x c2 - mc) with mc = fl(M c2), M the warp
// maximum (not -inf): every exponent is one FMA.  Per lane: fp32 pairwise
// within a vector and over groups of four vectors, fp64 across the groups;
// the warp's lanes in a fixed fp64 butterfly.  Every lane returns the same
// value.
template <bool BF16, class View>
__device__ __forceinline__ double chunk_expsum_at_mc(const View& v, float M, float c2) {
    const int lane = threadIdx.x & 31;
    const float nmc = -(M * c2);
    double s = 0.0;
#pragma unroll
    for (int g = 0; g < NVL / 4; ++g) {
        float e4[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) e4[j] = vec_expsum<BF16>(v.vec_or(32 * (4 * g + j) + lane), c2, nmc);
        s += (double)((e4[0] + e4[1]) + (e4[2] + e4[3]));
    }
    return warp_sum(s);
}
// The same sum against M itself: the product's rounding error M c2 - mc
// (exact in fp32 by the FMA) taken out once, in fp64.
template <bool BF16, class View>
__device__ __forceinline__ double chunk_expsum(const View& v, float M, float c2) {
    const float mc = M * c2;
    return chunk_expsum_at_mc<BF16>(v, M, c2) * exp2(-(double)fmaf(M, c2, -mc));
}

// ---------------------------------------------------------------------------
// Host side: one CTA per SM (at most one per unit), and the kernel's dynamic
// shared-memory ceiling raised to the ring's size once per device.
inline int ring_grid(int64_t units) {
    static int sms[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if (sms[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
            n = 1;
        sms[dev] = n;
    }
    return (int)(units < sms[dev] ? units : sms[dev]);
}

template <class Kernel>
inline int ring_prepare(Kernel k, size_t dyn) {
    static std::mutex mu;
    static const void* done[64][16] = {};
    if (dyn <= 48 * 1024) return DFLASH2_OK;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DFLASH2_ECUDA;
    std::lock_guard<std::mutex> g(mu);
    for (int i = 0; i < 16; ++i)
        if (done[dev][i] == (const void*)k) return DFLASH2_OK;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn) != cudaSuccess)
        return DFLASH2_ECUDA;
    for (int i = 0; i < 16; ++i)
        if (!done[dev][i]) {
            done[dev][i] = (const void*)k;
            break;
        }
    return DFLASH2_OK;
}

}  // namespace dfl
