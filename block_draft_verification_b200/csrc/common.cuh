// common.cuh -- device helpers shared by the dflash2 kernels (sm_100a).
//
// Nothing here is specific to one call: orderable keys for exact top-k and
// argmax, warp bitonic sort/merge of 64-bit keys, log-sum-exp merging,
// streaming vocabulary-row loads, Philox4x32-10, and the host-side checks.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "dflash2.h"

namespace dfl {

constexpr unsigned FULL = 0xFFFFFFFFu;
constexpr int K = DFLASH2_K;

constexpr int NT = 256;  // threads per CTA of the select and fp32 conv kernels

// ---------------------------------------------------------------------------
// Orderable keys.  ord32 maps a float to a uint32 whose unsigned order is the
// float order, with -0 and +0 mapped to the same code (they compare equal).
// key = ord32(x) << 32 | ~v: a larger key is a larger value, and among equal
// values the lower index.  Key 0 is below every finite value's key, so it
// marks "no element".
__device__ __forceinline__ uint32_t ord32(float x) {
    uint32_t b = (x == 0.0f) ? 0u : __float_as_uint(x);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float unord32(uint32_t o) {
    uint32_t b = (o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o;
    return __uint_as_float(b);
}
__device__ __forceinline__ uint64_t make_key(float x, uint32_t v) {
    return ((uint64_t)ord32(x) << 32) | (uint32_t)(~v);
}
__device__ __forceinline__ uint32_t key_index(uint64_t k) { return ~(uint32_t)k; }
__device__ __forceinline__ float key_value(uint64_t k) { return unord32((uint32_t)(k >> 32)); }

__device__ __forceinline__ uint64_t shfl_xor(uint64_t v, int m) {
    uint32_t lo = __shfl_xor_sync(FULL, (uint32_t)v, m);
    uint32_t hi = __shfl_xor_sync(FULL, (uint32_t)(v >> 32), m);
    return ((uint64_t)hi << 32) | lo;
}
__device__ __forceinline__ uint32_t shfl_xor(uint32_t v, int m) {
    return __shfl_xor_sync(FULL, v, m);
}
// Lane l gets lane l - 1's value (lane 0 keeps its own).
__device__ __forceinline__ uint64_t shfl64_up1(uint64_t v) {
    const uint32_t lo = __shfl_up_sync(FULL, (uint32_t)v, 1);
    const uint32_t hi = __shfl_up_sync(FULL, (uint32_t)(v >> 32), 1);
    return ((uint64_t)hi << 32) | lo;
}
__device__ __forceinline__ uint64_t shfl64(uint64_t v, int src) {
    uint32_t lo = __shfl_sync(FULL, (uint32_t)v, src);
    uint32_t hi = __shfl_sync(FULL, (uint32_t)(v >> 32), src);
    return ((uint64_t)hi << 32) | lo;
}

// Bitonic sort of one key per lane, descending in lane order (KeyT is
// uint32_t or uint64_t).
template <typename KeyT>
__device__ __forceinline__ KeyT warp_sort_desc(KeyT key) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            KeyT other = shfl_xor(key, j);
            bool desc_block = (lane & k) == 0;
            bool lower = (lane & j) == 0;
            key = (lower == desc_block) ? (key > other ? key : other) : (key < other ? key : other);
        }
    }
    return key;
}

// Lanes 0..15 hold a descending list, lanes 16..31 an ascending one (a
// bitonic sequence): after the merge all 32 lanes are descending, so lanes
// 0..15 hold the 16 largest keys of the union.
template <typename KeyT>
__device__ __forceinline__ KeyT warp_merge_desc(KeyT key) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) {
        KeyT other = shfl_xor(key, j);
        bool lower = (lane & j) == 0;
        key = lower ? (key > other ? key : other) : (key < other ? key : other);
    }
    return key;
}

// ---------------------------------------------------------------------------
// Log-sum-exp state (m, s): s = sum exp2((x - m) * c) over the elements seen,
// c = inv_temperature * log2(e).  An empty state is (-inf, 0).
struct Lse {
    float m;
    float s;
};
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Two fp32 values in one 64-bit register (lo, hi) for the paired fp32
// instructions of sm_100 (fma / add .f32x2): each half is rounded exactly as
// the scalar instruction would round it.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
    return d;
}
__device__ __forceinline__ float f2_lo(uint64_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float f2_hi(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ Lse lse_merge(Lse a, Lse b, float c) {
    if (a.m == -INFINITY) return b;
    if (b.m == -INFINITY) return a;
    float M = fmaxf(a.m, b.m);
    return {M, a.s * ex2((a.m - M) * c) + b.s * ex2((b.m - M) * c)};
}
// Butterfly over the warp: every lane ends with the same state (the merge is
// commutative bit for bit, so both partners of a step agree).
__device__ __forceinline__ Lse warp_lse(Lse v, float c) {
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) {
        Lse o{__shfl_xor_sync(FULL, v.m, j), __shfl_xor_sync(FULL, v.s, j)};
        v = lse_merge(v, o, c);
    }
    return v;
}

// The same state with an fp64 sum, for the verify path, whose accept
// decisions compare a uniform with a ratio of two normalisers.
struct LseD {
    float m;
    float pad;
    double s;
};
__device__ __forceinline__ LseD lse_merge(LseD a, LseD b, float c) {
    if (a.m == -INFINITY) return b;
    if (b.m == -INFINITY) return a;
    float M = fmaxf(a.m, b.m);
    return {M, 0.0f,
            a.s * exp2((double)(a.m - M) * (double)c) + b.s * exp2((double)(b.m - M) * (double)c)};
}
__device__ __forceinline__ LseD warp_lse(LseD v, float c) {
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) {
        LseD o{__shfl_xor_sync(FULL, v.m, j), 0.0f, __shfl_xor_sync(FULL, v.s, j)};
        v = lse_merge(v, o, c);
    }
    return v;
}

// ---------------------------------------------------------------------------
// Elements of a 16-byte vector of bf16 (8) or fp32 (4) values, widened to
// fp32 (exact).
template <bool BF16>
struct Row {
    static constexpr int VW = BF16 ? 8 : 4;  // elements per 16-byte vector
    __device__ static __forceinline__ uint32_t comp(const uint4& r, int i) {
        return i == 0 ? r.x : i == 1 ? r.y : i == 2 ? r.z : r.w;
    }
    // Element e (0 <= e < VW) of a raw vector.
    __device__ static __forceinline__ float elem(const uint4& r, int e) {
        if (BF16) {
            uint32_t w = comp(r, e >> 1);
            return __uint_as_float((e & 1) ? (w & 0xFFFF0000u) : (w << 16));
        }
        return __uint_as_float(comp(r, e));
    }
};

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon et al., SC'11, section 5): ten rounds of
//   (c0,c1,c2,c3) -> (hi(M1*c2)^c1^k0, lo(M1*c2), hi(M0*c0)^c3^k1, lo(M0*c0))
// with the key advanced by the Weyl increments between rounds.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
    const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
    const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k0 += W0;
            k1 += W1;
        }
        uint32_t hi0 = __umulhi(M0, c.x), lo0 = M0 * c.x;
        uint32_t hi1 = __umulhi(M1, c.z), lo1 = M1 * c.z;
        c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
    }
    return c;
}
// u in [0, 1) on the 2^-24 grid (exact in fp32) for counter
// (step, seq_id, position, purpose) and key (seed low 32, seed high 32).
__device__ __forceinline__ float philox_uniform(uint64_t seed, uint32_t step, uint32_t seq_id,
                                                uint32_t pos, uint32_t purpose) {
    uint4 o = philox4x32_10(make_uint4(step, seq_id, pos, purpose), (uint32_t)seed,
                            (uint32_t)(seed >> 32));
    return (float)(o.x >> 8) * (1.0f / 16777216.0f);
}

// ---------------------------------------------------------------------------
// "Last CTA to arrive" ticket: publish this CTA's partial (already written and
// followed by __syncthreads), count arrivals, and tell the block whether it
// is the last of `expected`.  No CTA waits on another.
__device__ __forceinline__ bool arrive_last(unsigned* counter, unsigned expected) {
    __shared__ bool last;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        unsigned t = atomicAdd(counter, 1u);
        last = (t == expected - 1);
        if (last) __threadfence();
    }
    __syncthreads();
    return last;
}

}  // namespace dfl

// ---------------------------------------------------------------------------
// Host-side argument checks shared by the entry points.
namespace dfl_host {

inline bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }
inline bool finite_pos(float x) { return isfinite(x) && x > 0.0f; }
inline int elem_size(int dtype) { return dtype == DFLASH2_BF16 ? 2 : 4; }
inline bool dtype_ok(int dtype) { return dtype == DFLASH2_F32 || dtype == DFLASH2_BF16; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline int launch_status() {
    return cudaGetLastError() == cudaSuccess ? DFLASH2_OK : DFLASH2_ECUDA;
}

}  // namespace dfl_host
