// greedy.cuh -- the pieces of the greedy verify that its two kernels share:
// the per-chunk (maximum, lowest index) key and the per-sequence decision
// from the chunk keys.
#pragma once

#include "common.cuh"
#include "ring.cuh"
#include "stream.cuh"

namespace dfl {

// One chunk, one warp: the chunk maximum M and the lowest index holding it,
// as one key.  Pass 1 keeps every vector's packed maximum; a lane holding M
// finds it in its first vector whose maximum is M (vectors of a lane are in
// index order), and the warp takes the lowest index.
template <bool BF16, class View>
__device__ __forceinline__ uint64_t greedy_chunk(const View& v) {
    using C = ChunkT<BF16>;
    const int lane = threadIdx.x & 31;
    uint32_t vm[NVL];
    const float m = chunk_pass1<BF16>(v, vm);
    const float M = warp_max(m);
    uint32_t first = 0xFFFFFFFFu;
    if (m == M) {
        const uint32_t m2 = pack_value<BF16>(M);
        int i0 = NVL;
#pragma unroll
        for (int i = NVL - 1; i >= 0; --i)
            if (any_ge<BF16>(vm[i], m2)) i0 = i;
        if (i0 < NVL) {
            const int q = 32 * i0 + lane;
            const uint4 w = v.vec(q);
#pragma unroll
            for (int e = C::VW - 1; e >= 0; --e)  // -0 == +0
                if (C::elem(w, e) == M && q * C::VW + e < v.n) first = (uint32_t)v.index(q, e);
        }
    }
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) first = min(first, __shfl_xor_sync(FULL, first, j));
    return make_key(M, first);
}

// Largest key of rows r0 .. r0+NB-1 (of S chunk keys each), warp-collective:
// lane c takes chunks c, c + 32, ...; the loads of all NB rows are issued
// together.  Every lane returns the same keys.
template <int NB>
__device__ __forceinline__ void rows_max_key(const uint64_t* P, int S, int r0, int nrows,
                                             uint64_t (&out)[NB]) {
    const int lane = threadIdx.x & 31;
    const unsigned long long* Q = (const unsigned long long*)P;
#pragma unroll
    for (int j = 0; j < NB; ++j) out[j] = 0ull;
    for (int c = lane; c < S; c += 32) {
        uint64_t k[NB];
#pragma unroll
        for (int j = 0; j < NB; ++j) k[j] = (j < nrows) ? (uint64_t)__ldcg(Q + (int64_t)(r0 + j) * S + c) : 0ull;
#pragma unroll
        for (int j = 0; j < NB; ++j) out[j] = k[j] > out[j] ? k[j] : out[j];
    }
#pragma unroll
    for (int j = 0; j < NB; ++j)
#pragma unroll
        for (int h = 16; h > 0; h >>= 1) {
            const uint64_t o = shfl_xor(out[j], h);
            out[j] = o > out[j] ? o : out[j];
        }
}

__device__ __forceinline__ void greedy_finish(const uint64_t* P, int S, int G, int64_t V, int b,
                                              const int32_t* __restrict__ draft_tok,
                                              int32_t* __restrict__ n_accept,
                                              int32_t* __restrict__ out_tok) {
    const int lane = threadIdx.x & 31;
    int32_t tj = -1;  // lane j: argmax of target row j (G + 1 <= 32)
    for (int r0 = 0; r0 <= G; r0 += 8) {
        uint64_t best[8];
        rows_max_key<8>(P, S, r0, min(8, G + 1 - r0), best);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (lane == r0 + j) tj = (int32_t)key_index(best[j]);
    }
    const int32_t dj = (lane < G) ? draft_tok[(int64_t)b * G + lane] : -1;
    // a drafted token outside [0, V) never equals an argmax: a mismatch, flagged
    if (lane < G && (uint32_t)dj >= (uint32_t)V) atomicOr(&g_dev_err, ERR_INPUT);
    const unsigned miss = __ballot_sync(FULL, lane < G && dj != tj);
    const int n = miss ? (__ffs(miss) - 1) : G;
    if (lane <= G) out_tok[(int64_t)b * (G + 1) + lane] = (lane < n) ? dj : (lane == n ? tj : -1);
    if (lane == 0) n_accept[b] = n;
}

}  // namespace dfl
