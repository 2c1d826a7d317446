// verify.cu -- lossless verification of one drafted block per sequence:
// greedy (longest prefix match against the target argmax) and sampling
// (rejection sampling with residual resample and bonus draw).
//
// Sources: "DFlash 2 — 3× plus de tokens sur Qwen3.8-27B, même sortie"
// (tamsi.dev), section "Les chiffres qui comptent sur Qwen3.8-27B": greedy
// gives exactly the target's output, sampling through rejection sampling keeps
// the target's distribution; "DFlash 2: un drafter de 3.43× que cae a 1.45×
// bajo carga" (latenode.com), section "El desacuerdo empieza en las propias
// tablas del proveedor": acceptance length = tokens completed per verify step.
// Uniforms: Philox4x32-10 (Salmon et al., SC'11, section 5).
//
// Both verifies stream every logit row once in 16384-element chunks: work
// unit = (sequence, row, chunk); persistent CTAs each take a contiguous range
// of units through a two-slot shared-memory ring filled by TMA bulk copies,
// and publish a sequence's finished units with one acquire-release add.  The
// publisher that completes a sequence (no CTA waits) reduces the partials in
// chunk order and decides.  The sampling draw needs the normalisers first, so
// it is a second kernel over the one row each sequence draws from
// (L2-resident after the first pass): one thread-block cluster per sequence,
// each CTA holding its chunks in shared memory; the chunk sums of the draw
// weights are exchanged through distributed shared memory, and the CTA that
// holds the chunk where the inverse CDF crosses t = u' * R scans it there.
// No probability vector is ever written to memory.
#include "common.cuh"
#include "stream.cuh"
#include "workspace.cuh"

#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

namespace dfl {

constexpr double LOG2E = 1.4426950408889634;
// Chunks per row the sampling draw handles (its per-chunk sums sit in shared
// memory): V <= 4096 * 16384.
constexpr int64_t DRAW_MAX_CHUNKS = 4096;
// Dynamic shared memory of the draw: the target and draft chunks, then two
// rounds of per-chunk sums.
inline size_t draw_smem(int es, int64_t S) { return 2 * (size_t)CHUNK * es + (size_t)S * 2 * sizeof(double); }

// ------------------------------------------------------------------ greedy
struct GreedySmem {
    float wmax[NT / 32];
    unsigned first;
};

template <bool BF16, class C>
__device__ __forceinline__ void greedy_unit(const C& ch, GreedySmem& sm, uint64_t* slot) {
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const float m = view_max<BF16>(ch);
    float wm = m;
#pragma unroll
    for (int k = 16; k > 0; k >>= 1) wm = fmaxf(wm, __shfl_xor_sync(FULL, wm, k));
    if (lane == 0) sm.wmax[warp] = wm;
    if (t == 0) sm.first = 0xFFFFFFFFu;
    __syncthreads();
    float M = sm.wmax[0];
#pragma unroll
    for (int w = 1; w < NT / 32; ++w) M = fmaxf(M, sm.wmax[w]);
    if (m == M) atomicMin(&sm.first, view_first<BF16>(ch, M));  // -0 == +0
    __syncthreads();
    if (t == 0) *slot = make_key(M, sm.first);  // published by thread 0's release add
}

__device__ __forceinline__ void greedy_finish(const uint64_t* P, int S, int G, int b,
                                              const int32_t* __restrict__ draft_tok,
                                              int32_t* __restrict__ n_accept,
                                              int32_t* __restrict__ out_tok) {
    const int lane = threadIdx.x & 31;
    uint64_t best = 0;  // lane j reduces target row j over its chunks (G + 1 <= 32)
    if (lane <= G)
        for (int c = 0; c < S; ++c) {
            const uint64_t k = (uint64_t)__ldcg((const unsigned long long*)&P[(int64_t)lane * S + c]);
            best = k > best ? k : best;
        }
    const int32_t tj = (int32_t)key_index(best);
    const int32_t dj = (lane < G) ? draft_tok[(int64_t)b * G + lane] : -1;
    const unsigned miss = __ballot_sync(FULL, lane < G && dj != tj);
    const int n = miss ? (__ffs(miss) - 1) : G;
    if (lane <= G) out_tok[(int64_t)b * (G + 1) + lane] = (lane < n) ? dj : (lane == n ? tj : -1);
    if (lane == 0) n_accept[b] = n;
}

template <bool BF16, bool TMA>
__global__ void __launch_bounds__(NT, 3) verify_greedy_kernel(
    const void* __restrict__ target, int G, int64_t V, int S, int64_t units,
    const int32_t* __restrict__ draft_tok, int32_t* __restrict__ n_accept,
    int32_t* __restrict__ out_tok, uint64_t* __restrict__ part, unsigned* __restrict__ counters) {
    constexpr int ES = BF16 ? 2 : 4;
    constexpr int SLOT = CHUNK * ES;
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ GreedySmem sm;
    __shared__ __align__(8) uint64_t s_bar[2];
    const int t = threadIdx.x, warp = t >> 5;
    const uint32_t bar0 = smem_u32(&s_bar[0]);
    const int per_seq = (G + 1) * S;
    auto geom = [&](int64_t u, int& b, int64_t& row, int64_t& v0, int64_t& vend) {
        b = (int)(u / per_seq);
        const int rem = (int)(u - (int64_t)b * per_seq);
        const int j = rem / S;
        row = (int64_t)b * (G + 1) + j;
        v0 = (int64_t)(rem - j * S) * CHUNK;
        vend = min(V, v0 + (int64_t)CHUNK);
    };
    auto issue = [&](int64_t u, int slot) {
        int b;
        int64_t row, v0, vend;
        geom(u, b, row, v0, vend);
        bulk_g2s(smem_u32(ring + slot * SLOT), (const char*)target + (row * V + v0) * ES,
                 (uint32_t)((vend - v0) * ES), bar0 + 8 * slot);
    };
    int64_t lo, hi;
    cta_range(units, lo, hi);
    if (TMA) {
        if (t == 0) {
            mbar_init(bar0, 1);
            mbar_init(bar0 + 8, 1);
            mbar_fence_init();
            if (lo < hi) issue(lo, 0);
        }
        __syncthreads();
    }
    __shared__ bool s_last;
    unsigned pending = 0;
    int k = 0;
    for (int64_t u = lo; u < hi; ++u, ++k) {
        int b;
        int64_t row, v0, vend;
        geom(u, b, row, v0, vend);
        uint64_t* slot = part + row * S + (v0 / CHUNK);
        if (TMA) {
            if (t == 0 && u + 1 < hi) issue(u + 1, (k + 1) & 1);
            if (!__syncthreads_and(mbar_wait(bar0 + 8 * (k & 1), (k >> 1) & 1))) {
                if (t == 0) {
                    atomicOr(&g_dev_err, ERR_STREAM);
                    if (u + 1 < hi) mbar_wait(bar0 + 8 * ((k + 1) & 1), ((k + 1) >> 1) & 1);
                }
                return;
            }
            greedy_unit<BF16>(SmemChunk<BF16>{ring + (k & 1) * SLOT, v0, vend}, sm, slot);
        } else {
            RegChunk<BF16> ch;
            ch.load((const char*)target + row * V * ES, v0, vend);
            greedy_unit<BF16>(ch, sm, slot);
        }
        ++pending;
        if (u + 1 == hi || (u + 1) / per_seq != b) {  // done with this sequence: publish
            __syncthreads();
            if (t == 0) s_last = publish(&counters[b], pending, (unsigned)per_seq);
            __syncthreads();
            if (s_last && warp == 0)
                greedy_finish(part + (int64_t)b * (G + 1) * S, S, G, b, draft_tok, n_accept, out_tok);
            pending = 0;
        }
        __syncthreads();  // ring slot k & 1 is free for the prefetch of iteration k + 1
    }
}

// ------------------------------------------------------------------ sampling, pass 1
// Units: for sequence b, rows 0..G are target rows, G+1..2G draft rows (softmax
// mode only).  Each unit writes its (max, fp64 sum-exp) partial; the last
// unit of the sequence runs the accept tests.
__device__ __forceinline__ void sample_finish(
    const void* __restrict__ target, const void* __restrict__ draft, const LseD* P, int G,
    int64_t V, int S, int es, float inv_t, float c2, const int32_t* __restrict__ draft_tok,
    uint64_t seed, uint32_t step, uint32_t sid, int q_mode, int b, int32_t* __restrict__ n_accept,
    int32_t* __restrict__ out_tok, float* __restrict__ ratio_dbg, float* __restrict__ u_dbg,
    SampleInfo* __restrict__ info) {
    const int lane = threadIdx.x & 31;
    auto row_lse = [&](int rrow) {  // chunk order
        LseD acc{-INFINITY, 0.0f, 0.0};
        for (int c = 0; c < S; ++c) {
            LseD p{__ldcg(&P[(int64_t)rrow * S + c].m), 0.0f, __ldcg(&P[(int64_t)rrow * S + c].s)};
            acc = lse_merge(acc, p, c2);
        }
        return acc;
    };
    auto elem = [&](const void* base, int64_t row, int32_t v) -> double {
        if (es == 2)
            return (double)__uint_as_float((uint32_t)((const uint16_t*)base)[row * V + v] << 16);
        return (double)((const float*)base)[row * V + v];
    };
    LseD lt{-INFINITY, 0.0f, 0.0}, lq{-INFINITY, 0.0f, 0.0};
    if (lane <= G) lt = row_lse(lane);
    if (q_mode == DFLASH2_Q_SOFTMAX && lane < G) lq = row_lse(G + 1 + lane);
    bool reject = false;
    if (lane < G) {
        const int32_t d = draft_tok[(int64_t)b * G + lane];
        // lp = z_t[d] - logZ_t = (x - m) * invT - ln(s); likewise lq
        double lr = (elem(target, (int64_t)b * (G + 1) + lane, d) - (double)lt.m) * (double)inv_t -
                    log(lt.s);
        if (q_mode == DFLASH2_Q_SOFTMAX)
            lr -= (elem(draft, (int64_t)b * G + lane, d) - (double)lq.m) * (double)inv_t - log(lq.s);
        const double ratio = exp(lr);
        const float u = philox_uniform(seed, step, sid, (uint32_t)lane, 0u);
        reject = !((double)u < ratio);
        if (ratio_dbg) ratio_dbg[(int64_t)b * G + lane] = (float)ratio;
        if (u_dbg) u_dbg[(int64_t)b * G + lane] = u;
    }
    const unsigned rej = __ballot_sync(FULL, reject);
    const int n = rej ? (__ffs(rej) - 1) : G;
    const int32_t dn = (lane < G) ? draft_tok[(int64_t)b * G + lane] : -1;
    if (lane <= G) out_tok[(int64_t)b * (G + 1) + lane] = (lane < n) ? dn : -1;  // draw fills n
    const float ltm = __shfl_sync(FULL, lt.m, n);
    const double lts = __shfl_sync(FULL, lt.s, n);
    const float lqm = __shfl_sync(FULL, lq.m, n);
    const double lqs = __shfl_sync(FULL, lq.s, n);
    const int32_t d_n = __shfl_sync(FULL, dn, n);
    if (lane == 0) {
        SampleInfo I;
        const bool resid = n < G && q_mode == DFLASH2_Q_SOFTMAX;
        I.mt = ltm;
        I.l2t = (float)log2(lts);
        I.mq = lqm;
        I.l2q = resid ? (float)log2(lqs) : 0.0f;
        I.dl = resid ? (float)(((double)ltm - (double)lqm) * (double)inv_t + log(lts) - log(lqs))
                     : 0.0f;
        I.u_res = philox_uniform(seed, step, sid, (uint32_t)n, 1u);
        I.n = n;
        I.mode = (n == G) ? 2 : (q_mode == DFLASH2_Q_SOFTMAX ? 0 : 1);
        I.d = d_n;
        I.pad = 0;
        info[b] = I;
        n_accept[b] = n;
    }
}

// A chunk's (max, sum-exp) in two levels.  Each thread holds its 64
// elements in registers, takes its own max m and s = sum exp2(x c - m c)
// (fp32 within a 16-byte vector, fp64 across vectors), each exponent one FMA
// against mc = fl(m c); its warp rescales the thread sums to the warp max,
// taking out the product's rounding error e = m c - mc (exact in fp32, and as
// large as 6e-5 at |m c| ~ 1e3) in the same factor, adds them (butterfly),
// and lane 0 leaves (M_w, S_w) in shared memory.  The CTA's eight warp pairs are merged later by
// thread 0 in warp order (warp_pairs_merge).
template <bool BF16, class C>
__device__ __forceinline__ void warp_lse_pair(const C& ch, float c2, float* s_m, double* s_s) {
    using R = Row<BF16>;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint4 v[R::NV];
#pragma unroll
    for (int i = 0; i < R::NV; ++i) v[i] = ch.vec(i);
    float m = vec_max<BF16>(v[0]);
#pragma unroll
    for (int i = 1; i < R::NV; ++i) m = fmaxf(m, vec_max<BF16>(v[i]));
    double s = 0.0;
    const float mc = -m * c2;
    if (m != -INFINITY) {
#pragma unroll
        for (int i = 0; i < R::NV; ++i) {
            float tt[R::VW];
#pragma unroll
            for (int e = 0; e < R::VW; ++e) tt[e] = ex2(fmaf(R::elem(v[i], e), c2, mc));
#pragma unroll
            for (int w = R::VW / 2; w > 0; w >>= 1)
#pragma unroll
                for (int e = 0; e < w; ++e) tt[e] += tt[e + w];
            s += (double)tt[0];
        }
    }
    float M = m;
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, j));
    if (s > 0.0) s *= (double)ex2((m - M) * c2 - fmaf(m, c2, mc));
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) s += __shfl_xor_sync(FULL, s, j);
    if (lane == 0) {
        s_m[warp] = M;
        s_s[warp] = s;
    }
}
__device__ __forceinline__ LseD warp_pairs_merge(const float* s_m, const double* s_s, float c2) {
    float M = s_m[0];
#pragma unroll
    for (int w = 1; w < NT / 32; ++w) M = fmaxf(M, s_m[w]);
    double S = 0.0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w)
        if (s_s[w] > 0.0) S += s_s[w] * (double)ex2((s_m[w] - M) * c2);
    return {M, 0.0f, S};
}

// Units are (sequence b, row rr, chunk): rows 0..G of a sequence are its
// target rows, G+1..2G its draft rows (softmax mode only).  Per unit the
// block meets once: after the unit's copy has landed.  At that barrier every
// warp has also left its pair for the previous unit and finished reading the
// previous slot, so warp 0 then refills that slot with the unit after next,
// merges the previous unit's pairs and stores its partial; the publisher that
// completes a sequence runs its accept tests in warp 0.
template <bool BF16, bool TMA>
__global__ void __launch_bounds__(NT, 3) verify_sample_scan_kernel(
    const void* __restrict__ target, const void* __restrict__ draft, int G, int64_t V, int S,
    int rows_per_seq, int64_t units, float inv_t, float c2, const int32_t* __restrict__ draft_tok,
    uint64_t seed, uint32_t step, const uint32_t* __restrict__ seq_id, int q_mode,
    int32_t* __restrict__ n_accept, int32_t* __restrict__ out_tok, float* __restrict__ ratio_dbg,
    float* __restrict__ u_dbg, LseD* __restrict__ part, SampleInfo* __restrict__ info,
    unsigned* __restrict__ counters) {
    constexpr int ES = BF16 ? 2 : 4;
    constexpr int SLOT = CHUNK * ES;
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ float s_m[2][NT / 32];
    __shared__ double s_s[2][NT / 32];
    __shared__ __align__(8) uint64_t s_bar[2];
    const int t = threadIdx.x, warp = t >> 5;
    const uint32_t bar0 = smem_u32(&s_bar[0]);
    const int per_seq = rows_per_seq * S;  // units of one sequence (fits int: checked on the host)
    struct Geo {
        int b, rr, c;
        const char* rowp;
        int64_t v0, vend;
    };
    auto geom = [&](int u) {
        Geo g;
        g.b = u / per_seq;
        const int rem = u - g.b * per_seq;
        g.rr = rem / S;
        g.c = rem - g.rr * S;
        g.rowp = (g.rr <= G) ? (const char*)target + ((int64_t)g.b * (G + 1) + g.rr) * V * ES
                             : (const char*)draft + ((int64_t)g.b * G + (g.rr - G - 1)) * V * ES;
        g.v0 = (int64_t)g.c * CHUNK;
        g.vend = min(V, g.v0 + (int64_t)CHUNK);
        return g;
    };
    auto issue = [&](int u, int slot) {
        const Geo g = geom(u);
        bulk_g2s(smem_u32(ring + slot * SLOT), g.rowp + g.v0 * ES, (uint32_t)((g.vend - g.v0) * ES),
                 bar0 + 8 * slot);
    };
    int64_t lo64, hi64;
    cta_range(units, lo64, hi64);
    const int lo = (int)lo64, hi = (int)hi64;
    if (TMA) {
        if (t == 0) {
            mbar_init(bar0, 1);
            mbar_init(bar0 + 8, 1);
            mbar_fence_init();
            if (lo < hi) issue(lo, 0);
            if (lo + 1 < hi) issue(lo + 1, 1);
        }
        __syncthreads();
    }
    // warp 0's record of the previous unit, finished at the next barrier
    int pb = 0, ppart = 0;
    bool plast = false;
    unsigned pending = 0;
    auto finish_prev = [&](int kk) {  // warp 0
        if (t == 0) part[ppart] = warp_pairs_merge(s_m[kk & 1], s_s[kk & 1], c2);
        ++pending;
        if (plast) {  // done with this sequence: publish its units
            bool last = false;
            if (t == 0) last = publish(&counters[pb], pending, (unsigned)per_seq);
            last = __shfl_sync(FULL, last, 0);
            if (last)
                sample_finish(target, draft, part + (int64_t)pb * rows_per_seq * S, G, V, S, ES, inv_t,
                              c2, draft_tok, seed, step, seq_id ? seq_id[pb] : (uint32_t)pb, q_mode,
                              pb, n_accept, out_tok, ratio_dbg, u_dbg, info);
            pending = 0;
        }
    };
    int k = 0;
    for (int u = lo; u < hi; ++u, ++k) {
        const Geo g = geom(u);
        if (TMA) {
            if (!__syncthreads_and(mbar_wait(bar0 + 8 * (k & 1), (k >> 1) & 1))) {
                if (t == 0) {
                    atomicOr(&g_dev_err, ERR_STREAM);
                    if (u + 1 < hi) mbar_wait(bar0 + 8 * ((k + 1) & 1), ((k + 1) >> 1) & 1);
                }
                return;
            }
        } else {
            __syncthreads();
        }
        if (warp == 0) {
            if (TMA && t == 0 && k >= 1 && u + 1 < hi) issue(u + 1, (k + 1) & 1);
            if (k >= 1) finish_prev(k - 1);
            pb = g.b;
            ppart = (g.b * rows_per_seq + g.rr) * S + g.c;
            plast = (u + 1 == hi) || ((u + 1) / per_seq != g.b);
        }
        if (TMA) {
            warp_lse_pair<BF16>(SmemChunk<BF16>{ring + (k & 1) * SLOT, g.v0, g.vend}, c2, s_m[k & 1],
                                s_s[k & 1]);
        } else {
            RegChunk<BF16> ch;
            ch.load(g.rowp, g.v0, g.vend);
            warp_lse_pair<BF16>(ch, c2, s_m[k & 1], s_s[k & 1]);
        }
    }
    __syncthreads();
    if (warp == 0 && k >= 1) finish_prev(k - 1);
}

// ------------------------------------------------------------------ sampling, pass 2
// Draw weight of one element of the row the sequence draws from:
//   p_v = exp2((x_v - mt) * c - l2t),  q_v likewise,
//   mode 0: w = max(0, p - q), evaluated as q * expm1(ln p - ln q) with
//           ln p - ln q = (xt - xq) * invT - (logZ_t - logZ_q): the same
//           value, without the cancellation of p - q when p and q agree;
//   mode 1: w = p, 0 at d;  mode 2: w = p.
// With use_p (the residual was empty by rounding) the weight is p.
// e^d - 1 for d > 0: the Taylor series to d^8 for d <= 1/2 (truncation below
// 6e-9 relative there), e^d - 1 from exp2 above, where the subtraction costs
// at most two bits.
__device__ __forceinline__ float expm1_pos(float d) {
    if (d > 0.5f) return ex2(d * 1.4426950408889634f) - 1.0f;
    float p = 1.0f / 40320.0f;
    p = fmaf(p, d, 1.0f / 5040.0f);
    p = fmaf(p, d, 1.0f / 720.0f);
    p = fmaf(p, d, 1.0f / 120.0f);
    p = fmaf(p, d, 1.0f / 24.0f);
    p = fmaf(p, d, 1.0f / 6.0f);
    p = fmaf(p, d, 0.5f);
    p = fmaf(p, d, 1.0f);
    return p * d;
}

__device__ __forceinline__ float draw_weight(float xt, float xq, int64_t v, const SampleInfo& I,
                                             float c, float inv_t, bool use_p) {
    if (I.mode == 0 && !use_p) {
        const float dlog = (xt - xq) * inv_t - I.dl;
        if (!(dlog > 0.0f)) return 0.0f;
        return ex2((xq - I.mq) * c - I.l2q) * expm1_pos(dlog);
    }
    if (I.mode == 1 && !use_p && v == I.d) return 0.0f;
    return ex2((xt - I.mt) * c - I.l2t);
}

// Element `off` of a chunk held in shared memory, widened to fp32 (exact).
template <bool BF16>
__device__ __forceinline__ float smem_elem(const uint8_t* buf, int off) {
    if (BF16) return __uint_as_float((uint32_t)((const uint16_t*)buf)[off] << 16);
    return ((const float*)buf)[off];
}

// Sum of the draw weights of thread t's 64 contiguous elements
// [v0 + 64 t, v0 + 64 t + 64) of the chunk in shared memory: fp32 within a
// 16-byte vector (index order), fp64 across the vectors.  Thread t starts at
// its vector t mod NV, so the eight threads of a quarter warp read eight
// different bank groups.
template <bool BF16>
__device__ __forceinline__ double chunk_thread_sum(const uint8_t* tb, const uint8_t* qb, int64_t v0,
                                                   int64_t vend, const SampleInfo& I, float c2,
                                                   float inv_t, bool use_p) {
    using R = Row<BF16>;
    constexpr int ES = BF16 ? 2 : 4;
    const int t = threadIdx.x;
    const bool with_q = I.mode == 0 && !use_p;
    double s = 0.0;
#pragma unroll 2
    for (int j = 0; j < R::NV; ++j) {
        const int off = t * EPT + ((j + t) & (R::NV - 1)) * R::VW;
        if (v0 + off >= vend) continue;
        const uint4 rt = *(const uint4*)(tb + off * ES);
        const uint4 rq = with_q ? *(const uint4*)(qb + off * ES) : make_uint4(0, 0, 0, 0);
        float sv = 0.0f;
#pragma unroll
        for (int e = 0; e < R::VW; ++e) {
            const int64_t v = v0 + off + e;
            if (v < vend)
                sv += draw_weight(R::elem(rt, e), R::elem(rq, e), v, I, c2, inv_t, use_p);
        }
        s += (double)sv;
    }
    return s;
}

// Block sum in a fixed order (warp butterflies, then the warps in order).
__device__ __forceinline__ double block_sum(double v, double* s_warp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int k = 16; k > 0; k >>= 1) v += __shfl_xor_sync(FULL, v, k);
    __syncthreads();
    if (lane == 0) s_warp[warp] = v;
    __syncthreads();
    double tot = 0.0;
    for (int w = 0; w < NT / 32; ++w) tot += s_warp[w];
    return tot;
}

// Thread-block cluster plumbing (PTX ISA: barrier.cluster, mapa).
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Store v at `local` (a shared-memory address of this kernel) in CTA `rank`
// of the cluster.
__device__ __forceinline__ void st_cluster(double* local, double v, uint32_t rank) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(rank));
    asm volatile("st.shared::cluster.f64 [%0], %1;" ::"r"(ra), "d"(v) : "memory");
}

// One cluster of CL CTAs per sequence; CTA r holds the chunks
// [r S / CL, (r + 1) S / CL) of the row the sequence draws from (and of the
// draft row in mode 0), brought into shared memory by one bulk copy each.
// Every CTA sums its chunks' draw weights and stores each chunk sum into
// every CTA of the cluster; after one cluster barrier all CTAs hold the same
// S sums, take R and the crossing chunk c* (the first c whose inclusive
// prefix exceeds t = u' R) in the same order, and the CTA holding c* finds the
// thread, then the element, from the data it already has.  Control flow up to
// the last cluster barrier is the same in every CTA of the cluster (the
// fallback to p is decided from the same sums everywhere).
template <bool BF16, bool TMA>
__global__ void __launch_bounds__(NT, 3) verify_sample_draw_kernel(
    const void* __restrict__ target, const void* __restrict__ draft, int G, int64_t V, int S,
    float c2, float inv_t, const SampleInfo* __restrict__ info, int32_t* __restrict__ out_tok) {
    constexpr int ES = BF16 ? 2 : 4;
    using R = Row<BF16>;
    extern __shared__ __align__(128) uint8_t s_dyn[];  // target chunk | draft chunk | sums[2][S]
    uint8_t* tbuf = s_dyn;
    uint8_t* qbuf = s_dyn + CHUNK * ES;
    double* s_all = (double*)(s_dyn + 2 * CHUNK * ES);
    __shared__ double s_warp[NT / 32];
    __shared__ double s_scan[NT];
    __shared__ double s_base, s_t;
    __shared__ int s_cstar, s_fallback, s_pick_thread, s_done, s_last;
    __shared__ __align__(8) uint64_t s_bar;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int CL = (int)cluster_size(), rank = (int)cluster_rank();
    const int b = blockIdx.x / CL;
    const SampleInfo I = info[b];
    const char* trow = (const char*)target + ((int64_t)b * (G + 1) + I.n) * V * ES;
    const char* qrow = (I.mode == 0) ? (const char*)draft + ((int64_t)b * G + I.n) * V * ES : nullptr;
    const int c0 = (int)((int64_t)rank * S / CL), c1 = (int)((int64_t)(rank + 1) * S / CL);
    const uint32_t bar = smem_u32(&s_bar);
    if (TMA && t == 0) {
        mbar_init(bar, 1);
        mbar_fence_init();
    }
    __syncthreads();
    cluster_arrive_relaxed();  // this CTA has started: its shared memory may be written

    int loaded = -1, nload = 0;
    bool copies_ok = true;
    // Bring chunk c of the target row (and of the draft row if need_q) into
    // shared memory; block-uniform.
    auto load_chunk = [&](int c, bool need_q) {
        const int64_t v0 = (int64_t)c * CHUNK, vend = min(V, v0 + (int64_t)CHUNK);
        const int n = (int)(vend - v0);
        __syncthreads();  // every thread is done with the previous chunk
        if (TMA) {
            if (!copies_ok) return;
            if (t == 0) {
                const uint32_t bytes = (uint32_t)n * ES;
                mbar_expect_tx(bar, need_q ? 2 * bytes : bytes);
                bulk_g2s_nx(smem_u32(tbuf), trow + v0 * ES, bytes, bar);
                if (need_q) bulk_g2s_nx(smem_u32(qbuf), qrow + v0 * ES, bytes, bar);
            }
            const bool ok = __syncthreads_and(mbar_wait(bar, (uint32_t)(nload & 1)));
            ++nload;
            if (!ok) {  // the copy never landed: flag it and issue no more
                if (t == 0) atomicOr(&g_dev_err, ERR_STREAM);
                copies_ok = false;
            }
        } else {
            for (int e = t; e < n; e += NT) {
                if (BF16) {
                    ((uint16_t*)tbuf)[e] = ((const uint16_t*)trow)[v0 + e];
                    if (need_q) ((uint16_t*)qbuf)[e] = ((const uint16_t*)qrow)[v0 + e];
                } else {
                    ((float*)tbuf)[e] = ((const float*)trow)[v0 + e];
                    if (need_q) ((float*)qbuf)[e] = ((const float*)qrow)[v0 + e];
                }
            }
            __syncthreads();
        }
        loaded = c;
    };
    // One round: every owned chunk's sum into sums[round][c] of every CTA,
    // then the cluster barrier.  Returns this thread's sum of the last chunk.
    auto round_sums = [&](int round, bool use_p) -> double {
        const bool need_q = I.mode == 0 && !use_p;
        double my = 0.0;
        for (int c = c0; c < c1; ++c) {
            if (loaded != c) load_chunk(c, need_q);
            const int64_t v0 = (int64_t)c * CHUNK, vend = min(V, v0 + (int64_t)CHUNK);
            my = chunk_thread_sum<BF16>(tbuf, qbuf, v0, vend, I, c2, inv_t, use_p);
            const double cs = block_sum(my, s_warp);
            if (round == 0 && c == c0) cluster_wait();  // every CTA of the cluster has started
            if (t < CL) st_cluster(&s_all[round * S + c], cs, (uint32_t)t);
        }
        cluster_arrive();
        cluster_wait();
        return my;
    };

    double mysum = round_sums(0, false);
    if (t == 0) {
        double Rm = 0.0;
        for (int c = 0; c < S; ++c) Rm += s_all[c];
        s_fallback = !(Rm > 0.0);
    }
    __syncthreads();
    const bool use_p = s_fallback != 0;  // the same in every CTA of the cluster
    if (use_p) mysum = round_sums(1, true);  // residual empty by rounding: draw from p_n (rare)
    const double* sums = s_all + (use_p ? S : 0);
    if (t == 0) {
        double Rm = 0.0;
        for (int c = 0; c < S; ++c) Rm += sums[c];
        const double tt = (double)I.u_res * Rm;
        double pre = 0.0;
        int cstar = -1, clast = 0;
        for (int c = 0; c < S; ++c) {
            const double wc = sums[c];
            if (wc > 0.0) clast = c;
            if (cstar < 0 && pre + wc > tt) cstar = c;
            if (cstar < 0) pre += wc;
        }
        if (cstar < 0) {  // rounding left t at the top: the last chunk with mass
            cstar = clast;
            pre = 0.0;
            for (int c = 0; c < clast; ++c) pre += sums[c];
        }
        s_cstar = cstar;
        s_base = pre;
        s_t = tt;
        s_pick_thread = NT;
        s_done = 0;
        s_last = -1;
    }
    __syncthreads();
    const int cstar = s_cstar;
    if (cstar < c0 || cstar >= c1) return;  // another CTA of the cluster draws
    if (loaded != cstar) {  // this CTA holds several chunks: fetch c* again
        load_chunk(cstar, I.mode == 0 && !use_p);
        const int64_t v0 = (int64_t)cstar * CHUNK, vend = min(V, v0 + (int64_t)CHUNK);
        mysum = chunk_thread_sum<BF16>(tbuf, qbuf, v0, vend, I, c2, inv_t, use_p);
    }
    const int64_t v0 = (int64_t)cstar * CHUNK, vend = min(V, v0 + (int64_t)CHUNK);
    const double tt = s_t;
    // inclusive scan of the thread sums in thread (= index) order
    double incl = mysum;
#pragma unroll
    for (int k = 1; k < 32; k <<= 1) {
        const double o = __shfl_up_sync(FULL, incl, k);
        if (lane >= k) incl += o;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    double wbase = 0.0;
    for (int w = 0; w < warp; ++w) wbase += s_warp[w];
    incl += wbase;
    s_scan[t] = incl;
    if (s_base + incl > tt) atomicMin(&s_pick_thread, t);
    __syncthreads();
    const int pt = s_pick_thread;
    const bool with_q = I.mode == 0 && !use_p;
    if (pt < NT && warp == 0) {
        // warp 0 walks thread pt's 64 elements, two per lane, in index order
        const int off = pt * EPT + 2 * lane;
        const int64_t vb = v0 + off;
        float w0 = 0.0f, w1 = 0.0f;
        if (vb < vend)
            w0 = draw_weight(smem_elem<BF16>(tbuf, off), with_q ? smem_elem<BF16>(qbuf, off) : 0.0f,
                             vb, I, c2, inv_t, use_p);
        if (vb + 1 < vend)
            w1 = draw_weight(smem_elem<BF16>(tbuf, off + 1),
                             with_q ? smem_elem<BF16>(qbuf, off + 1) : 0.0f, vb + 1, I, c2, inv_t,
                             use_p);
        double incl2 = (double)w0 + (double)w1;
#pragma unroll
        for (int kk = 1; kk < 32; kk <<= 1) {
            const double o = __shfl_up_sync(FULL, incl2, kk);
            if (lane >= kk) incl2 += o;
        }
        const double base = s_base + (pt > 0 ? s_scan[pt - 1] : 0.0);
        const double before = base + incl2 - ((double)w0 + (double)w1);
        const bool p0 = before + (double)w0 > tt;
        const bool p1 = before + (double)w0 + (double)w1 > tt;
        const unsigned m0 = __ballot_sync(FULL, p0), m1 = __ballot_sync(FULL, p1);
        const unsigned has = __ballot_sync(FULL, w0 > 0.0f || w1 > 0.0f);
        int pick = -1;
        if (m0 | m1) {  // the first element whose inclusive prefix exceeds t
            const int l0 = m0 ? __ffs(m0) - 1 : 32, l1 = m1 ? __ffs(m1) - 1 : 32;
            pick = (l0 <= l1) ? 2 * l0 : 2 * l1 + 1;
        } else if (has) {  // rounding: the last element with mass
            const int ll = 31 - __clz(has);
            const float lw1 = __shfl_sync(FULL, w1, ll);
            pick = 2 * ll + (lw1 > 0.0f ? 1 : 0);
        }
        if (lane == 0 && pick >= 0) {
            out_tok[(int64_t)b * (G + 1) + I.n] = (int32_t)(v0 + pt * EPT + pick);
            s_done = 1;
        }
    }
    __syncthreads();
    if (!s_done) {  // block-uniform: rounding left t above the chunk's scan
        if (mysum > 0.0) {
            int lastpos = -1;
#pragma unroll 1
            for (int e = 0; e < EPT; ++e) {
                const int off = t * EPT + e;
                const int64_t v = v0 + off;
                if (v < vend &&
                    draw_weight(smem_elem<BF16>(tbuf, off), with_q ? smem_elem<BF16>(qbuf, off) : 0.0f,
                                v, I, c2, inv_t, use_p) > 0.0f)
                    lastpos = e;
            }
            if (lastpos >= 0) atomicMax(&s_last, t * EPT + lastpos);
        }
        __syncthreads();
        if (t == 0 && s_last >= 0) out_tok[(int64_t)b * (G + 1) + I.n] = (int32_t)(v0 + s_last);
    }
}

}  // namespace dfl

using namespace dfl;
using namespace dfl_host;

unsigned dfl_errors_verify(int clear) {
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_dev_err, sizeof v) != cudaSuccess) return 0xFFFFFFFFu;
    if (clear && v) {
        unsigned z = 0;
        cudaMemcpyToSymbol(g_dev_err, &z, sizeof z);
    }
    return v;
}

template <class Kern>
static int prep_stream_kernel(Kern kern, size_t dyn) {
    if (dyn > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn) != cudaSuccess)
        return DFLASH2_ECUDA;
    return DFLASH2_OK;
}

// Cluster size of the draw: one CTA per chunk up to 16 (the non-portable
// maximum), fewer if the device cannot co-schedule that many CTAs of this
// shared-memory size.  The kernel's shared-memory ceiling is set once per
// device to the largest size any vocabulary needs (the ceiling is a property
// of the kernel, so a smaller call must not lower it); the cluster limit is
// looked up once per device, kernel and size.
template <class Kern>
static int draw_cluster(Kern kern, size_t dyn, size_t dyn_max, int S) {
    static std::mutex mu;
    static std::map<std::tuple<int, const void*, size_t>, int> limit;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> g(mu);
    const auto kkey = std::make_tuple(dev, (const void*)kern, (size_t)0);
    if (limit.find(kkey) == limit.end()) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn_max) !=
                cudaSuccess ||
            cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                cudaSuccess)
            return 0;
        limit.emplace(kkey, 1);
    }
    const auto key = std::make_tuple(dev, (const void*)kern, dyn);
    auto it = limit.find(key);
    if (it == limit.end()) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(16);
        cfg.blockDim = dim3(NT);
        cfg.dynamicSmemBytes = dyn;
        int n = 0;
        if (cudaOccupancyMaxPotentialClusterSize(&n, (const void*)kern, &cfg) != cudaSuccess) return 0;
        it = limit.emplace(key, n).first;
    }
    return std::min(std::min(S, 16), it->second);
}

template <class Kern, class... Args>
static int launch_cluster(Kern kern, int grid, int cl, size_t dyn, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = dyn;
    cfg.stream = s;
    cudaLaunchAttribute a[1];
    a[0].id = cudaLaunchAttributeClusterDimension;
    a[0].val.clusterDim.x = (unsigned)cl;
    a[0].val.clusterDim.y = 1;
    a[0].val.clusterDim.z = 1;
    cfg.attrs = a;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...) == cudaSuccess ? DFLASH2_OK : DFLASH2_ECUDA;
}

extern "C" int dflash2_verify_greedy(const void* target, int dtype, int B, int G, int64_t V,
                                     const int32_t* draft_tok, int32_t* n_accept, int32_t* out_tok,
                                     void* ws, size_t ws_bytes, dflash2_stream_t stream) {
    if (!dtype_ok(dtype)) return DFLASH2_EDTYPE;
    if (B < 0 || G < 1 || G >= DFLASH2_MAX_BLOCK || V < 1 || V > INT32_MAX) return DFLASH2_ESHAPE;
    if (B == 0) return DFLASH2_OK;
    if (!target || !draft_tok || !n_accept || !out_tok) return DFLASH2_EINVAL;
    const int es = elem_size(dtype);
    if (!aligned(target, es) || !aligned(draft_tok, 4) || !aligned(n_accept, 4) ||
        !aligned(out_tok, 4))
        return DFLASH2_EALIGN;
    const int64_t S = n_chunks(V);
    const int64_t units = (int64_t)B * (G + 1) * S;
    if (units > (int64_t)INT32_MAX) return DFLASH2_ESHAPE;
    const Layout L = greedy_layout(B, G, V);
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return DFLASH2_EWORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned* counters = (unsigned*)((char*)ws + L.counters_off);
    uint64_t* part = (uint64_t*)((char*)ws + L.part_off);
    if (cudaMemsetAsync(counters, 0, (size_t)B * 4, s) != cudaSuccess) return DFLASH2_ECUDA;
    // TMA bulk copies need 16-byte aligned chunk starts and 16-byte multiples
    const bool tma = aligned(target, 16) && (V * es) % 16 == 0;
#define DFL_GREEDY(BF, TM)                                                                      \
    do {                                                                                        \
        auto kern = verify_greedy_kernel<BF, TM>;                                               \
        const size_t dyn = TM ? 2 * (size_t)CHUNK * (BF ? 2 : 4) : 0;                           \
        if (prep_stream_kernel(kern, dyn) != DFLASH2_OK) return DFLASH2_ECUDA;                  \
        kern<<<persistent_grid(kern, NT, dyn, units), NT, dyn, s>>>(target, G, V, (int)S, units, \
                                                                  draft_tok, n_accept, out_tok, \
                                                                  part, counters);              \
    } while (0)
    if (dtype == DFLASH2_BF16) {
        if (tma) DFL_GREEDY(true, true);
        else DFL_GREEDY(true, false);
    } else {
        if (tma) DFL_GREEDY(false, true);
        else DFL_GREEDY(false, false);
    }
#undef DFL_GREEDY
    return launch_status();
}

extern "C" int dflash2_verify_sample(const void* target, const void* draft, int dtype, int B, int G,
                                     int64_t V, const int32_t* draft_tok, float inv_temperature,
                                     uint64_t seed, uint32_t step, const uint32_t* seq_id,
                                     int q_mode, int32_t* n_accept, int32_t* out_tok,
                                     float* ratio_dbg, float* u_dbg, void* ws, size_t ws_bytes,
                                     dflash2_stream_t stream) {
    if (!dtype_ok(dtype)) return DFLASH2_EDTYPE;
    if (B < 0 || G < 1 || G >= DFLASH2_MAX_BLOCK || V < 1 || V > INT32_MAX) return DFLASH2_ESHAPE;
    if (!finite_pos(inv_temperature)) return DFLASH2_EINVAL;
    if (q_mode != DFLASH2_Q_SOFTMAX && q_mode != DFLASH2_Q_ONEHOT) return DFLASH2_EINVAL;
    if (B == 0) return DFLASH2_OK;
    if (!target || !draft_tok || !n_accept || !out_tok) return DFLASH2_EINVAL;
    if (q_mode == DFLASH2_Q_SOFTMAX && !draft) return DFLASH2_EINVAL;
    const int es = elem_size(dtype);
    if (!aligned(target, es) || (draft && !aligned(draft, es)) || !aligned(draft_tok, 4) ||
        !aligned(n_accept, 4) || !aligned(out_tok, 4) || (seq_id && !aligned(seq_id, 4)) ||
        (ratio_dbg && !aligned(ratio_dbg, 4)) || (u_dbg && !aligned(u_dbg, 4)))
        return DFLASH2_EALIGN;
    const int64_t S = n_chunks(V);
    if (S > DRAW_MAX_CHUNKS) return DFLASH2_ESHAPE;
    const int rows_per_seq = (q_mode == DFLASH2_Q_SOFTMAX) ? 2 * G + 1 : G + 1;
    const int64_t units = (int64_t)B * rows_per_seq * S;
    if (units > (int64_t)INT32_MAX) return DFLASH2_ESHAPE;
    const Layout L = sample_layout(B, G, V);
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return DFLASH2_EWORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned* counters = (unsigned*)((char*)ws + L.counters_off);
    LseD* part = (LseD*)((char*)ws + L.part_off);
    SampleInfo* info = (SampleInfo*)((char*)ws + L.info_off);
    if (cudaMemsetAsync(counters, 0, (size_t)B * 4, s) != cudaSuccess) return DFLASH2_ECUDA;
    const void* q = (q_mode == DFLASH2_Q_SOFTMAX) ? draft : nullptr;
    const bool tma = aligned(target, 16) && (!q || aligned(q, 16)) && (V * es) % 16 == 0;
    const float c2 = (float)((double)inv_temperature * LOG2E);
    const size_t dyn2 = draw_smem(es, S);
#define DFL_SAMPLE(BF, TM)                                                                        \
    do {                                                                                          \
        auto kern = verify_sample_scan_kernel<BF, TM>;                                            \
        const size_t dyn = TM ? 2 * (size_t)CHUNK * (BF ? 2 : 4) : 0;                             \
        if (prep_stream_kernel(kern, dyn) != DFLASH2_OK) return DFLASH2_ECUDA;                    \
        kern<<<persistent_grid(kern, NT, dyn, units), NT, dyn, s>>>(                              \
            target, q, G, V, (int)S, rows_per_seq, units, inv_temperature, c2, draft_tok, seed,   \
            step, seq_id, q_mode, n_accept, out_tok, ratio_dbg, u_dbg, part, info, counters);     \
        auto kern2 = verify_sample_draw_kernel<BF, TM>;                                           \
        const int cl = draw_cluster(kern2, dyn2, draw_smem((BF ? 2 : 4), DRAW_MAX_CHUNKS), (int)S); \
        if (cl < 1) return DFLASH2_ECUDA;                                                         \
        if (launch_cluster(kern2, B * cl, cl, dyn2, s, target, q, G, V, (int)S, c2,               \
                           inv_temperature, (const SampleInfo*)info, out_tok) != DFLASH2_OK)      \
            return DFLASH2_ECUDA;                                                                 \
    } while (0)
    if (dtype == DFLASH2_BF16) {
        if (tma) DFL_SAMPLE(true, true);
        else DFL_SAMPLE(true, false);
    } else {
        if (tma) DFL_SAMPLE(false, true);
        else DFL_SAMPLE(false, false);
    }
#undef DFL_SAMPLE
    return launch_status();
}
