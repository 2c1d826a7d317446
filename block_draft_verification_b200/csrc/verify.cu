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
// Both verifies stream every logit row once, in chunks of 8 KB: work unit =
// (sequence, row, chunk), one CTA per SM over a contiguous range of units,
// each warp bringing its own chunks in with TMA bulk copies and reducing them
// (ring.cuh).  A unit's partial is published with one acquire-release add on
// its sequence's counter; the warp whose add completes the sequence (no warp
// waits) reduces the partials in chunk order and decides.  The sampling draw
// needs the normalisers first; it runs in the same launch: a warp done with
// its scan units takes draw units of the sequences that have finished (a
// queue in finishing order), half a chunk of the row the sequence draws from
// each, and the warp completing a sequence's draw units walks the inverse
// CDF to t = u' * R.  No probability vector is ever written to memory.
#include "common.cuh"
#include "greedy.cuh"
#include "ring.cuh"
#include "workspace.cuh"

#include <algorithm>
#include <mutex>

namespace dfl {

constexpr double LOG2E = 1.4426950408889634;

// ------------------------------------------------------------------ greedy
// Units (sequence b, row j, chunk): one CTA per SM over a contiguous range,
// each warp a contiguous part of it streamed through its own ring slots; a
// warp publishes its consecutive units of one sequence together, and the
// warp whose add completes the sequence decides it.
template <bool BF16, bool TMA>
__global__ void __launch_bounds__(RING_THREADS, 1) verify_greedy_kernel(
    const void* __restrict__ target, int G, int64_t V, int S, int64_t units,
    const int32_t* __restrict__ draft_tok, int32_t* __restrict__ n_accept,
    int32_t* __restrict__ out_tok, uint64_t* __restrict__ part, unsigned* __restrict__ counters) {
    constexpr int ES = BF16 ? 2 : 4;
    constexpr int LEN = chunk_len(ES);
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ __align__(8) uint64_t bars[2 * NCW];
    const int lane = threadIdx.x & 31;
    int64_t lo, hi;
    warp_range(units, lo, hi);
    const int n = (int)(hi - lo);
    UnitCursor uc, ic;  // (sequence, target row, chunk) being reduced / to bring in
    uc.init(lo, S, G + 1);
    ic = uc;
    auto src = [&](const UnitCursor& cu, const char*& p, uint32_t& bytes) {
        const int64_t v0 = (int64_t)cu.c * LEN;
        p = (const char*)target + ((cu.g * (G + 1) + cu.r) * V + v0) * ES;
        bytes = (uint32_t)(min((int64_t)LEN, V - v0) * ES);
    };
    WarpRing r{nullptr, 0u};
    if (TMA) r = warp_ring_start(ring, bars, n, ic, ChunkT<BF16>::NEG_INF_WORD, src);
    unsigned seg = 0;
    for (int k = 0; k < n; ++k, uc.next()) {
        const int64_t b = uc.g, v0 = (int64_t)uc.c * LEN;
        const int64_t row = b * (G + 1) + uc.r;
        const int len = (int)min((int64_t)LEN, V - v0);
        uint64_t key;
        if (TMA) {
            if (!r.wait(k)) {
                warp_ring_abort(r, k, n);
                return;
            }
            key = greedy_chunk<BF16>(SmemView<BF16>{r.slot(k), v0, len});
            warp_ring_next(r, k, n, ic, ChunkT<BF16>::NEG_INF_WORD, src);
        } else {
            key = greedy_chunk<BF16>(GlobalView<BF16>{(const uint8_t*)target + row * V * ES, v0, len});
        }
        ++seg;
        if (lane == 0) part[row * S + uc.c] = key;
        if (k + 1 == n || uc.last_of_group()) {  // done with this sequence: publish
            bool last = false;
            if (lane == 0) last = publish(&counters[b], seg, (unsigned)((G + 1) * S));
            if (__shfl_sync(FULL, last, 0)) {
                __syncwarp();  // lane 0's acquire covers the whole warp's reads
                greedy_finish(part + b * (G + 1) * S, S, G, V, (int)b, draft_tok, n_accept, out_tok);
                if (lane == 0) counters[b] = 0u;  // the sequence is done: leave its counter zero
            }
            seg = 0;
        }
    }
}

// ------------------------------------------------------------------ sampling, the scan
// (maximum, fp64 sum of exp2((x - maximum) c)) of rows r0 .. r0+7 (the first
// nrows of them) from their S chunk partials (chunk maximum m, sum of
// exp2(x c - fl(m c))), lane-parallel: lanes 4j .. 4j+3
// take row r0 + j, lane 4j + s its chunks s, s + 4, ... (the first 4 RC of
// them held in registers, so a row of up to 4 RC chunks is read once); the
// maximum, then the fp64 sum against it in chunk order; two butterfly steps
// within the four lanes.  Every lane of group j returns row r0 + j's pair.
constexpr int RC = 12;
__device__ __forceinline__ void rows_lse8(const LseD* P, int S, int r0, int nrows, float c2,
                                          float& Mo, double& So) {
    const int lane = threadIdx.x & 31, j = lane >> 2, sub = lane & 3;
    const bool on = j < nrows;
    const LseD* p = P + (int64_t)(r0 + (on ? j : 0)) * S;
    float pm[RC];
    double ps[RC];
#pragma unroll
    for (int i = 0; i < RC; ++i) {
        const int c = sub + 4 * i;
        pm[i] = -INFINITY;
        ps[i] = 0.0;
        if (on && c < S) {
            pm[i] = __ldcg(&p[c].m);
            ps[i] = __ldcg(&p[c].s);
        }
    }
    float M = -INFINITY;
#pragma unroll
    for (int i = 0; i < RC; ++i) M = fmaxf(M, pm[i]);
    if (on)
        for (int c = sub + 4 * RC; c < S; c += 4) M = fmaxf(M, __ldcg(&p[c].m));
    M = fmaxf(M, __shfl_xor_sync(FULL, M, 1));
    M = fmaxf(M, __shfl_xor_sync(FULL, M, 2));
    double t = 0.0;
    if (M != -INFINITY) {
        // a chunk's sum is against fl(m c2); M c2 is exact in fp64
        const double Mc = (double)M * (double)c2;
#pragma unroll
        for (int i = 0; i < RC; ++i)
            if (pm[i] != -INFINITY) t += ps[i] * exp2((double)(pm[i] * c2) - Mc);
        if (on)
            for (int c = sub + 4 * RC; c < S; c += 4) {
                const float m = __ldcg(&p[c].m);
                if (m != -INFINITY) t += __ldcg(&p[c].s) * exp2((double)(m * c2) - Mc);
            }
    }
    t += __shfl_xor_sync(FULL, t, 1);
    t += __shfl_xor_sync(FULL, t, 2);
    Mo = M;
    So = t;
}

// The accept tests of one sequence, by the warp whose unit completed it:
// lane j takes target row j (and draft row j) from the chunk partials.
__device__ __forceinline__ void sample_finish(
    const void* __restrict__ target, const void* __restrict__ draft, const LseD* P, int G,
    int64_t V, int S, int es, float inv_t, float c2, const int32_t* __restrict__ draft_tok,
    uint64_t seed, uint32_t step, uint32_t sid, int q_mode, int b, int32_t* __restrict__ n_accept,
    int32_t* __restrict__ out_tok, float* __restrict__ ratio_dbg, float* __restrict__ u_dbg,
    SampleInfo* __restrict__ info, const float* __restrict__ q_max, const float* __restrict__ q_lse) {
    const int lane = threadIdx.x & 31;
    auto elem = [&](const void* base, int64_t row, int32_t v) -> double {
        if (es == 2)
            return (double)__uint_as_float((uint32_t)((const uint16_t*)base)[row * V + v] << 16);
        return (double)((const float*)base)[row * V + v];
    };
    // the drafted tokens and their logits first (independent of the partials)
    const int32_t dn = (lane < G) ? draft_tok[(int64_t)b * G + lane] : -1;
    // a drafted token outside [0, V) is rejected (r = 0) without a load, and flagged
    const bool dn_ok = lane < G && (uint32_t)dn < (uint32_t)V;
    if (lane < G && !dn_ok) atomicOr(&g_dev_err, ERR_INPUT);
    double xt_d = 0.0, xq_d = 0.0;
    if (dn_ok) {
        xt_d = elem(target, (int64_t)b * (G + 1) + lane, dn);
        if (q_mode == DFLASH2_Q_SOFTMAX) xq_d = elem(draft, (int64_t)b * G + lane, dn);
    }
    // lane j: (max, sum-exp) of target row j, and the draft row's max and
    // ln sum-exp: from its partials, or as given (rows scanned: target only)
    LseD lt{-INFINITY, 0.0f, 0.0}, lq{-INFINITY, 0.0f, 0.0};
    double lnq = 0.0;
    const bool given = q_mode == DFLASH2_Q_SOFTMAX && q_max != nullptr;
    if (given && lane < G) {
        lq.m = q_max[(int64_t)b * G + lane];
        lnq = (double)q_lse[(int64_t)b * G + lane];
    }
    const bool scan_q = q_mode == DFLASH2_Q_SOFTMAX && !given;
    const int nrows = scan_q ? 2 * G + 1 : G + 1;
    for (int r0 = 0; r0 < nrows; r0 += 8) {
        float Mr;
        double Sr;
        rows_lse8(P, S, r0, min(8, nrows - r0), c2, Mr, Sr);
        // lane j takes target row j (and draft row j, row G + 1 + j) from group row - r0
        const int jt = lane - r0, jq = lane + G + 1 - r0;
        const float mt_ = __shfl_sync(FULL, Mr, 4 * (jt & 7));
        const double st_ = __shfl_sync(FULL, Sr, 4 * (jt & 7));
        if (lane <= G && jt >= 0 && jt < 8) lt = LseD{mt_, 0.0f, st_};
        if (scan_q) {
            const float mq_ = __shfl_sync(FULL, Mr, 4 * (jq & 7));
            const double sq_ = __shfl_sync(FULL, Sr, 4 * (jq & 7));
            if (lane < G && jq >= 0 && jq < 8) lq = LseD{mq_, 0.0f, sq_};
        }
    }
    if (scan_q && lane < G) lnq = log(lq.s);
    bool reject = false;
    if (lane < G) {
        // lp = z_t[d] - logZ_t = (x - m) * invT - ln(s); likewise lq
        double lr = (xt_d - (double)lt.m) * (double)inv_t - log(lt.s);
        if (q_mode == DFLASH2_Q_SOFTMAX) lr -= (xq_d - (double)lq.m) * (double)inv_t - lnq;
        const double ratio = dn_ok ? exp(lr) : 0.0;
        const float u = philox_uniform(seed, step, sid, (uint32_t)lane, 0u);
        reject = !((double)u < ratio);
        if (ratio_dbg) ratio_dbg[(int64_t)b * G + lane] = (float)ratio;
        if (u_dbg) u_dbg[(int64_t)b * G + lane] = u;
    }
    const unsigned rej = __ballot_sync(FULL, reject);
    const int n = rej ? (__ffs(rej) - 1) : G;
    if (lane <= G && lane != n) out_tok[(int64_t)b * (G + 1) + lane] = (lane < n) ? dn : -1;
    const float ltm = __shfl_sync(FULL, lt.m, n);
    const double lts = __shfl_sync(FULL, lt.s, n);
    const float lqm = __shfl_sync(FULL, lq.m, n);
    const double lqn = __shfl_sync(FULL, lnq, n);
    const int32_t d_n = __shfl_sync(FULL, dn, n);
    if (lane == 0) {
        SampleInfo I;
        const bool resid = n < G && q_mode == DFLASH2_Q_SOFTMAX;
        I.mt = ltm;
        I.l2t = (float)log2(lts);
        I.mq = lqm;
        I.l2q = resid ? (float)(lqn * 1.4426950408889634) : 0.0f;
        I.dl = resid ? (float)(((double)ltm - (double)lqm) * (double)inv_t + log(lts) - lqn) : 0.0f;
        I.u_res = philox_uniform(seed, step, sid, (uint32_t)n, 1u);
        I.n = n;
        I.mode = (n == G) ? 2 : (q_mode == DFLASH2_Q_SOFTMAX ? 0 : 1);
        I.d = d_n;
        I.pad = 0;
        info[b] = I;
        n_accept[b] = n;
    }
}

// ------------------------------------------------------------------ sampling, the draw
// A sequence draws from one row (target row n, with draft row n for the
// residual).  The row is cut into draw units of half a scan chunk (a unit
// fills half a ring slot), and lane l of the warp that takes a unit owns its
// vectors DRAW_NVL l .. DRAW_NVL l + DRAW_NVL - 1: a contiguous run of the
// row in index order.  Per unit the lanes' inclusive prefix sums of their
// weights are stored (fp64, lane order); units in row order, lanes in unit
// order and elements in run order give the inverse CDF the draw walks.
//
// Draw weight of one element:
//   p_v = exp2((x_v - mt) * c - l2t),  q_v likewise,
//   mode 0: w = max(0, p - q).  With d = ln p - ln q = (xt - xq) * invT -
//           (logZ_t - logZ_q): w = 0 for d <= 0; for 0 < d <= 1/8,
//           w = q * (e^d - 1) (the same value, without the cancellation of
//           p - q when p and q agree); above, w = p - q directly (p > 1.13 q:
//           the subtraction costs at most three bits; q = 0 gives p);
//   mode 1: w = p, 0 at d;  mode 2: w = p (also the fallback when the
//   residual is empty by rounding).
// e^d - 1 for 0 < d <= 1/8: the Taylor series to d^5 (truncation below
// 5e-8 relative there).
// A draw unit is half a scan chunk: DRAW_NVL 16-byte vectors per lane, so a
// row's draw work spreads over twice as many warps (most warps are idle by
// the time the last sequences are decided).
constexpr int DRAW_NVL = NVL / 2;
template <bool BF16>
__host__ __device__ constexpr int draw_len() { return 32 * DRAW_NVL * ChunkT<BF16>::VW; }
__host__ __device__ inline int64_t draw_units(int64_t V, int es) {
    const int64_t len = (int64_t)32 * DRAW_NVL * (16 / es);
    return (V + len - 1) / len;
}
constexpr float EXPM1_SPLIT = 0.125f;
__device__ __forceinline__ float expm1_small(float d) {
    float p = 1.0f / 120.0f;
    p = fmaf(p, d, 1.0f / 24.0f);
    p = fmaf(p, d, 1.0f / 6.0f);
    p = fmaf(p, d, 0.5f);
    p = fmaf(p, d, 1.0f);
    return p * d;
}

// The weights of one 16-byte vector (first element index i0); -inf elements
// (past the row) weigh 0 in every mode.  RESID: mode 0; else p, with the
// element at index excl (mode 1's d; -1 for mode 2) weighing 0.
template <bool BF16, bool RESID>
__device__ __forceinline__ void draw_vec(const uint4& xt, const uint4& xq, int64_t i0,
                                         const SampleInfo& I, int64_t excl, float c2, float inv_t,
                                         float (&w)[ChunkT<BF16>::VW]) {
    using C = ChunkT<BF16>;
#pragma unroll
    for (int e = 0; e < C::VW; ++e) {
        const float t = C::elem(xt, e);
        if (RESID) {  // both exponentials always, then selects: no branch per element
            const float q = C::elem(xq, e);
            const float dlog = (t - q) * inv_t - I.dl;
            const float qv = ex2((q - I.mq) * c2 - I.l2q);
            const float pv = ex2((t - I.mt) * c2 - I.l2t);
            const float near = qv * expm1_small(fminf(dlog, EXPM1_SPLIT));
            const float r = (dlog > EXPM1_SPLIT) ? pv - qv : near;
            w[e] = (dlog > 0.0f) ? r : 0.0f;
        } else {
            const float pv = ex2((t - I.mt) * c2 - I.l2t);
            w[e] = (i0 + e == excl) ? 0.0f : pv;
        }
    }
}
template <bool BF16>
__device__ __forceinline__ void draw_vec(int mode, const uint4& xt, const uint4& xq, int64_t i0,
                                         const SampleInfo& I, float c2, float inv_t,
                                         float (&w)[ChunkT<BF16>::VW]) {
    if (mode == 0) draw_vec<BF16, true>(xt, xq, i0, I, -1, c2, inv_t, w);
    else draw_vec<BF16, false>(xt, xq, i0, I, mode == 1 ? (int64_t)I.d : -1, c2, inv_t, w);
}

// This lane's weight sum over its run of a unit: fp32 pairwise within a
// vector, fp64 across the run's vectors.  The lanes of a warp read the run's
// vectors in rotated order (lane l starts at its vector l mod DRAW_NVL), so the
// 16-byte reads of a quarter-warp fall in distinct banks; the order is fixed
// per lane, so the sum is the same bits in any batch.
template <bool BF16, bool RESID, class View>
__device__ __forceinline__ double draw_lane_sum(const View& vt, const View& vq,
                                                const SampleInfo& I, int64_t excl, float c2,
                                                float inv_t) {
    using C = ChunkT<BF16>;
    const int lane = threadIdx.x & 31;
    double s = 0.0;
#pragma unroll 2
    for (int g = 0; g < DRAW_NVL; ++g) {
        const int q = DRAW_NVL * lane + ((g + lane) & (DRAW_NVL - 1));
        const uint4 xt = vt.vec(q);
        const uint4 xq = RESID ? vq.vec(q) : make_uint4(0u, 0u, 0u, 0u);
        float w[C::VW];
        draw_vec<BF16, RESID>(xt, xq, vt.index(q, 0), I, excl, c2, inv_t, w);
#pragma unroll
        for (int h = C::VW / 2; h > 0; h >>= 1)
#pragma unroll
            for (int e = 0; e < h; ++e) w[e] += w[e + h];
        s += (double)w[0];
    }
    return s;
}
template <bool BF16, class View>
__device__ __forceinline__ double draw_lane_sum(const View& vt, const View& vq, int mode,
                                                const SampleInfo& I, float c2, float inv_t) {
    if (mode == 0) return draw_lane_sum<BF16, true>(vt, vq, I, -1, c2, inv_t);
    return draw_lane_sum<BF16, false>(vt, vq, I, mode == 1 ? (int64_t)I.d : -1, c2, inv_t);
}

// Inclusive warp scan (fp64, lane order).
__device__ __forceinline__ double warp_incl_scan(double x) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 1; k < 32; k <<= 1) {
        const double o = __shfl_up_sync(FULL, x, k);
        if (lane >= k) x += o;
    }
    return x;
}

// A row read straight from global memory as the vectors of a unit starting
// at element v0: AL (16-byte aligned rows, V * es a multiple of 16) reads
// whole vectors, else element by element; elements past V read as -inf.
template <bool BF16, bool AL>
struct RowView {
    using C = ChunkT<BF16>;
    const char* row;
    int64_t v0, V;
    __device__ __forceinline__ uint4 vec(int q) const {
        const int64_t i0 = v0 + (int64_t)q * C::VW;
        if (AL && i0 + C::VW <= V) return __ldg((const uint4*)(row + i0 * C::ES));
        const GlobalView<BF16> g{(const uint8_t*)row, i0,
                                 (int)max((int64_t)0, min((int64_t)C::VW, V - i0))};
        return g.vec(0);
    }
    __device__ __forceinline__ int64_t index(int q, int e) const { return v0 + (int64_t)q * C::VW + e; }
};

// The walk inside the run holding t (first element rb, inverse CDF `base`
// before it): lane j < DRAW_NVL takes the run's vector j, the vector sums go
// through an inclusive warp scan, and the first lane with mass whose prefix
// exceeds t walks its elements to the first whose running prefix exceeds t
// (else its last element with mass; if no lane crosses, the run's last
// element with mass).  Returns the element index on every lane (-1: no mass).
template <bool BF16, bool AL>
__device__ __forceinline__ int64_t draw_walk(const char* trow, const char* qrow, int64_t V,
                                             int mode, const SampleInfo& I, float c2, float inv_t,
                                             int64_t rb, double base, double tt) {
    using C = ChunkT<BF16>;
    const int lane = threadIdx.x & 31;
    float w[C::VW];
    double sj = 0.0;
    const int64_t i0 = rb + (int64_t)lane * C::VW;
    if (lane < DRAW_NVL) {
        const RowView<BF16, AL> vt{trow, i0, V}, vq{qrow, i0, V};
        const uint4 xt = vt.vec(0);
        const uint4 xq = (mode == 0) ? vq.vec(0) : make_uint4(0u, 0u, 0u, 0u);
        draw_vec<BF16>(mode, xt, xq, i0, I, c2, inv_t, w);
#pragma unroll
        for (int e = 0; e < C::VW; ++e) sj += (double)w[e];
    } else {
#pragma unroll
        for (int e = 0; e < C::VW; ++e) w[e] = 0.0f;
    }
    const double incl = warp_incl_scan(sj);
    const unsigned mass = __ballot_sync(FULL, sj > 0.0);
    const unsigned cross = __ballot_sync(FULL, base + incl > tt) & mass;
    if (!mass) return -1;
    const int src = cross ? __ffs(cross) - 1 : 31 - __clz(mass);
    int64_t pick = -1;
    if (lane == src) {
        double run = base + incl - sj;
        int first = -1, last = -1;
#pragma unroll
        for (int e = 0; e < C::VW; ++e) {
            if (w[e] > 0.0f) last = e;
            run += (double)w[e];
            if (first < 0 && run > tt && cross) first = e;
        }
        pick = i0 + (first >= 0 ? first : last);
    }
    return __shfl_sync(FULL, pick, src);
}

// The draw from p_n when the residual is empty by rounding (rare): the warp
// sums the mode-2 weights of every unit's runs itself, twice (R, then the
// crossing of t = u' R), and locates the run.  False if the row has no mass.
template <bool BF16, bool AL>
__device__ __noinline__ bool draw_locate_p(const char* trow, int64_t V, int ND,
                                           const SampleInfo& I, float c2, float inv_t,
                                           int& cstar, int& lstar, double& base, double& tt) {
    using C = ChunkT<BF16>;
    double R = 0.0;
    for (int c = 0; c < ND; ++c) {
        const RowView<BF16, AL> v{trow, (int64_t)c * draw_len<BF16>(), V};
        const double my = draw_lane_sum<BF16>(v, v, 2, I, c2, inv_t);
        R = __shfl_sync(FULL, warp_incl_scan(my) + R, 31);
    }
    if (!(R > 0.0)) return false;
    tt = (double)I.u_res * R;
    double carry = 0.0;
    int lastc = -1, lastl = -1;
    double last_base = 0.0;
    for (int c = 0; c < ND; ++c) {
        const RowView<BF16, AL> v{trow, (int64_t)c * draw_len<BF16>(), V};
        const double my = draw_lane_sum<BF16>(v, v, 2, I, c2, inv_t);
        const double incl = warp_incl_scan(my) + carry;
        const unsigned mass = __ballot_sync(FULL, my > 0.0);
        const unsigned cross = __ballot_sync(FULL, incl > tt) & mass;
        if (cross) {
            cstar = c;
            lstar = __ffs(cross) - 1;
            base = __shfl_sync(FULL, incl - my, lstar);
            return true;
        }
        if (mass) {
            lastc = c;
            lastl = 31 - __clz(mass);
            last_base = __shfl_sync(FULL, incl - my, lastl);
        }
        carry = __shfl_sync(FULL, incl, 31);
    }
    cstar = lastc;  // rounding left t at or above the total
    lstar = lastl;
    base = last_base;
    return true;
}

// The pick of one sequence, by the warp whose draw unit completed it.
// R = the unit totals in unit order (fp64 inclusive scan), t = u' R; the
// first unit whose inclusive prefix exceeds t, in it the first lane with mass
// whose prefix exceeds t (from the stored prefixes), then the walk in that
// lane's run.  R = 0 (the residual empty by rounding) redraws from p_n.
// Writes out_tok[n] (-1 if the row has no mass at all; nothing if out is
// null).
template <bool BF16, bool AL>
__device__ __noinline__ void draw_pick(const char* trow, const char* qrow, int64_t V, int ND,
                                       SampleInfo I, float c2, float inv_t,
                                       const double* __restrict__ P, int32_t* __restrict__ out) {
    using C = ChunkT<BF16>;
    const int lane = threadIdx.x & 31;
    int mode = I.mode;
    // the unit totals (each unit's last lane prefix): rows of up to 32 PT
    // units are loaded once, into registers; longer ones are read per pass
    constexpr int PT = 4;
    double tot[PT], incl[PT];
    double R = 0.0;
    const bool held = ND <= 32 * PT;
    if (held) {
#pragma unroll
        for (int k = 0; k < PT; ++k) {
            const int c = 32 * k + lane;
            tot[k] = (c < ND) ? __ldcg(&P[(int64_t)c * 32 + 31]) : 0.0;
        }
#pragma unroll
        for (int k = 0; k < PT; ++k) {
            incl[k] = warp_incl_scan(tot[k]) + R;
            R = __shfl_sync(FULL, incl[k], 31);
        }
    } else {
        for (int c0 = 0; c0 < ND; c0 += 32) {
            const int c = c0 + lane;
            const double cs = (c < ND) ? __ldcg(&P[(int64_t)c * 32 + 31]) : 0.0;
            R = __shfl_sync(FULL, warp_incl_scan(cs) + R, 31);
        }
    }
    int cstar = -1, lstar = -1;
    double base = 0.0, tt = 0.0;
    if (R > 0.0) {
        tt = (double)I.u_res * R;
        double pre = 0.0, lastc_pre = 0.0;
        int lastc = -1;
        // the first unit with mass whose inclusive prefix exceeds t, and the
        // last unit with mass (for t at or above R by rounding)
        auto look = [&](int c0, double cs, double in) {
            const unsigned mass = __ballot_sync(FULL, cs > 0.0);
            const unsigned cross = __ballot_sync(FULL, in > tt) & mass;
            if (mass) {
                const int l = 31 - __clz(mass);
                lastc = c0 + l;
                lastc_pre = __shfl_sync(FULL, in - cs, l);
            }
            if (cross && cstar < 0) {
                const int l = __ffs(cross) - 1;
                cstar = c0 + l;
                pre = __shfl_sync(FULL, in - cs, l);
            }
        };
        if (held) {
#pragma unroll
            for (int k = 0; k < PT; ++k) look(32 * k, tot[k], incl[k]);
        } else {
            double carry = 0.0;
            for (int c0 = 0; c0 < ND && cstar < 0; c0 += 32) {
                const int c = c0 + lane;
                const double cs = (c < ND) ? __ldcg(&P[(int64_t)c * 32 + 31]) : 0.0;
                const double in = warp_incl_scan(cs) + carry;
                look(c0, cs, in);
                carry = __shfl_sync(FULL, in, 31);
            }
        }
        if (cstar < 0) {  // rounding left t at or above R: the last unit with mass
            cstar = lastc;
            pre = lastc_pre;
        }
        const double li = __ldcg(&P[(int64_t)cstar * 32 + lane]);
        double lp = __shfl_up_sync(FULL, li, 1);
        if (lane == 0) lp = 0.0;
        const unsigned mass = __ballot_sync(FULL, li > lp);
        const unsigned cross = __ballot_sync(FULL, pre + li > tt) & mass;
        lstar = cross ? __ffs(cross) - 1 : (mass ? 31 - __clz(mass) : -1);
        if (lstar >= 0) base = pre + __shfl_sync(FULL, lp, lstar);
    } else {
        mode = 2;
        if (!draw_locate_p<BF16, AL>(trow, V, ND, I, c2, inv_t, cstar, lstar, base, tt)) lstar = -1;
    }
    int64_t pick = -1;
    if (lstar >= 0)
        pick = draw_walk<BF16, AL>(trow, qrow, V, mode, I, c2, inv_t,
                                   (int64_t)cstar * draw_len<BF16>() + (int64_t)lstar * DRAW_NVL * C::VW,
                                   base, tt);
    if (lane == 0 && out) *out = (int32_t)pick;
}

// One pick on a scratch table of 32 lane prefixes 1 .. 32 (one unit, target
// row 0 for both rows, a residual of zero mass), and with rings one draw sum
// over the warp's slots: the same code as the real ones, run early by an
// idle warp so it is fetched into L2 while no pick waits on it.  Writes only
// the scratch table; reads only row 0 and the warp's own slots.
template <bool BF16, bool TMA>
__device__ __noinline__ void warm_draw_code(const void* target, int64_t V, float c2, float inv_t,
                                            double* scratch, WarpRing r) {
    const int lane = threadIdx.x & 31;
    SampleInfo I;
    I.mt = I.l2t = I.mq = I.l2q = I.dl = 0.0f;
    I.u_res = 0.5f;
    I.n = I.mode = I.d = I.pad = 0;
    double my = 0.0;
    if (TMA) {
        const SmemView<BF16> v{r.slot(0), 0, draw_len<BF16>()};
        my = draw_lane_sum<BF16, true>(v, v, I, -1, c2, inv_t);
    }
    scratch[lane] = (double)(lane + 1) + 0.0 * my;
    __syncwarp();
    draw_pick<BF16, TMA>((const char*)target, (const char*)target, V, 1, I, c2, inv_t, scratch,
                         nullptr);
}

// The per-sequence hand-over from the scan to the draw, read in L2 (written
// by another SM in this launch).
__device__ __forceinline__ SampleInfo load_info(const SampleInfo* p) {
    SampleInfo I;
    I.mt = __ldcg(&p->mt);
    I.l2t = __ldcg(&p->l2t);
    I.mq = __ldcg(&p->mq);
    I.l2q = __ldcg(&p->l2q);
    I.dl = __ldcg(&p->dl);
    I.u_res = __ldcg(&p->u_res);
    I.n = __ldcg(&p->n);
    I.mode = __ldcg(&p->mode);
    I.d = __ldcg(&p->d);
    I.pad = 0;
    return I;
}

// Sampling verify in one cooperative launch (every CTA resident).
//
// Scan: units are (sequence b, row rr, chunk): rows 0..G of a sequence are
// its target rows, G+1..2G its draft rows (when their normalisers are not
// given).  A unit's partial is the chunk maximum and the fp64 sum of
// exp2((x - m) c) against it; a warp publishes its consecutive units of one
// sequence together, and the warp whose add completes the sequence decides
// its accept tests and appends it to the finish queue.
//
// Draw: draw unit i is (position i / ND in the finish queue, unit i % ND of
// the row), and CTA c takes units c, c + grid, c + 2 grid, ... in that order
// (a shared-memory counter hands them to its warps as they run out of scan
// units), so every SM draws the same share.  A warp waits (bounded) until
// the sequence at that position has finished, brings the unit of target row
// n (and draft row n for the residual) into the two halves of one ring slot,
// and stores its lanes' prefix sums.  The warp whose unit completes a sequence picks the
// token.  No warp waits on a warp that is itself waiting: a sequence
// finishes within the scan, and a warp draws only after its own scan units.
//
// Control words (zero on entry, zero again on exit; sample_ctl_words): the
// queue length and the count of warps done, each in a 128-byte line of its
// own; scan units per sequence [B]; draw units per sequence [B]; then the
// finish queue, one line per position (b + 1 of the sequence that finished
// there), so the warps polling it spread over as many lines and never meet
// the counters' adds.
template <bool BF16, bool TMA>
__global__ void __launch_bounds__(RING_THREADS, 1) verify_sample_kernel(
    const void* __restrict__ target, const void* __restrict__ draft, int B, int G, int64_t V, int S,
    int rows_per_seq, int64_t units, float inv_t, float c2, const int32_t* __restrict__ draft_tok,
    uint64_t seed, uint32_t step, const uint32_t* __restrict__ seq_id, int q_mode,
    int32_t* __restrict__ n_accept, int32_t* __restrict__ out_tok, float* __restrict__ ratio_dbg,
    float* __restrict__ u_dbg, LseD* __restrict__ part, double* __restrict__ dsum,
    SampleInfo* __restrict__ info, unsigned* __restrict__ ctl, const float* __restrict__ q_max,
    const float* __restrict__ q_lse) {
    using C = ChunkT<BF16>;
    constexpr int ES = C::ES;
    constexpr int LEN = C::LEN;
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ __align__(8) uint64_t bars[2 * NCW];
    __shared__ unsigned s_next;  // this CTA's next draw unit (k: unit blockIdx.x + k grid)
    __shared__ unsigned s_warm;  // warps of this CTA done with their scan
    const int lane = threadIdx.x & 31;
    unsigned* const fin_count = ctl;
    unsigned* const retire = ctl + CTL_LINE;
    unsigned* const counters = ctl + 2 * CTL_LINE;
    unsigned* const dcount = counters + B;
    unsigned* const fin = ctl + sample_fin_off(B);
    auto rowp = [&](int64_t b, int rr) {
        return (rr <= G) ? (const char*)target + (b * (G + 1) + rr) * V * ES
                         : (const char*)draft + (b * G + (rr - G - 1)) * V * ES;
    };
    if (threadIdx.x == 0) {
        s_next = 0u;
        s_warm = 0u;
    }
    {  // the accept tests' scattered reads (drafted tokens, their logits) into L2 now
        const int64_t t = (int64_t)blockIdx.x * RING_THREADS + threadIdx.x;
        if (t < (int64_t)B * G) {
            const int64_t b = t / G, j = t - b * G;
            const int32_t d = draft_tok[t];
            if (d >= 0 && d < V) {
                prefetch_l2_last((const char*)target + ((b * (G + 1) + j) * V + d) * ES);
                if (q_mode == DFLASH2_Q_SOFTMAX)
                    prefetch_l2_last((const char*)draft + ((b * G + j) * V + d) * ES);
            }
        }
    }
    __syncthreads();
    int64_t lo, hi;
    warp_range(units, lo, hi);
    const int n = (int)(hi - lo);
    UnitCursor uc, ic;  // (sequence, row, chunk) being reduced / to bring in
    uc.init(lo, S, rows_per_seq);
    ic = uc;
    auto src = [&](const UnitCursor& cu, const char*& p, uint32_t& bytes) {
        const int64_t v0 = (int64_t)cu.c * LEN;
        p = rowp(cu.g, cu.r) + v0 * ES;
        bytes = (uint32_t)(min((int64_t)LEN, V - v0) * ES);
    };
    WarpRing r{nullptr, 0u};
    if (TMA) r = warp_ring_start(ring, bars, n, ic, C::NEG_INF_WORD, src);
    unsigned seg = 0;
    for (int k = 0; k < n; ++k, uc.next()) {
        const int64_t b = uc.g, v0 = (int64_t)uc.c * LEN;
        const int len = (int)min((int64_t)LEN, V - v0);
        float M;
        double Ssum;
        if (TMA) {
            if (!r.wait(k)) {
                warp_ring_abort(r, k, n);
                return;
            }
            const SmemView<BF16> view{r.slot(k), v0, len};
            uint32_t vm[NVL];
            M = warp_max(chunk_pass1<BF16>(view, vm));
            Ssum = chunk_expsum_at_mc<BF16>(view, M, c2);
            warp_ring_next(r, k, n, ic, C::NEG_INF_WORD, src);
        } else {
            const GlobalView<BF16> view{(const uint8_t*)rowp(b, uc.r), v0, len};
            uint32_t vm[NVL];
            M = warp_max(chunk_pass1<BF16>(view, vm));
            Ssum = chunk_expsum_at_mc<BF16>(view, M, c2);
        }
        ++seg;
        if (lane == 0) part[(b * rows_per_seq + uc.r) * S + uc.c] = LseD{M, 0.0f, Ssum};
        if (k + 1 == n || uc.last_of_group()) {  // done with this sequence: publish
            bool last = false;
            if (lane == 0) last = publish(&counters[b], seg, (unsigned)(rows_per_seq * S));
            if (__shfl_sync(FULL, last, 0)) {
                __syncwarp();  // lane 0's acquire covers the whole warp's reads
                sample_finish(target, draft, part + b * rows_per_seq * S, G, V, S, ES, inv_t, c2,
                              draft_tok, seed, step, seq_id ? seq_id[b] : (uint32_t)b, q_mode,
                              (int)b, n_accept, out_tok, ratio_dbg, u_dbg, info, q_max, q_lse);
                if (lane == 0) {  // info[b] (lane 0's store) before the queue entry
                    counters[b] = 0u;
                    st_release(&fin[(size_t)atomicAdd(fin_count, 1u) * CTL_LINE], (unsigned)b + 1u);
                }
            }
            seg = 0;
        }
    }

    // ---- the draw
    const int ND = (int)draw_units(V, ES);  // draw units per row
    constexpr int LEN_D = draw_len<BF16>();
    const unsigned total = (unsigned)B * (unsigned)ND;
    double* const dsum_scratch = dsum + (int64_t)B * ND * 32;  // 32 doubles
    // The first warp of the CTA done with its scan runs the draw sum and the
    // pick once on a scratch table (storing nothing else): their code is then
    // in this SM's instruction cache before the real calls need it.
    {
        unsigned first = 0;
        if (lane == 0) first = atomicAdd(&s_warm, 1u) == 0u;
        if (__shfl_sync(FULL, first, 0))
            warm_draw_code<BF16, TMA>(target, V, c2, inv_t, dsum_scratch, r);
    }
    // Units in queue order, per CTA: unit blockIdx.x + k grid, k from s_next
    // (total: none left).
    auto grab = [&]() -> unsigned {
        unsigned k = 0;
        if (lane == 0) k = atomicAdd(&s_next, 1u);
        k = __shfl_sync(FULL, k, 0);
        const uint64_t i64 = (uint64_t)blockIdx.x + (uint64_t)k * gridDim.x;
        return i64 < total ? (unsigned)i64 : total;
    };
    // A unit's lane prefixes out, and its sequence's pick by the warp whose
    // unit completes the row.
    auto publish_unit = [&](unsigned c, double my, int b, const SampleInfo& I) {
        dsum[((int64_t)b * ND + c) * 32 + lane] = warp_incl_scan(my);
        __syncwarp();  // every lane's prefix before lane 0's release
        bool lastu = false;
        if (lane == 0) lastu = publish(&dcount[b], 1u, (unsigned)ND);
        if (__shfl_sync(FULL, lastu, 0)) {
            __syncwarp();
            const char* trow = (const char*)target + ((int64_t)b * (G + 1) + I.n) * V * ES;
            const char* qrow =
                (I.mode == 0) ? (const char*)draft + ((int64_t)b * G + I.n) * V * ES : nullptr;
            draw_pick<BF16, TMA>(trow, qrow, V, ND, I, c2, inv_t, dsum + (int64_t)b * ND * 32,
                                 &out_tok[(int64_t)b * (G + 1) + I.n]);
            if (lane == 0) dcount[b] = 0u;
        }
    };
    if (TMA) {
        // One unit per ring slot: its target run in the first half, its draft
        // run (residual draws) in the second, both copies on the slot's barrier.
        constexpr uint32_t HALF = (uint32_t)SLOT_BYTES / 2;
        static_assert(LEN_D * ES == (int)HALF, "a draw unit fills half a ring slot");
        int kk = n;  // this warp's next ring unit
        while (true) {
            const unsigned i = grab();
            if (i >= total) break;
            unsigned b1 = 0;
            if (lane == 0) b1 = wait_nonzero(&fin[(size_t)(i / (unsigned)ND) * CTL_LINE]);
            b1 = __shfl_sync(FULL, b1, 0);
            if (b1 == 0u) {  // the bound ran out
                if (lane == 0) atomicOr(&g_dev_err, ERR_STREAM);
                return;
            }
            __syncwarp();  // lane 0's acquire covers the warp's reads of info[b]
            const int b = (int)b1 - 1;
            const SampleInfo I = load_info(&info[b]);
            const unsigned c = i - (i / (unsigned)ND) * (unsigned)ND;
            const int64_t v0 = (int64_t)c * LEN_D;
            const char* trow = (const char*)target + ((int64_t)b * (G + 1) + I.n) * V * ES;
            const char* qrow = (const char*)draft + ((int64_t)b * G + I.n) * V * ES;
            const bool two = I.mode == 0;
            const uint32_t bytes = (uint32_t)(min((int64_t)LEN_D, V - v0) * ES);
            uint8_t* sl = r.slot(kk);
            if (bytes < HALF) {  // past the row: -inf, in both runs
                const uint4 f = make_uint4(C::NEG_INF_WORD, C::NEG_INF_WORD, C::NEG_INF_WORD,
                                           C::NEG_INF_WORD);
                for (uint32_t q = bytes / 16 + lane; q < HALF / 16; q += 32) {
                    ((uint4*)sl)[q] = f;
                    if (two) ((uint4*)(sl + HALF))[q] = f;
                }
                __syncwarp();
            }
            if (lane == 0) {
                const uint32_t bar = r.bar + 8 * (kk & 1);
                mbar_expect_tx(bar, two ? 2 * bytes : bytes);
                bulk_g2s_nx(smem_u32(sl), trow + v0 * ES, bytes, bar);
                if (two) bulk_g2s_nx(smem_u32(sl + HALF), qrow + v0 * ES, bytes, bar);
            }
            __syncwarp();
            if (!r.wait_fresh(kk)) {
                warp_ring_abort(r, kk, kk + 1);
                return;
            }
            const SmemView<BF16> vt{sl, v0, LEN_D}, vq{sl + HALF, v0, LEN_D};
            const double my = draw_lane_sum<BF16>(vt, vq, I.mode, I, c2, inv_t);
            r.done(kk);  // the slot is read: it may be refilled
            ++kk;
            publish_unit(c, my, b, I);
        }
    } else {
        while (true) {
            const unsigned i = grab();
            if (i >= total) break;
            unsigned b1 = 0;
            if (lane == 0) b1 = wait_nonzero(&fin[(size_t)(i / (unsigned)ND) * CTL_LINE]);
            b1 = __shfl_sync(FULL, b1, 0);
            if (b1 == 0u) {  // the bound ran out
                if (lane == 0) atomicOr(&g_dev_err, ERR_STREAM);
                return;
            }
            __syncwarp();  // lane 0's acquire covers the warp's reads of info[b]
            const int b = (int)b1 - 1;
            const SampleInfo I = load_info(&info[b]);
            const unsigned c = i - (i / (unsigned)ND) * (unsigned)ND;
            const int64_t v0 = (int64_t)c * LEN_D;
            const char* trow = (const char*)target + ((int64_t)b * (G + 1) + I.n) * V * ES;
            const char* qrow =
                (I.mode == 0) ? (const char*)draft + ((int64_t)b * G + I.n) * V * ES : nullptr;
            const RowView<BF16, false> vt{trow, v0, V}, vq{qrow, v0, V};
            publish_unit(c, draw_lane_sum<BF16>(vt, vq, I.mode, I, c2, inv_t), b, I);
        }
    }
    // the last warp out leaves the queue words zero (every other warp is past
    // its last access to them)
    bool lastw = false;
    if (lane == 0) lastw = publish(retire, 1u, gridDim.x * (unsigned)NCW);
    if (__shfl_sync(FULL, lastw, 0)) {
        for (int p = lane; p < B; p += 32) fin[(size_t)p * CTL_LINE] = 0u;
        if (lane == 0) {
            *fin_count = 0u;
            *retire = 0u;
        }
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
    const int64_t S = row_chunks(V, es);
    const int64_t units = (int64_t)B * (G + 1) * S;
    if (units > (int64_t)INT32_MAX) return DFLASH2_ESHAPE;
    const Layout L = greedy_layout(B, G, V, es);
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return DFLASH2_EWORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned* counters = (unsigned*)((char*)ws + L.counters_off);
    uint64_t* part = (uint64_t*)((char*)ws + L.part_off);
    if (!L.self_clean && cudaMemsetAsync(counters, 0, (size_t)B * 4, s) != cudaSuccess)
        return DFLASH2_ECUDA;
    // TMA bulk copies need 16-byte aligned chunk starts and 16-byte multiples
    const bool tma = aligned(target, 16) && (V * es) % 16 == 0;
#define DFL_GREEDY(BF, TM)                                                                       \
    do {                                                                                         \
        auto kern = verify_greedy_kernel<BF, TM>;                                                \
        const size_t dyn = TM ? (size_t)RING_BYTES : 0;                                          \
        if (ring_prepare(kern, dyn) != DFLASH2_OK) return DFLASH2_ECUDA;                         \
        kern<<<ring_grid(units), RING_THREADS, dyn, s>>>(target, G, V, (int)S, units, draft_tok, \
                                                         n_accept, out_tok, part, counters);     \
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

static int verify_sample_impl(const void* target, const void* draft, int dtype, int B, int G,
                              int64_t V, const int32_t* draft_tok, const float* q_max,
                              const float* q_lse, float inv_temperature, uint64_t seed,
                              uint32_t step, const uint32_t* seq_id, int q_mode, int32_t* n_accept,
                              int32_t* out_tok, float* ratio_dbg, float* u_dbg, void* ws,
                              size_t ws_bytes, dflash2_stream_t stream) {
    if (!dtype_ok(dtype)) return DFLASH2_EDTYPE;
    if (B < 0 || G < 1 || G >= DFLASH2_MAX_BLOCK || V < 1 || V > INT32_MAX) return DFLASH2_ESHAPE;
    if (!finite_pos(inv_temperature)) return DFLASH2_EINVAL;
    if (q_mode != DFLASH2_Q_SOFTMAX && q_mode != DFLASH2_Q_ONEHOT) return DFLASH2_EINVAL;
    if (B == 0) return DFLASH2_OK;
    if (!target || !draft_tok || !n_accept || !out_tok) return DFLASH2_EINVAL;
    if (q_mode == DFLASH2_Q_SOFTMAX && !draft) return DFLASH2_EINVAL;
    const int es = elem_size(dtype);
    if ((q_max == nullptr) != (q_lse == nullptr)) return DFLASH2_EINVAL;
    if (q_mode != DFLASH2_Q_SOFTMAX) q_max = q_lse = nullptr;  // one-hot q needs no normaliser
    if ((q_max && !aligned(q_max, 4)) || (q_lse && !aligned(q_lse, 4))) return DFLASH2_EALIGN;
    if (!aligned(target, es) || (draft && !aligned(draft, es)) || !aligned(draft_tok, 4) ||
        !aligned(n_accept, 4) || !aligned(out_tok, 4) || (seq_id && !aligned(seq_id, 4)) ||
        (ratio_dbg && !aligned(ratio_dbg, 4)) || (u_dbg && !aligned(u_dbg, 4)))
        return DFLASH2_EALIGN;
    const int64_t S = row_chunks(V, es);
    // draft rows are scanned only when their normalisers are not given
    const int rows_per_seq = (q_mode == DFLASH2_Q_SOFTMAX && !q_max) ? 2 * G + 1 : G + 1;
    const int64_t units = (int64_t)B * rows_per_seq * S;
    if (units > (int64_t)INT32_MAX || B > 65535) return DFLASH2_ESHAPE;
    const Layout L = sample_layout(B, G, V, es);
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return DFLASH2_EWORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned* ctl = (unsigned*)((char*)ws + L.counters_off);  // sample_ctl_words(B)
    LseD* part = (LseD*)((char*)ws + L.part_off);
    double* dsum = (double*)((char*)ws + L.part2_off);
    SampleInfo* info = (SampleInfo*)((char*)ws + L.info_off);
    if (!L.self_clean && cudaMemsetAsync(ctl, 0, L.counters_bytes, s) != cudaSuccess)
        return DFLASH2_ECUDA;
    const void* q = (q_mode == DFLASH2_Q_SOFTMAX) ? draft : nullptr;
    const bool tma = aligned(target, 16) && (!q || aligned(q, 16)) && (V * es) % 16 == 0;
    const float c2 = (float)((double)inv_temperature * LOG2E);
    // cooperative: every CTA is resident, so a warp's bounded wait for a
    // sequence to finish waits on warps that are running
    auto launch = [&](auto kern, size_t dyn) -> int {
        if (ring_prepare(kern, dyn) != DFLASH2_OK) return DFLASH2_ECUDA;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)ring_grid(units));
        cfg.blockDim = dim3(RING_THREADS);
        cfg.dynamicSmemBytes = dyn;
        cfg.stream = s;
        cudaLaunchAttribute a[1];
        a[0].id = cudaLaunchAttributeCooperative;
        a[0].val.cooperative = 1;
        cfg.attrs = a;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, kern, target, q, B, G, V, (int)S, rows_per_seq, units,
                               inv_temperature, c2, draft_tok, seed, step, seq_id, q_mode,
                               n_accept, out_tok, ratio_dbg, u_dbg, part, dsum, info, ctl, q_max,
                               q_lse) != cudaSuccess)
            return DFLASH2_ECUDA;
        return DFLASH2_OK;
    };
    int rc;
    if (dtype == DFLASH2_BF16)
        rc = tma ? launch(verify_sample_kernel<true, true>, RING_BYTES)
                 : launch(verify_sample_kernel<true, false>, 0);
    else
        rc = tma ? launch(verify_sample_kernel<false, true>, RING_BYTES)
                 : launch(verify_sample_kernel<false, false>, 0);
    if (rc != DFLASH2_OK) return rc;
    return launch_status();
}

extern "C" int dflash2_verify_sample(const void* target, const void* draft, int dtype, int B, int G,
                                     int64_t V, const int32_t* draft_tok, float inv_temperature,
                                     uint64_t seed, uint32_t step, const uint32_t* seq_id,
                                     int q_mode, int32_t* n_accept, int32_t* out_tok,
                                     float* ratio_dbg, float* u_dbg, void* ws, size_t ws_bytes,
                                     dflash2_stream_t stream) {
    return verify_sample_impl(target, draft, dtype, B, G, V, draft_tok, nullptr, nullptr,
                              inv_temperature, seed, step, seq_id, q_mode, n_accept, out_tok,
                              ratio_dbg, u_dbg, ws, ws_bytes, stream);
}

extern "C" int dflash2_verify_sample_ex(const void* target, const void* draft, int dtype, int B,
                                        int G, int64_t V, const int32_t* draft_tok,
                                        const float* draft_max, const float* draft_lse,
                                        float inv_temperature, uint64_t seed, uint32_t step,
                                        const uint32_t* seq_id, int q_mode, int32_t* n_accept,
                                        int32_t* out_tok, float* ratio_dbg, float* u_dbg, void* ws,
                                        size_t ws_bytes, dflash2_stream_t stream) {
    return verify_sample_impl(target, draft, dtype, B, G, V, draft_tok, draft_max, draft_lse,
                              inv_temperature, seed, step, seq_id, q_mode, n_accept, out_tok,
                              ratio_dbg, u_dbg, ws, ws_bytes, stream);
}
