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
// Both verifies stream every logit row once, in chunks of 16 KB: work unit =
// (sequence, row, chunk), one CTA per SM over a contiguous range of units, a
// producer warp keeping TMA bulk copies in flight and consumer warps each
// reducing whole chunks (ring.cuh).  A unit's partial is published with one
// acquire-release add on its sequence's counter; the warp whose add completes
// the sequence (no warp waits) reduces the partials in chunk order and
// decides.  The sampling draw needs the normalisers first, so it is a second
// kernel over the one row each sequence draws from (launched as a dependent
// of the scan, so its launch overlaps the scan's tail): one CTA per 4096
// elements of that row sums its draw weights; the last CTA of the sequence
// finds the chunk where the inverse CDF crosses t = u' * R and scans it.
// No probability vector is ever written to memory.
#include "common.cuh"
#include "ring.cuh"
#include "workspace.cuh"

#include <algorithm>
#include <mutex>

namespace dfl {

constexpr double LOG2E = 1.4426950408889634;

// Programmatic dependent launch (PTX griddepcontrol): the scan lets its
// dependent grid launch early; the draw waits for the scan's results.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ------------------------------------------------------------------ greedy
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

__device__ __forceinline__ void greedy_finish(const uint64_t* P, int S, int G, int b,
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
    const unsigned miss = __ballot_sync(FULL, lane < G && dj != tj);
    const int n = miss ? (__ffs(miss) - 1) : G;
    if (lane <= G) out_tok[(int64_t)b * (G + 1) + lane] = (lane < n) ? dj : (lane == n ? tj : -1);
    if (lane == 0) n_accept[b] = n;
}

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
                greedy_finish(part + b * (G + 1) * S, S, G, (int)b, draft_tok, n_accept, out_tok);
                if (lane == 0) counters[b] = 0u;  // the sequence is done: leave its counter zero
            }
            seg = 0;
        }
    }
}

// ------------------------------------------------------------------ sampling, pass 1
// (maximum, fp64 sum of exp2((x - maximum) c)) of rows r0 .. r0+NB-1 from
// their S chunk partials, warp-collective: lane c takes chunks c, c + 32, ...
// then fixed butterflies.  With S <= 64 every partial of the NB rows is
// loaded in one round (kept in registers); longer rows take two passes.
// Every lane returns the same values.
template <int NB>
__device__ __forceinline__ void rows_lse(const LseD* P, int S, int r0, int nrows, float c2,
                                         float (&Mo)[NB], double (&So)[NB]) {
    const int lane = threadIdx.x & 31;
    if (S <= 64) {
        float m[NB][2];
        double sv[NB][2];
#pragma unroll
        for (int j = 0; j < NB; ++j)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int c = lane + 32 * h;
                m[j][h] = -INFINITY;
                sv[j][h] = 0.0;
                if (j < nrows && c < S) {
                    const LseD* p = &P[(int64_t)(r0 + j) * S + c];
                    m[j][h] = __ldcg(&p->m);
                    sv[j][h] = __ldcg(&p->s);
                }
            }
#pragma unroll
        for (int j = 0; j < NB; ++j) {
            const float M = warp_max(fmaxf(m[j][0], m[j][1]));
            double t = 0.0;
#pragma unroll
            for (int h = 0; h < 2; ++h)
                if (m[j][h] != -INFINITY) t += sv[j][h] * exp2(((double)m[j][h] - (double)M) * (double)c2);
            Mo[j] = M;
            So[j] = warp_sum(t);
        }
        return;
    }
#pragma unroll
    for (int j = 0; j < NB; ++j) {
        Mo[j] = -INFINITY;
        So[j] = 0.0;
    }
    for (int c = lane; c < S; c += 32) {
#pragma unroll
        for (int j = 0; j < NB; ++j)
            if (j < nrows) Mo[j] = fmaxf(Mo[j], __ldcg(&P[(int64_t)(r0 + j) * S + c].m));
    }
#pragma unroll
    for (int j = 0; j < NB; ++j) Mo[j] = warp_max(Mo[j]);
    for (int c = lane; c < S; c += 32) {
#pragma unroll
        for (int j = 0; j < NB; ++j)
            if (j < nrows) {
                const LseD* p = &P[(int64_t)(r0 + j) * S + c];
                const float pm = __ldcg(&p->m);
                const double ps = __ldcg(&p->s);
                if (pm != -INFINITY) So[j] += ps * exp2(((double)pm - (double)Mo[j]) * (double)c2);
            }
    }
#pragma unroll
    for (int j = 0; j < NB; ++j) So[j] = warp_sum(So[j]);
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
    double xt_d = 0.0, xq_d = 0.0;
    if (lane < G) {
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
    const int nrows = (q_mode == DFLASH2_Q_SOFTMAX && !given) ? 2 * G + 1 : G + 1;
    for (int r0 = 0; r0 < nrows; r0 += 8) {
        float Mr[8];
        double Sr[8];
        rows_lse<8>(P, S, r0, min(8, nrows - r0), c2, Mr, Sr);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int rr = r0 + j;
            if (rr <= G && lane == rr) lt = LseD{Mr[j], 0.0f, Sr[j]};
            if (rr > G && rr < nrows && lane == rr - G - 1) lq = LseD{Mr[j], 0.0f, Sr[j]};
        }
    }
    if (q_mode == DFLASH2_Q_SOFTMAX && !given && lane < G) lnq = log(lq.s);
    bool reject = false;
    if (lane < G) {
        // lp = z_t[d] - logZ_t = (x - m) * invT - ln(s); likewise lq
        double lr = (xt_d - (double)lt.m) * (double)inv_t - log(lt.s);
        if (q_mode == DFLASH2_Q_SOFTMAX) lr -= (xq_d - (double)lq.m) * (double)inv_t - lnq;
        const double ratio = exp(lr);
        const float u = philox_uniform(seed, step, sid, (uint32_t)lane, 0u);
        reject = !((double)u < ratio);
        if (ratio_dbg) ratio_dbg[(int64_t)b * G + lane] = (float)ratio;
        if (u_dbg) u_dbg[(int64_t)b * G + lane] = u;
    }
    const unsigned rej = __ballot_sync(FULL, reject);
    const int n = rej ? (__ffs(rej) - 1) : G;
    if (lane <= G) out_tok[(int64_t)b * (G + 1) + lane] = (lane < n) ? dn : -1;  // draw fills n
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

// Units are (sequence b, row rr, chunk): rows 0..G of a sequence are its
// target rows, G+1..2G its draft rows (softmax mode only).  A unit's partial
// is the chunk maximum and the fp64 sum of exp2((x - m) c) against it; a
// warp publishes its consecutive units of one sequence together.
template <bool BF16, bool TMA>
__global__ void __launch_bounds__(RING_THREADS, 1) verify_sample_scan_kernel(
    const void* __restrict__ target, const void* __restrict__ draft, int G, int64_t V, int S,
    int rows_per_seq, int64_t units, float inv_t, float c2, const int32_t* __restrict__ draft_tok,
    uint64_t seed, uint32_t step, const uint32_t* __restrict__ seq_id, int q_mode,
    int32_t* __restrict__ n_accept, int32_t* __restrict__ out_tok, float* __restrict__ ratio_dbg,
    float* __restrict__ u_dbg, LseD* __restrict__ part, SampleInfo* __restrict__ info,
    unsigned* __restrict__ counters, const float* __restrict__ q_max,
    const float* __restrict__ q_lse) {
    constexpr int ES = BF16 ? 2 : 4;
    constexpr int LEN = chunk_len(ES);
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ __align__(8) uint64_t bars[2 * NCW];
    const int lane = threadIdx.x & 31;
    auto rowp = [&](int64_t b, int rr) {
        return (rr <= G) ? (const char*)target + (b * (G + 1) + rr) * V * ES
                         : (const char*)draft + (b * G + (rr - G - 1)) * V * ES;
    };
    pdl_launch_dependents();
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
    if (TMA) r = warp_ring_start(ring, bars, n, ic, ChunkT<BF16>::NEG_INF_WORD, src);
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
            Ssum = chunk_expsum<BF16>(view, M, c2);
            warp_ring_next(r, k, n, ic, ChunkT<BF16>::NEG_INF_WORD, src);
        } else {
            const GlobalView<BF16> view{(const uint8_t*)rowp(b, uc.r), v0, len};
            uint32_t vm[NVL];
            M = warp_max(chunk_pass1<BF16>(view, vm));
            Ssum = chunk_expsum<BF16>(view, M, c2);
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
                if (lane == 0) counters[b] = 0u;  // the sequence is done: leave its counter zero
            }
            seg = 0;
        }
    }
}

// ------------------------------------------------------------------ sampling, pass 2
// Draw weight of one element of the row the sequence draws from (draw_w):
//   p_v = exp2((x_v - mt) * c - l2t),  q_v likewise,
//   mode 0: w = max(0, p - q), evaluated as q * expm1(ln p - ln q) with
//           ln p - ln q = (xt - xq) * invT - (logZ_t - logZ_q): the same
//           value, without the cancellation of p - q when p and q agree;
//   mode 1: w = p, 0 at d;  mode 2: w = p (also the fallback when the
//   residual is empty by rounding).
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

// The draw of one sequence covers DLEN elements per CTA of the row it draws
// from; thread t holds DEPT consecutive elements.  A thread's sum: fp32 over a
// 16-byte vector (index order, pairwise), fp64 across vectors.
constexpr int DLEN = DRAW_LEN;
constexpr int DT = 256;
constexpr int DEPT = DLEN / DT;  // 40: 5 bf16 / 10 fp32 vectors
// CTAs per row the draw handles (their sums sit in shared memory): V <= 3072 * 10240.
constexpr int64_t DRAW_MAX_CHUNKS = 3072;

// The draw weight of one element (mode 0: residual, 1: p without d, 2: p;
// the residual-empty fallback draws with mode 2).  The mode is the same for
// a whole CTA, so the branch is uniform.
// off: the element's offset in the thread's run, d_off: the offset of d
// there (anything outside [0, DEPT) when d is not in the run).
__device__ __forceinline__ float draw_w(int mode, float xt, float xq, int off, int64_t d_off,
                                        const SampleInfo& I, float c2, float inv_t) {
    if (mode == 0) {
        const float dlog = (xt - xq) * inv_t - I.dl;
        if (!(dlog > 0.0f)) return 0.0f;
        return ex2((xq - I.mq) * c2 - I.l2q) * expm1_pos(dlog);
    }
    if (mode == 1 && (int64_t)off == d_off) return 0.0f;
    return ex2((xt - I.mt) * c2 - I.l2t);
}

// The DEPT elements [vb, vb + DEPT) of a row as 16-byte vectors (-inf past V).
template <bool BF16, bool VEC>
__device__ __forceinline__ void draw_load(const char* row, int64_t vb, int64_t V,
                                          uint4 (&x)[DEPT / ChunkT<BF16>::VW]) {
    using C = ChunkT<BF16>;
    constexpr int NV = DEPT / C::VW;
    if (VEC && vb + DEPT <= V) {
        const uint4* p = (const uint4*)(row + vb * C::ES);
#pragma unroll
        for (int g = 0; g < NV; ++g) x[g] = __ldg(p + g);
    } else {
        const GlobalView<BF16> view{(const uint8_t*)row, vb,
                                    (int)max((int64_t)0, min((int64_t)DEPT, V - vb))};
#pragma unroll
        for (int g = 0; g < NV; ++g) x[g] = view.vec(g);
    }
}

// A thread's weights over its DEPT elements and their sum (fp32 pairwise
// within a 16-byte vector, fp64 across vectors); w may be null.
template <bool BF16, bool VEC>
__device__ __forceinline__ double draw_thread(const char* trow, const char* qrow, int64_t vb,
                                              int64_t V, int mode, const SampleInfo& I, float c2,
                                              float inv_t, float* w) {
    using C = ChunkT<BF16>;
    constexpr int NV = DEPT / C::VW;
    uint4 xt[NV], xq[NV];
    draw_load<BF16, VEC>(trow, vb, V, xt);
    if (mode == 0) draw_load<BF16, VEC>(qrow, vb, V, xq);
    const int64_t d_off = (int64_t)I.d - vb;
    double s = 0.0;
#pragma unroll
    for (int g = 0; g < NV; ++g) {
        float sv[C::VW];
#pragma unroll
        for (int e = 0; e < C::VW; ++e) {
            sv[e] = draw_w(mode, C::elem(xt[g], e), mode == 0 ? C::elem(xq[g], e) : 0.0f,
                           g * C::VW + e, d_off, I, c2, inv_t);
            if (w) w[g * C::VW + e] = sv[e];
        }
#pragma unroll
        for (int h = C::VW / 2; h > 0; h >>= 1)
#pragma unroll
            for (int e = 0; e < h; ++e) sv[e] += sv[e + h];
        s += (double)sv[0];
    }
    return s;
}

// Inclusive scan of the threads' values in thread order (fp64): warp scans,
// then the warps' totals in warp order.  `total` is the last thread's value,
// bit for bit.  Block-wide (two barriers).
__device__ __forceinline__ double block_incl_scan(double x, double* s_warp, double& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    double incl = x;
#pragma unroll
    for (int k = 1; k < 32; k <<= 1) {
        const double o = __shfl_up_sync(FULL, incl, k);
        if (lane >= k) incl += o;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    double base = 0.0;
    for (int w = 0; w < warp; ++w) base += s_warp[w];
    double tot = 0.0;
    for (int w = 0; w < DT / 32 - 1; ++w) tot += s_warp[w];
    total = tot + s_warp[DT / 32 - 1];
    __syncthreads();
    return base + incl;
}

// Draw, part 1: grid (chunks of the drawn row, sequences).  Every thread's
// inclusive prefix within the chunk is stored (dsum[b][c][t]); the last one
// is the chunk's sum.
template <bool BF16, bool VEC>
__global__ void __launch_bounds__(DT) verify_sample_draw_kernel(
    const void* __restrict__ target, const void* __restrict__ draft, int G, int64_t V, int D,
    float c2, float inv_t, const SampleInfo* __restrict__ info, double* __restrict__ dsum) {
    constexpr int ES = BF16 ? 2 : 4;
    __shared__ double s_warp[DT / 32];
    const int c = blockIdx.x, b = blockIdx.y;
    pdl_wait();  // the scan's SampleInfo, and every earlier write, are visible
    pdl_launch_dependents();
    const SampleInfo I = info[b];
    const char* trow = (const char*)target + ((int64_t)b * (G + 1) + I.n) * V * ES;
    const char* qrow = (I.mode == 0) ? (const char*)draft + ((int64_t)b * G + I.n) * V * ES : nullptr;
    const double my = draw_thread<BF16, VEC>(trow, qrow, (int64_t)c * DLEN + (int64_t)DEPT * threadIdx.x,
                                             V, I.mode, I, c2, inv_t, nullptr);
    double total;
    const double incl = block_incl_scan(my, s_warp, total);
    dsum[((int64_t)b * D + c) * DT + threadIdx.x] = incl;
}

// The draw when the residual is empty by rounding: from p_n.  Two passes
// over the row, chunk by chunk, the lanes taking part-1 threads 32 j + lane:
// the thread sums in one inclusive scan (lane order within a group of 32,
// groups and chunks in order), whose last value is R; then the same scan
// against t = u' R, and the crossing thread walks its own elements.  Rare,
// so kept out of line (the pick's common path stays small).  Returns the
// element offset within the run starting at vb (lane 0; -1 if none).
template <bool BF16, bool VEC>
__device__ __noinline__ int draw_fallback(const char* trow, const char* qrow, int64_t V, int D,
                                          const SampleInfo& I, float c2, float inv_t, int64_t& vb) {
    const int lane = threadIdx.x & 31;
    const int mode = 2;
    int pick = -1;
    auto scan_pass = [&](bool find, double tcut, int& cc_hit, int& t_hit, double& base) {
        double acc = 0.0;
        for (int cc = 0; cc < D; ++cc)
            for (int j = 0; j < DT / 32; ++j) {
                const int t = 32 * j + lane;
                const double ts = draw_thread<BF16, VEC>(
                    trow, qrow, (int64_t)cc * DLEN + (int64_t)DEPT * t, V, mode, I, c2, inv_t,
                    nullptr);
                double incl = ts;
#pragma unroll
                for (int k = 1; k < 32; k <<= 1) {
                    const double o = __shfl_up_sync(FULL, incl, k);
                    if (lane >= k) incl += o;
                }
                incl += acc;
                if (find) {
                    const unsigned cross = __ballot_sync(FULL, incl > tcut);
                    if (cross) {
                        const int l = __ffs(cross) - 1;
                        cc_hit = cc;
                        t_hit = 32 * j + l;
                        base = __shfl_sync(FULL, incl - ts, l);
                        return acc;
                    }
                }
                acc = __shfl_sync(FULL, incl, 31);
            }
        return acc;
    };
    int cc_hit = -1, t_hit = -1;
    double base = 0.0;
    const double R = scan_pass(false, 0.0, cc_hit, t_hit, base);
    const double tt = (double)I.u_res * R;
    scan_pass(true, tt, cc_hit, t_hit, base);
    if (cc_hit >= 0 && lane == 0) {
        float w[DEPT];
        vb = (int64_t)cc_hit * DLEN + (int64_t)DEPT * t_hit;
        draw_thread<BF16, VEC>(trow, qrow, vb, V, mode, I, c2, inv_t, w);
        double run = base;
        int lm = -1;
        for (int e = 0; e < DEPT; ++e) {
            if (w[e] > 0.0f) lm = e;
            run += (double)w[e];
            if (pick < 0 && run > tt) pick = e;
        }
        if (pick < 0) pick = lm;
    }
    return pick;
}

// Draw, part 2: one warp per sequence.  R = the chunk sums in chunk order,
// t = u' R; in the first chunk whose inclusive prefix exceeds t, the first
// thread of part 1 whose inclusive prefix exceeds t (from the stored
// prefixes) recomputes its weights and walks them to the first element whose
// running prefix exceeds t (else, rounding, the last element with mass).  If
// the residual is empty by rounding (R = 0) the draw is redone from p_n by
// this warp (rare, slow).
template <bool BF16, bool VEC>
__global__ void __launch_bounds__(32) verify_sample_pick_kernel(
    const void* __restrict__ target, const void* __restrict__ draft, int G, int64_t V, int D,
    float c2, float inv_t, const SampleInfo* __restrict__ info, const double* __restrict__ dsum,
    int32_t* __restrict__ out_tok) {
    constexpr int ES = BF16 ? 2 : 4;
    const int lane = threadIdx.x, b = blockIdx.x;
    pdl_wait();  // part 1's prefixes
    const SampleInfo I = info[b];
    const char* trow = (const char*)target + ((int64_t)b * (G + 1) + I.n) * V * ES;
    const char* qrow = (I.mode == 0) ? (const char*)draft + ((int64_t)b * G + I.n) * V * ES : nullptr;
    const double* P = dsum + (int64_t)b * D * DT;
    // The chunk sums, loaded together, in an inclusive warp scan (fixed
    // order; R is its last value); carried across groups of 32 chunks.
    double carry = 0.0, tt = 0.0, pre = 0.0;
    int cstar = -1, lastc = -1;
    double lastc_pre = 0.0;
    int mode = I.mode;
    {
        double R = 0.0;
        for (int c0 = 0; c0 < D; c0 += 32) {
            const int cc = c0 + lane;
            const double cs = (cc < D) ? __ldcg(&P[(int64_t)cc * DT + DT - 1]) : 0.0;
            double incl = cs;
#pragma unroll
            for (int k = 1; k < 32; k <<= 1) {
                const double o = __shfl_up_sync(FULL, incl, k);
                if (lane >= k) incl += o;
            }
            incl += carry;
            carry = __shfl_sync(FULL, incl, 31);
        }
        R = carry;
        if (!(R > 0.0)) mode = 2;  // residual empty by rounding: draw from p_n (rare)
        tt = (double)I.u_res * R;
        carry = 0.0;
        for (int c0 = 0; c0 < D && cstar < 0; c0 += 32) {  // the same scan again, now against t
            const int cc = c0 + lane;
            const double cs = (cc < D) ? __ldcg(&P[(int64_t)cc * DT + DT - 1]) : 0.0;
            double incl = cs;
#pragma unroll
            for (int k = 1; k < 32; k <<= 1) {
                const double o = __shfl_up_sync(FULL, incl, k);
                if (lane >= k) incl += o;
            }
            incl += carry;
            const unsigned cross = __ballot_sync(FULL, cc < D && incl > tt);
            const unsigned mass = __ballot_sync(FULL, cc < D && cs > 0.0);
            if (mass) {
                const int l = 31 - __clz(mass);
                lastc = c0 + l;
                lastc_pre = __shfl_sync(FULL, incl - cs, l);
            }
            if (cross) {
                const int l = __ffs(cross) - 1;
                cstar = c0 + l;
                pre = __shfl_sync(FULL, incl - cs, l);
            }
            carry = __shfl_sync(FULL, incl, 31);
        }
        if (cstar < 0) {  // unreachable while R > 0: the last chunk with mass
            cstar = max(lastc, 0);
            pre = lastc >= 0 ? lastc_pre : 0.0;
        }
    }
    int pick = -1;
    int64_t vb = 0;
    if (mode == I.mode) {
        // the first thread of chunk cstar whose inclusive prefix exceeds t;
        // all 256 prefixes loaded in one round
        const double* Q = P + (int64_t)cstar * DT;
        double incl[DT / 32], prev[DT / 32];
#pragma unroll
        for (int j = 0; j < DT / 32; ++j) {
            const int t = 32 * j + lane;
            incl[j] = __ldcg(&Q[t]);
            prev[j] = (t > 0) ? __ldcg(&Q[t - 1]) : 0.0;
        }
        int pt = DT, lastm = -1;
#pragma unroll
        for (int j = DT / 32 - 1; j >= 0; --j) {
            const unsigned cross = __ballot_sync(FULL, pre + incl[j] > tt);
            const unsigned mass = __ballot_sync(FULL, incl[j] > prev[j]);
            if (cross) pt = 32 * j + __ffs(cross) - 1;
            if (mass && lastm < 0) lastm = 32 * j + 31 - __clz(mass);
        }
        if (pt == DT) pt = lastm;  // rounding left t above the chunk's scan
        if (pt >= 0) {
            vb = (int64_t)cstar * DLEN + (int64_t)DEPT * pt;
            const double base = pre + (pt > 0 ? __ldcg(&Q[pt - 1]) : 0.0);
            if (lane == 0) {
                float w[DEPT];
                draw_thread<BF16, VEC>(trow, qrow, vb, V, mode, I, c2, inv_t, w);
                double run = base;
                int lm = -1;
                for (int e = 0; e < DEPT; ++e) {
                    if (w[e] > 0.0f) lm = e;
                    run += (double)w[e];
                    if (pick < 0 && run > tt) pick = e;
                }
                if (pick < 0) pick = lm;
            }
        }
    } else {
        pick = draw_fallback<BF16, VEC>(trow, qrow, V, D, I, c2, inv_t, vb);
    }
    if (lane == 0 && pick >= 0) out_tok[(int64_t)b * (G + 1) + I.n] = (int32_t)(vb + pick);
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

// Launch as a programmatic dependent of the previous kernel on the stream:
// the grid may start while that kernel finishes, and waits (griddepcontrol)
// for its results before reading them.
template <class Kern, class... Args>
static cudaError_t launch_dependent(Kern kern, dim3 grid, dim3 block, size_t dyn, cudaStream_t s,
                                    Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = dyn;
    cfg.stream = s;
    cudaLaunchAttribute a[1];
    a[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = a;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Draw grid size per sequence: DLEN-element chunks of the drawn row.
static inline int64_t draw_chunks(int64_t V) { return (V + DLEN - 1) / DLEN; }

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
    const int64_t D = draw_chunks(V);
    if (D > DRAW_MAX_CHUNKS) return DFLASH2_ESHAPE;
    // draft rows are scanned only when their normalisers are not given
    const int rows_per_seq = (q_mode == DFLASH2_Q_SOFTMAX && !q_max) ? 2 * G + 1 : G + 1;
    const int64_t units = (int64_t)B * rows_per_seq * S;
    if (units > (int64_t)INT32_MAX || B > 65535) return DFLASH2_ESHAPE;
    const Layout L = sample_layout(B, G, V, es);
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return DFLASH2_EWORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned* counters = (unsigned*)((char*)ws + L.counters_off);  // [B] scan
    LseD* part = (LseD*)((char*)ws + L.part_off);
    double* dsum = (double*)((char*)ws + L.part2_off);
    SampleInfo* info = (SampleInfo*)((char*)ws + L.info_off);
    if (!L.self_clean && cudaMemsetAsync(counters, 0, (size_t)B * 4, s) != cudaSuccess)
        return DFLASH2_ECUDA;
    const void* q = (q_mode == DFLASH2_Q_SOFTMAX) ? draft : nullptr;
    const bool tma = aligned(target, 16) && (!q || aligned(q, 16)) && (V * es) % 16 == 0;
    const float c2 = (float)((double)inv_temperature * LOG2E);
#define DFL_SAMPLE(BF, TM)                                                                        \
    do {                                                                                          \
        auto kern = verify_sample_scan_kernel<BF, TM>;                                            \
        const size_t dyn = TM ? (size_t)RING_BYTES : 0;                                           \
        if (ring_prepare(kern, dyn) != DFLASH2_OK) return DFLASH2_ECUDA;                          \
        kern<<<ring_grid(units), RING_THREADS, dyn, s>>>(                                         \
            target, q, G, V, (int)S, rows_per_seq, units, inv_temperature, c2, draft_tok, seed,   \
            step, seq_id, q_mode, n_accept, out_tok, ratio_dbg, u_dbg, part, info, counters,      \
            q_max, q_lse);                                                                        \
        auto kern2 = verify_sample_draw_kernel<BF, TM>;                                           \
        if (launch_dependent(kern2, dim3((unsigned)D, (unsigned)B), dim3(DT), 0, s, target, q, G, \
                             V, (int)D, c2, inv_temperature, (const SampleInfo*)info, dsum) !=    \
            cudaSuccess)                                                                          \
            return DFLASH2_ECUDA;                                                                 \
        auto kern3 = verify_sample_pick_kernel<BF, TM>;                                           \
        if (launch_dependent(kern3, dim3((unsigned)B), dim3(32), 0, s, target, q, G, V, (int)D,    \
                             c2, inv_temperature, (const SampleInfo*)info, (const double*)dsum,   \
                             out_tok) != cudaSuccess)                                             \
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
