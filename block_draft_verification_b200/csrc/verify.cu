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
// chunk order and decides.  The sampling draw needs the normalisers first, so it is a second
// kernel over the one row each sequence draws from (L2-resident after the
// first pass): one CTA per chunk sums the draw weights, and the last of them
// finds the chunk where the inverse CDF crosses t = u' * R and scans only that
// chunk.  No probability vector is ever written to memory.
#include "common.cuh"
#include "stream.cuh"
#include "workspace.cuh"

namespace dfl {

constexpr double LOG2E = 1.4426950408889634;

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

// A chunk's (max, sum-exp): the block max first, then each thread's sum of
// exp2((x - M) c) (fp32 per vector, fp64 across vectors), then the block
// sum in a fixed order -- no rescaling, no exp in the merge.
template <bool BF16, class C>
__device__ __forceinline__ LseD block_lse(const C& ch, float c2, float* s_max, double* s_sum) {
    using R = Row<BF16>;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float m = view_max<BF16>(ch);
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, j));
    if (lane == 0) s_max[warp] = m;
    __syncthreads();
    float M = s_max[0];
#pragma unroll
    for (int w = 1; w < NT / 32; ++w) M = fmaxf(M, s_max[w]);
    double s = 0.0;
    if (M != -INFINITY) {
#pragma unroll
        for (int i = 0; i < R::NV; ++i) {
            const uint4 v4 = ch.vec(i);
            float tt[R::VW];
#pragma unroll
            for (int e = 0; e < R::VW; ++e) tt[e] = ex2((R::elem(v4, e) - M) * c2);
#pragma unroll
            for (int w = R::VW / 2; w > 0; w >>= 1)
#pragma unroll
                for (int e = 0; e < w; ++e) tt[e] += tt[e + w];
            s += (double)tt[0];
        }
    }
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) s += __shfl_xor_sync(FULL, s, j);
    if (lane == 0) s_sum[warp] = s;
    __syncthreads();
    double S = 0.0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) S += s_sum[w];
    return {M, 0.0f, S};
}

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
    __shared__ float s_max[NT / 32];
    __shared__ double s_sum[NT / 32];
    __shared__ __align__(8) uint64_t s_bar[2];
    const int t = threadIdx.x, warp = t >> 5;
    const uint32_t bar0 = smem_u32(&s_bar[0]);
    const int per_seq = rows_per_seq * S;
    auto geom = [&](int64_t u, int& b, int& rr, const char*& rowp, int64_t& v0, int64_t& vend) {
        b = (int)(u / per_seq);
        const int rem = (int)(u - (int64_t)b * per_seq);
        rr = rem / S;
        rowp = (rr <= G) ? (const char*)target + ((int64_t)b * (G + 1) + rr) * V * ES
                         : (const char*)draft + ((int64_t)b * G + (rr - G - 1)) * V * ES;
        v0 = (int64_t)(rem - rr * S) * CHUNK;
        vend = min(V, v0 + (int64_t)CHUNK);
    };
    auto issue = [&](int64_t u, int slot) {
        int b, rr;
        const char* rowp;
        int64_t v0, vend;
        geom(u, b, rr, rowp, v0, vend);
        bulk_g2s(smem_u32(ring + slot * SLOT), rowp + v0 * ES, (uint32_t)((vend - v0) * ES),
                 bar0 + 8 * slot);
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
        int b, rr;
        const char* rowp;
        int64_t v0, vend;
        geom(u, b, rr, rowp, v0, vend);
        LseD tot;
        if (TMA) {
            if (t == 0 && u + 1 < hi) issue(u + 1, (k + 1) & 1);
            if (!__syncthreads_and(mbar_wait(bar0 + 8 * (k & 1), (k >> 1) & 1))) {
                if (t == 0) {
                    atomicOr(&g_dev_err, ERR_STREAM);
                    if (u + 1 < hi) mbar_wait(bar0 + 8 * ((k + 1) & 1), ((k + 1) >> 1) & 1);
                }
                return;
            }
            tot = block_lse<BF16>(SmemChunk<BF16>{ring + (k & 1) * SLOT, v0, vend}, c2, s_max, s_sum);
        } else {
            RegChunk<BF16> ch;
            ch.load(rowp, v0, vend);
            tot = block_lse<BF16>(ch, c2, s_max, s_sum);
        }
        if (t == 0)  // thread 0 alone stores the partial (published by its release add)
            part[((int64_t)b * rows_per_seq + rr) * S + v0 / CHUNK] = tot;
        ++pending;
        if (u + 1 == hi || (u + 1) / per_seq != b) {  // done with this sequence: publish
            if (t == 0) s_last = publish(&counters[b], pending, (unsigned)per_seq);
            __syncthreads();
            if (s_last && warp == 0)
                sample_finish(target, draft, part + (int64_t)b * rows_per_seq * S, G, V, S, ES, inv_t,
                              c2, draft_tok, seed, step, seq_id ? seq_id[b] : (uint32_t)b, q_mode, b,
                              n_accept, out_tok, ratio_dbg, u_dbg, info);
            pending = 0;
        }
        __syncthreads();  // ring slot k & 1 is free
    }
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

template <bool BF16>
__device__ __forceinline__ float draw_weight(const uint4& rt, const uint4& rq, int e, int64_t v,
                                             const SampleInfo& I, float c, float inv_t,
                                             bool use_p) {
    using R = Row<BF16>;
    const float xt = R::elem(rt, e);
    if (I.mode == 0 && !use_p) {
        const float xq = R::elem(rq, e);
        const float dlog = (xt - xq) * inv_t - I.dl;
        if (!(dlog > 0.0f)) return 0.0f;
        return ex2((xq - I.mq) * c - I.l2q) * expm1_pos(dlog);
    }
    if (I.mode == 1 && !use_p && v == I.d) return 0.0f;
    return ex2((xt - I.mt) * c - I.l2t);
}

// Thread t's contiguous 64 elements [v0 + 64 t, v0 + 64 t + 64) of a chunk:
// a thread's running sum follows index order (the inverse-CDF scan needs it).
template <bool BF16, bool VEC>
__device__ __forceinline__ void load_contig(const void* row, int64_t v0, int64_t vend,
                                            uint4 (&r)[Row<BF16>::NV]) {
    using R = Row<BF16>;
    const int64_t base = v0 + (int64_t)threadIdx.x * EPT;
#pragma unroll
    for (int i = 0; i < R::NV; ++i) {
        const int64_t vb = base + i * R::VW;
        if (VEC && vb + R::VW <= vend) {
            r[i] = *(const uint4*)((const char*)row + vb * (BF16 ? 2 : 4));
        } else {
            uint32_t w[4] = {R::NEG_INF_WORD, R::NEG_INF_WORD, R::NEG_INF_WORD, R::NEG_INF_WORD};
#pragma unroll
            for (int e = 0; e < R::VW; ++e)
                if (vb + e < vend) {
                    const uint32_t bits = R::scalar_bits(row, vb + e);
                    if (BF16) {
                        uint32_t& word = w[e >> 1];
                        word = (e & 1) ? ((word & 0x0000FFFFu) | (bits << 16))
                                       : ((word & 0xFFFF0000u) | bits);
                    } else {
                        w[e] = bits;
                    }
                }
            r[i] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

// One 16-byte vector (element vb .. vb + VW - 1) of a row; -inf past vend.
template <bool BF16, bool VEC>
__device__ __forceinline__ uint4 load_vec(const char* row, int64_t vb, int64_t vend) {
    using R = Row<BF16>;
    if (VEC && vb + R::VW <= vend) return *(const uint4*)(row + vb * (BF16 ? 2 : 4));
    uint32_t w[4] = {R::NEG_INF_WORD, R::NEG_INF_WORD, R::NEG_INF_WORD, R::NEG_INF_WORD};
    for (int e = 0; e < R::VW; ++e)
        if (vb + e < vend) {
            const uint32_t bits = R::scalar_bits(row, vb + e);
            if (BF16) {
                uint32_t& word = w[e >> 1];
                word = (e & 1) ? ((word & 0x0000FFFFu) | (bits << 16)) : ((word & 0xFFFF0000u) | bits);
            } else {
                w[e] = bits;
            }
        }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Sum of the draw weights of this thread's 64 elements (fp32 per vector,
// fp64 across vectors).  The vector loop is not unrolled: the kernel's code
// stays small enough for the instruction cache.
template <bool BF16, bool VEC>
__device__ __noinline__ double thread_weight_sum(const char* trow, const char* qrow, int64_t v0,
                                                 int64_t vend, const SampleInfo& I, float c2,
                                                 float inv_t, bool use_p) {
    using R = Row<BF16>;
    const bool with_q = I.mode == 0 && !use_p;
    double s = 0.0;
    const int64_t vb = v0 + (int64_t)threadIdx.x * EPT;
#pragma unroll 1
    for (int i = 0; i < R::NV; ++i) {
        const uint4 rt = load_vec<BF16, VEC>(trow, vb + i * R::VW, vend);
        const uint4 rq = with_q ? load_vec<BF16, VEC>(qrow, vb + i * R::VW, vend) : make_uint4(0, 0, 0, 0);
        float sv = 0.0f;
#pragma unroll
        for (int e = 0; e < R::VW; ++e)
            sv += draw_weight<BF16>(rt, rq, e, vb + i * R::VW + e, I, c2, inv_t, use_p);
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

template <bool BF16, bool VEC>
__global__ void __launch_bounds__(NT, 3) verify_sample_draw_kernel(
    const void* __restrict__ target, const void* __restrict__ draft, int G, int64_t V, int S,
    float c2, float inv_t, const SampleInfo* __restrict__ info, double* __restrict__ part2,
    unsigned* __restrict__ counters2, int32_t* __restrict__ out_tok) {
    constexpr int ES = BF16 ? 2 : 4;
    using R = Row<BF16>;
    __shared__ double s_warp[NT / 32];
    __shared__ double s_scan[NT];
    __shared__ double s_base, s_t;
    __shared__ int s_cstar, s_fallback, s_pick_thread, s_done, s_last;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int b = blockIdx.x / S, chunk = blockIdx.x - b * S;
    const SampleInfo I = info[b];
    const char* trow = (const char*)target + ((int64_t)b * (G + 1) + I.n) * V * ES;
    const char* qrow = (I.mode == 0) ? (const char*)draft + ((int64_t)b * G + I.n) * V * ES : nullptr;
    double* P2 = part2 + (int64_t)b * S;

    {
        const int64_t v0 = (int64_t)chunk * CHUNK, vend = min(V, v0 + (int64_t)CHUNK);
        const double W = block_sum(
            thread_weight_sum<BF16, VEC>(trow, qrow, v0, vend, I, c2, inv_t, false), s_warp);
        if (t == 0) {
            P2[chunk] = W;
            __threadfence();
        }
    }
    if (!arrive_last(&counters2[b], (unsigned)S)) return;

    // ---- last chunk of this sequence: total mass, crossing chunk, in-chunk scan
    if (t == 0) {
        double Rm = 0.0;
        for (int c = 0; c < S; ++c) Rm += __ldcg(&P2[c]);
        s_fallback = !(Rm > 0.0);
    }
    __syncthreads();
    const bool use_p = s_fallback != 0;
    if (use_p) {  // residual empty by rounding: draw from p_n instead (rare)
        for (int c = 0; c < S; ++c) {
            const int64_t v0 = (int64_t)c * CHUNK, vend = min(V, v0 + (int64_t)CHUNK);
            const double W = block_sum(
                thread_weight_sum<BF16, VEC>(trow, qrow, v0, vend, I, c2, inv_t, true), s_warp);
            if (t == 0) P2[c] = W;
        }
        __syncthreads();
    }
    if (t == 0) {
        double Rm = 0.0;
        for (int c = 0; c < S; ++c) Rm += __ldcg(&P2[c]);
        const double tt = (double)I.u_res * Rm;
        double pre = 0.0;
        int cstar = -1, clast = 0;
        for (int c = 0; c < S; ++c) {
            const double wc = __ldcg(&P2[c]);
            if (wc > 0.0) clast = c;
            if (cstar < 0 && pre + wc > tt) cstar = c;
            if (cstar < 0) pre += wc;
        }
        if (cstar < 0) {  // rounding left t at the top: the last chunk with mass
            cstar = clast;
            pre = 0.0;
            for (int c = 0; c < clast; ++c) pre += __ldcg(&P2[c]);
        }
        s_cstar = cstar;
        s_base = pre;
        s_t = tt;
        s_pick_thread = NT;
        s_done = 0;
        s_last = -1;
    }
    __syncthreads();
    const int64_t v0 = (int64_t)s_cstar * CHUNK, vend = min(V, v0 + (int64_t)CHUNK);
    const double tt = s_t;
    const double mysum = thread_weight_sum<BF16, VEC>(trow, qrow, v0, vend, I, c2, inv_t, use_p);
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
    if (pt < NT && warp == 0) {
        // warp 0 walks thread pt's 64 elements, two per lane, in index order
        const int64_t vb = v0 + (int64_t)pt * EPT + 2 * lane;
        const int i = (2 * lane) / R::VW, e = (2 * lane) % R::VW;
        uint4 xt = make_uint4(0, 0, 0, 0), xq = make_uint4(0, 0, 0, 0);
        if (vb < vend) {  // the 16-byte vector holding this lane's pair
            const int64_t v8 = v0 + (int64_t)pt * EPT + i * R::VW;
            if (VEC && v8 + R::VW <= vend) {
                xt = *(const uint4*)(trow + v8 * ES);
                if (I.mode == 0 && !use_p) xq = *(const uint4*)(qrow + v8 * ES);
            } else {
                uint32_t wt[4] = {R::NEG_INF_WORD, R::NEG_INF_WORD, R::NEG_INF_WORD, R::NEG_INF_WORD};
                uint32_t wq[4] = {R::NEG_INF_WORD, R::NEG_INF_WORD, R::NEG_INF_WORD, R::NEG_INF_WORD};
                for (int ee = 0; ee < R::VW; ++ee)
                    if (v8 + ee < vend) {
                        const uint32_t bt = R::scalar_bits(trow, v8 + ee);
                        const uint32_t bq = (I.mode == 0 && !use_p) ? R::scalar_bits(qrow, v8 + ee) : 0u;
                        if (BF16) {
                            const int sh = (ee & 1) ? 16 : 0;
                            const uint32_t msk = (ee & 1) ? 0x0000FFFFu : 0xFFFF0000u;
                            wt[ee >> 1] = (wt[ee >> 1] & msk) | (bt << sh);
                            wq[ee >> 1] = (wq[ee >> 1] & msk) | (bq << sh);
                        } else {
                            wt[ee] = bt;
                            wq[ee] = bq;
                        }
                    }
                xt = make_uint4(wt[0], wt[1], wt[2], wt[3]);
                xq = make_uint4(wq[0], wq[1], wq[2], wq[3]);
            }
        }
        const float w0 = (vb < vend) ? draw_weight<BF16>(xt, xq, e, vb, I, c2, inv_t, use_p) : 0.0f;
        const float w1 =
            (vb + 1 < vend) ? draw_weight<BF16>(xt, xq, e + 1, vb + 1, I, c2, inv_t, use_p) : 0.0f;
        double incl2 = (double)w0 + (double)w1;
#pragma unroll
        for (int kk = 1; kk < 32; kk <<= 1) {
            const double o = __shfl_up_sync(FULL, incl2, kk);
            if (lane >= kk) incl2 += o;
        }
        const double base = s_base + (pt > 0 ? s_scan[pt - 1] : 0.0);
        const double before = base + incl2 - ((double)w0 + (double)w1);
        const bool c0 = before + (double)w0 > tt;
        const bool c1 = before + (double)w0 + (double)w1 > tt;
        const unsigned m0 = __ballot_sync(FULL, c0), m1 = __ballot_sync(FULL, c1);
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
            out_tok[(int64_t)b * (G + 1) + I.n] = (int32_t)(v0 + (int64_t)pt * EPT + pick);
            s_done = 1;
        }
    }
    __syncthreads();
    if (!s_done) {  // block-uniform: rounding left t above the chunk's scan
        if (mysum > 0.0) {
            const bool with_q = I.mode == 0 && !use_p;
            int lastpos = -1;
            const int64_t vb = v0 + (int64_t)t * EPT;
#pragma unroll 1
            for (int i = 0; i < R::NV; ++i) {
                const uint4 rt = load_vec<BF16, VEC>(trow, vb + i * R::VW, vend);
                const uint4 rq =
                    with_q ? load_vec<BF16, VEC>(qrow, vb + i * R::VW, vend) : make_uint4(0, 0, 0, 0);
#pragma unroll 1
                for (int e = 0; e < R::VW; ++e)
                    if (draw_weight<BF16>(rt, rq, e, vb + i * R::VW + e, I, c2, inv_t, use_p) > 0.0f)
                        lastpos = i * R::VW + e;
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
    const int rows_per_seq = (q_mode == DFLASH2_Q_SOFTMAX) ? 2 * G + 1 : G + 1;
    const int64_t units = (int64_t)B * rows_per_seq * S;
    if (units > (int64_t)INT32_MAX) return DFLASH2_ESHAPE;
    const Layout L = sample_layout(B, G, V);
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return DFLASH2_EWORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned* counters = (unsigned*)((char*)ws + L.counters_off);
    LseD* part = (LseD*)((char*)ws + L.part_off);
    double* part2 = (double*)((char*)ws + L.part2_off);
    SampleInfo* info = (SampleInfo*)((char*)ws + L.info_off);
    if (cudaMemsetAsync(counters, 0, (size_t)B * 2 * 4, s) != cudaSuccess) return DFLASH2_ECUDA;
    const void* q = (q_mode == DFLASH2_Q_SOFTMAX) ? draft : nullptr;
    const bool tma = aligned(target, 16) && (!q || aligned(q, 16)) && (V * es) % 16 == 0;
    const float c2 = (float)((double)inv_temperature * LOG2E);
    const dim3 grid2((unsigned)((int64_t)B * S));
#define DFL_SAMPLE(BF, TM)                                                                        \
    do {                                                                                          \
        auto kern = verify_sample_scan_kernel<BF, TM>;                                            \
        const size_t dyn = TM ? 2 * (size_t)CHUNK * (BF ? 2 : 4) : 0;                             \
        if (prep_stream_kernel(kern, dyn) != DFLASH2_OK) return DFLASH2_ECUDA;                    \
        kern<<<persistent_grid(kern, NT, dyn, units), NT, dyn, s>>>(                              \
            target, q, G, V, (int)S, rows_per_seq, units, inv_temperature, c2, draft_tok, seed,   \
            step, seq_id, q_mode, n_accept, out_tok, ratio_dbg, u_dbg, part, info, counters);     \
        verify_sample_draw_kernel<BF, TM><<<grid2, NT, 0, s>>>(target, q, G, V, (int)S, c2,        \
                                                               inv_temperature, info, part2,      \
                                                               counters + B, out_tok);            \
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
