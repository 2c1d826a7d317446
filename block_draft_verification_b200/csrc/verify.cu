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
// Both verifies stream every logit row once in 16384-element chunks, one CTA
// per (sequence, row, chunk).  The last CTA of a sequence (arrival ticket, no
// waiting) reduces the per-chunk partials in chunk order and decides.  The
// sampling draw needs the normalisers first, so it is a second kernel: one
// CTA per chunk of the one row each sequence draws from (L2-resident after
// the first pass), then the last of them finds the chunk where the inverse
// CDF crosses t = u' * R and scans only that chunk.  No probability vector is
// ever written to memory.
#include "common.cuh"
#include "workspace.cuh"

namespace dfl {

constexpr double LOG2E = 1.4426950408889634;

// ------------------------------------------------------------------ greedy
template <bool BF16, bool VEC>
__global__ void __launch_bounds__(NT) verify_greedy_kernel(
    const void* __restrict__ target, int G, int64_t V, int S, const int32_t* __restrict__ draft_tok,
    int32_t* __restrict__ n_accept, int32_t* __restrict__ out_tok, uint64_t* __restrict__ part,
    unsigned* __restrict__ counters) {
    using R = Row<BF16>;
    __shared__ float s_max[NT / 32];
    __shared__ unsigned s_first;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int units = (G + 1) * S;
    const int b = blockIdx.x / units;
    const int rem = blockIdx.x - b * units;
    const int j = rem / S, chunk = rem - j * S;
    const int64_t row = (int64_t)b * (G + 1) + j;
    const int64_t v0 = (int64_t)chunk * CHUNK, vend = min(V, v0 + (int64_t)CHUNK);

    uint4 r[R::NV];
    R::template load<VEC>((const char*)target + row * V * (BF16 ? 2 : 4), v0, vend, r);
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < R::NV; ++i)
#pragma unroll
        for (int e = 0; e < R::VW; ++e) m = fmaxf(m, R::elem(r[i], e));
    float wm = m;
#pragma unroll
    for (int k = 16; k > 0; k >>= 1) wm = fmaxf(wm, __shfl_xor_sync(FULL, wm, k));
    if (lane == 0) s_max[warp] = wm;
    if (t == 0) s_first = 0xFFFFFFFFu;
    __syncthreads();
    float M = s_max[0];
#pragma unroll
    for (int w = 1; w < NT / 32; ++w) M = fmaxf(M, s_max[w]);
    // the lowest index holding the chunk max (-0 == +0 in the compare)
    if (m == M) {
        uint32_t first = 0xFFFFFFFFu;
#pragma unroll
        for (int i = R::NV - 1; i >= 0; --i)
#pragma unroll
            for (int e = R::VW - 1; e >= 0; --e)
                if (R::elem(r[i], e) == M) first = (uint32_t)R::index_of(v0, i, e);
        atomicMin(&s_first, first);
    }
    __syncthreads();
    if (t == 0) {
        part[row * S + chunk] = make_key(M, s_first);
        __threadfence();
    }
    if (!arrive_last(&counters[b], (unsigned)units)) return;
    if (warp != 0) return;

    // lane j reduces target row j over its chunks (G + 1 <= 32 rows)
    uint64_t best = 0;
    if (lane <= G) {
        const uint64_t* P = part + ((int64_t)b * (G + 1) + lane) * S;
        for (int c = 0; c < S; ++c) {
            uint64_t k = (uint64_t)__ldcg((const unsigned long long*)&P[c]);
            best = k > best ? k : best;
        }
    }
    const int32_t tj = (int32_t)key_index(best);
    const int32_t dj = (lane < G) ? draft_tok[(int64_t)b * G + lane] : -1;
    const unsigned miss = __ballot_sync(FULL, lane < G && dj != tj);
    const int n = miss ? (__ffs(miss) - 1) : G;
    if (lane <= G) {
        int32_t o = -1;
        if (lane < n) o = dj;
        else if (lane == n) o = tj;
        out_tok[(int64_t)b * (G + 1) + lane] = o;
    }
    if (lane == 0) n_accept[b] = n;
}

// ------------------------------------------------------------------ sampling, pass 1
// Units: for sequence b, rows 0..G are target rows, G+1..2G draft rows (softmax
// mode only).  Each unit writes its (max, fp64 sum-exp) partial.
template <bool BF16, bool VEC>
__global__ void __launch_bounds__(NT) verify_sample_scan_kernel(
    const void* __restrict__ target, const void* __restrict__ draft, int G, int64_t V, int S,
    int rows_per_seq, float inv_t, float c2, const int32_t* __restrict__ draft_tok, uint64_t seed,
    uint32_t step, const uint32_t* __restrict__ seq_id, int q_mode, int32_t* __restrict__ n_accept,
    int32_t* __restrict__ out_tok, float* __restrict__ ratio_dbg, float* __restrict__ u_dbg,
    LseD* __restrict__ part, SampleInfo* __restrict__ info, unsigned* __restrict__ counters) {
    using R = Row<BF16>;
    constexpr int ES = BF16 ? 2 : 4;
    __shared__ LseD s_lse[NT / 32];
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int units = rows_per_seq * S;
    const int b = blockIdx.x / units;
    const int rem = blockIdx.x - b * units;
    const int rr = rem / S, chunk = rem - rr * S;
    const int64_t v0 = (int64_t)chunk * CHUNK, vend = min(V, v0 + (int64_t)CHUNK);
    const char* rowp = (rr <= G)
                           ? (const char*)target + ((int64_t)b * (G + 1) + rr) * V * ES
                           : (const char*)draft + ((int64_t)b * G + (rr - G - 1)) * V * ES;

    uint4 r[R::NV];
    R::template load<VEC>(rowp, v0, vend, r);
    LseD mine = thread_lse_d<BF16>(r, c2);
    LseD wl = warp_lse(mine, c2);
    if (lane == 0) s_lse[warp] = wl;
    __syncthreads();
    if (t == 0) {
        LseD tot = s_lse[0];
        for (int w = 1; w < NT / 32; ++w) tot = lse_merge(tot, s_lse[w], c2);
        part[((int64_t)b * rows_per_seq + rr) * S + chunk] = tot;
        __threadfence();
    }
    if (!arrive_last(&counters[b], (unsigned)units)) return;
    if (warp != 0) return;

    // Lane j: logZ of target row j (j <= G) and of draft row j (j < G), in
    // chunk order; then the ratio and the accept test of position j.
    auto row_lse = [&](int rrow) {
        const LseD* P = part + ((int64_t)b * rows_per_seq + rrow) * S;
        LseD acc{-INFINITY, 0.0f, 0.0};
        for (int c = 0; c < S; ++c) {
            LseD p;
            p.m = __ldcg(&P[c].m);
            p.pad = 0.0f;
            p.s = __ldcg(&P[c].s);
            acc = lse_merge(acc, p, c2);
        }
        return acc;
    };
    const uint32_t sid = seq_id ? seq_id[b] : (uint32_t)b;
    LseD lt{-INFINITY, 0.0f, 0.0}, lq{-INFINITY, 0.0f, 0.0};
    if (lane <= G) lt = row_lse(lane);
    if (q_mode == DFLASH2_Q_SOFTMAX && lane < G) lq = row_lse(G + 1 + lane);
    bool reject = false;
    if (lane < G) {
        const int32_t d = draft_tok[(int64_t)b * G + lane];
        const char* trow = (const char*)target + ((int64_t)b * (G + 1) + lane) * V * ES;
        const double xt = BF16 ? (double)__uint_as_float((uint32_t)((const uint16_t*)trow)[d] << 16)
                               : (double)((const float*)trow)[d];
        // lp = z_t[d] - logZ_t = ((x - m) * invT) - ln(s)
        double lr = (xt - (double)lt.m) * (double)inv_t - log(lt.s);
        if (q_mode == DFLASH2_Q_SOFTMAX) {
            const char* qrow = (const char*)draft + ((int64_t)b * G + lane) * V * ES;
            const double xq = BF16
                ? (double)__uint_as_float((uint32_t)((const uint16_t*)qrow)[d] << 16)
                : (double)((const float*)qrow)[d];
            lr -= (xq - (double)lq.m) * (double)inv_t - log(lq.s);
        }
        const double ratio = exp(lr);
        const float u = philox_uniform(seed, step, sid, (uint32_t)lane, 0u);
        reject = !((double)u < ratio);
        if (ratio_dbg) ratio_dbg[(int64_t)b * G + lane] = (float)ratio;
        if (u_dbg) u_dbg[(int64_t)b * G + lane] = u;
    }
    const unsigned rej = __ballot_sync(FULL, reject);
    const int n = rej ? (__ffs(rej) - 1) : G;
    const int32_t dn = (lane < G) ? draft_tok[(int64_t)b * G + lane] : -1;
    if (lane <= G) {
        // the drawn token at position n is written by the draw kernel
        out_tok[(int64_t)b * (G + 1) + lane] = (lane < n) ? dn : -1;
    }
    const float ltm = __shfl_sync(FULL, lt.m, n);
    const double lts = __shfl_sync(FULL, lt.s, n);
    const float lqm = __shfl_sync(FULL, lq.m, n);
    const double lqs = __shfl_sync(FULL, lq.s, n);
    const int32_t d_n = __shfl_sync(FULL, dn, n);
    if (lane == 0) {
        SampleInfo I;
        I.mt = ltm;
        I.l2t = (float)log2(lts);
        I.mq = lqm;
        const bool resid = n < G && q_mode == DFLASH2_Q_SOFTMAX;
        I.l2q = resid ? (float)log2(lqs) : 0.0f;
        I.dl = resid ? (float)(((double)ltm - (double)lqm) * (double)inv_t + log(lts) - log(lqs))
                     : 0.0f;
        I.pad = 0;
        I.u_res = philox_uniform(seed, step, sid, (uint32_t)n, 1u);
        I.n = n;
        I.mode = (n == G) ? 2 : (q_mode == DFLASH2_Q_SOFTMAX ? 0 : 1);
        I.d = d_n;
        info[b] = I;
        n_accept[b] = n;
    }
}

// ------------------------------------------------------------------ sampling, pass 2
// The draw weights of element v of the row the sequence draws from:
//   p_v = exp2((x_v - mt) * c - l2t),  q_v likewise,
//   mode 0: w = max(0, p - q), evaluated as q * expm1(ln p - ln q) with
//           ln p - ln q = (xt - xq) * invT - (logZ_t - logZ_q): the same
//           value, without the cancellation of p - q when p and q agree;
//   mode 1: w = p, 0 at d;  mode 2: w = p.
// The fallback weight (R = 0) is p.
template <bool BF16>
__device__ __forceinline__ void draw_weight(const uint4& rt, const uint4& rq, int e, int64_t v,
                                            const SampleInfo& I, float c, float inv_t, float& w,
                                            float& p) {
    using R = Row<BF16>;
    const float xt = R::elem(rt, e);
    p = ex2((xt - I.mt) * c - I.l2t);
    if (I.mode == 0) {
        const float xq = R::elem(rq, e);
        const float q = ex2((xq - I.mq) * c - I.l2q);
        const float dlog = (xt - xq) * inv_t - I.dl;
        w = dlog > 0.0f ? q * expm1f(dlog) : 0.0f;
    } else if (I.mode == 1) {
        w = (v == I.d) ? 0.0f : p;
    } else {
        w = p;
    }
}

// Per-thread contiguous block of the chunk: thread t owns elements
// [v0 + t * 64, v0 + t * 64 + 64) as NV vectors, so a thread's running sum
// follows index order (needed by the inverse-CDF scan).
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
                    uint32_t bits = R::scalar_bits(row, vb + e);
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

template <bool BF16, bool VEC>
__global__ void __launch_bounds__(NT) verify_sample_draw_kernel(
    const void* __restrict__ target, const void* __restrict__ draft, int G, int64_t V, int S,
    float c2, float inv_t, const SampleInfo* __restrict__ info, double* __restrict__ part2,
    unsigned* __restrict__ counters2, int32_t* __restrict__ out_tok) {
    using R = Row<BF16>;
    constexpr int ES = BF16 ? 2 : 4;
    __shared__ double s_w[NT / 32], s_p[NT / 32];
    __shared__ double s_scan[NT];
    __shared__ int s_pick_thread;
    __shared__ int s_cstar;
    __shared__ double s_base, s_t;
    __shared__ int s_fallback, s_done, s_last;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int b = blockIdx.x / S, chunk = blockIdx.x - b * S;
    const SampleInfo I = info[b];
    const char* trow = (const char*)target + ((int64_t)b * (G + 1) + I.n) * V * ES;
    const char* qrow = (I.mode == 0) ? (const char*)draft + ((int64_t)b * G + I.n) * V * ES : nullptr;

    // chunk sums of w (and of p, for the fallback), fp64, thread order
    uint4 rt[R::NV], rq[R::NV];
#pragma unroll
    for (int i = 0; i < R::NV; ++i) rq[i] = make_uint4(0, 0, 0, 0);
    double sw = 0.0, sp = 0.0;
    {
        const int64_t v0 = (int64_t)chunk * CHUNK, vend = min(V, v0 + (int64_t)CHUNK);
        load_contig<BF16, VEC>(trow, v0, vend, rt);
        if (I.mode == 0) load_contig<BF16, VEC>(qrow, v0, vend, rq);
#pragma unroll
        for (int i = 0; i < R::NV; ++i)
#pragma unroll
            for (int e = 0; e < R::VW; ++e) {
                float w, p;
                draw_weight<BF16>(rt[i], rq[i], e, v0 + (int64_t)t * EPT + i * R::VW + e, I, c2, inv_t,
                                  w, p);
                sw += (double)w;
                sp += (double)p;
            }
    }
    double a = sw, bsum = sp;
#pragma unroll
    for (int k = 16; k > 0; k >>= 1) {
        a += __shfl_xor_sync(FULL, a, k);
        bsum += __shfl_xor_sync(FULL, bsum, k);
    }
    if (lane == 0) {
        s_w[warp] = a;
        s_p[warp] = bsum;
    }
    __syncthreads();
    if (t == 0) {
        double W = 0.0, Pp = 0.0;
        for (int w = 0; w < NT / 32; ++w) {
            W += s_w[w];
            Pp += s_p[w];
        }
        part2[((int64_t)b * S + chunk) * 2 + 0] = W;
        part2[((int64_t)b * S + chunk) * 2 + 1] = Pp;
        __threadfence();
    }
    if (!arrive_last(&counters2[b], (unsigned)S)) return;

    // Last chunk of this sequence: total mass, the chunk where the prefix
    // crosses t, then an in-chunk scan.
    if (t == 0) {
        const double* P2 = part2 + (int64_t)b * S * 2;
        double R_ = 0.0;
        for (int c = 0; c < S; ++c) R_ += __ldcg(&P2[c * 2]);
        int fb = 0;
        if (!(R_ > 0.0)) {  // residual empty by rounding: draw from p instead
            fb = 1;
            R_ = 0.0;
            for (int c = 0; c < S; ++c) R_ += __ldcg(&P2[c * 2 + 1]);
        }
        const double tt = (double)I.u_res * R_;
        double pre = 0.0;
        int cstar = -1, clast = 0;
        for (int c = 0; c < S; ++c) {
            const double wc = __ldcg(&P2[c * 2 + fb]);
            if (wc > 0.0) clast = c;
            if (cstar < 0 && pre + wc > tt) cstar = c;
            if (cstar < 0) pre += wc;
        }
        if (cstar < 0) {  // rounding left t at the top: last chunk with mass
            cstar = clast;
            pre = 0.0;
            for (int c = 0; c < clast; ++c) pre += __ldcg(&P2[c * 2 + fb]);
        }
        s_cstar = cstar;
        s_base = pre;
        s_t = tt;
        s_fallback = fb;
        s_pick_thread = NT;
        s_done = 0;
        s_last = -1;
    }
    __syncthreads();
    const int cstar = s_cstar;
    const int fb = s_fallback;
    const double tt = s_t;
    const int64_t v0 = (int64_t)cstar * CHUNK, vend = min(V, v0 + (int64_t)CHUNK);
    load_contig<BF16, VEC>(trow, v0, vend, rt);
    if (I.mode == 0) load_contig<BF16, VEC>(qrow, v0, vend, rq);
    float wreg[EPT];
    double mysum = 0.0;
#pragma unroll
    for (int i = 0; i < R::NV; ++i)
#pragma unroll
        for (int e = 0; e < R::VW; ++e) {
            float w, p;
            draw_weight<BF16>(rt[i], rq[i], e, v0 + (int64_t)t * EPT + i * R::VW + e, I, c2, inv_t, w,
                              p);
            wreg[i * R::VW + e] = fb ? p : w;
            mysum += (double)wreg[i * R::VW + e];
        }
    // inclusive scan of the thread sums in thread (= index) order
    s_scan[t] = mysum;
    __syncthreads();
    for (int off = 1; off < NT; off <<= 1) {
        double v = (t >= off) ? s_scan[t - off] : 0.0;
        __syncthreads();
        s_scan[t] += v;
        __syncthreads();
    }
    const double incl = s_base + s_scan[t];
    if (incl > tt) atomicMin(&s_pick_thread, t);
    __syncthreads();
    const int pt = s_pick_thread;
    if (pt < NT && t == pt) {
        double acc = s_base + (t > 0 ? s_scan[t - 1] : 0.0);
        int pick = -1, lastpos = -1;
        for (int k = 0; k < EPT; ++k) {
            const float w = wreg[k];
            if (w > 0.0f) lastpos = k;
            acc += (double)w;
            if (acc > tt) {
                pick = k;
                break;
            }
        }
        if (pick < 0) pick = lastpos;  // rounding: the last element with mass
        if (pick >= 0) {
            out_tok[(int64_t)b * (G + 1) + I.n] = (int32_t)(v0 + (int64_t)t * EPT + pick);
            s_done = 1;
        }
    }
    __syncthreads();
    if (!s_done) {  // block-uniform: rounding left t above the chunk's scan
        for (int k = EPT - 1; k >= 0; --k)
            if (wreg[k] > 0.0f) {
                atomicMax(&s_last, t * EPT + k);
                break;
            }
        __syncthreads();
        if (t == 0 && s_last >= 0) out_tok[(int64_t)b * (G + 1) + I.n] = (int32_t)(v0 + s_last);
    }
}

}  // namespace dfl

using namespace dfl;
using namespace dfl_host;

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
    if ((int64_t)B * (G + 1) * S > (int64_t)INT32_MAX) return DFLASH2_ESHAPE;
    const Layout L = greedy_layout(B, G, V);
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return DFLASH2_EWORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned* counters = (unsigned*)((char*)ws + L.counters_off);
    uint64_t* part = (uint64_t*)((char*)ws + L.part_off);
    if (cudaMemsetAsync(counters, 0, (size_t)B * 4, s) != cudaSuccess) return DFLASH2_ECUDA;
    const bool vec = aligned(target, 16) && (V * es) % 16 == 0;
    const dim3 grid((unsigned)((int64_t)B * (G + 1) * S)), block(NT);
#define DFL_GREEDY(BF, VE)                                                                      \
    verify_greedy_kernel<BF, VE><<<grid, block, 0, s>>>(target, G, V, (int)S, draft_tok, n_accept, \
                                                        out_tok, part, counters)
    if (dtype == DFLASH2_BF16) {
        if (vec) DFL_GREEDY(true, true);
        else DFL_GREEDY(true, false);
    } else {
        if (vec) DFL_GREEDY(false, true);
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
    if ((int64_t)B * rows_per_seq * S > (int64_t)INT32_MAX) return DFLASH2_ESHAPE;
    const Layout L = sample_layout(B, G, V);
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return DFLASH2_EWORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned* counters = (unsigned*)((char*)ws + L.counters_off);
    LseD* part = (LseD*)((char*)ws + L.part_off);
    double* part2 = (double*)((char*)ws + L.part2_off);
    SampleInfo* info = (SampleInfo*)((char*)ws + L.info_off);
    if (cudaMemsetAsync(counters, 0, (size_t)B * 2 * 4, s) != cudaSuccess) return DFLASH2_ECUDA;
    const bool vec = aligned(target, 16) && (!draft || aligned(draft, 16)) && (V * es) % 16 == 0;
    const float c2 = (float)((double)inv_temperature * LOG2E);
    const void* q = (q_mode == DFLASH2_Q_SOFTMAX) ? draft : nullptr;
    const dim3 grid1((unsigned)((int64_t)B * rows_per_seq * S)), grid2((unsigned)((int64_t)B * S));
    const dim3 block(NT);
#define DFL_SAMPLE(BF, VE)                                                                          \
    do {                                                                                            \
        verify_sample_scan_kernel<BF, VE><<<grid1, block, 0, s>>>(                                  \
            target, q, G, V, (int)S, rows_per_seq, inv_temperature, c2, draft_tok, seed, step,       \
            seq_id, q_mode, n_accept, out_tok, ratio_dbg, u_dbg, part, info, counters);             \
        verify_sample_draw_kernel<BF, VE><<<grid2, block, 0, s>>>(target, q, G, V, (int)S, c2,     \
                                                                  inv_temperature, info,        \
                                                                  part2, counters + B, out_tok);    \
    } while (0)
    if (dtype == DFLASH2_BF16) {
        if (vec) DFL_SAMPLE(true, true);
        else DFL_SAMPLE(true, false);
    } else {
        if (vec) DFL_SAMPLE(false, true);
        else DFL_SAMPLE(false, false);
    }
#undef DFL_SAMPLE
    return launch_status();
}
