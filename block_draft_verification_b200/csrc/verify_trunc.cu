// verify_trunc.cu -- sampling verify of target and drafter distributions
// truncated by top-k and top-p, the sampling settings a serving stack applies.
//
// Source: "DFlash 2: un drafter de 3.43× que cae a 1.45× bajo carga"
// (latenode.com), section "Preguntas frecuentes": the Qwen targets are sampled
// at temperature 1.0, top-p 0.95, top-k 20.  The pages do not say how
// truncation meets the verification; the reading here is that the truncated
// distribution is the one a token is drawn from, so the verification keeps the
// truncated target p~ exactly against the drafter's truncated q~ (rejection
// sampling as in "DFlash 2 — 3× plus de tokens sur Qwen3.8-27B, même sortie"
// (tamsi.dev), section "Les chiffres qui comptent sur Qwen3.8-27B").
//
// Truncation of one row, z = x * invT: order the tokens by (z descending,
// index ascending), keep the first min(top_k, V), renormalise over them, keep
// the shortest prefix whose cumulative sum reaches top_p (at least one), and
// renormalise again.  The full-row normaliser cancels in every step, so a row
// is described completely by its top_k values: the kernel streams every row
// once for its exact top 32 (value, -index) keys -- a maximum and a filter per
// element, no exponentials -- and the sequence's decision works on those
// lists alone.
//
// One launch.  Units are (sequence, row, 8 KB chunk): rows 0..G of a sequence
// are its target rows, G+1..2G its draft rows (q_mode softmax).  One CTA per
// SM takes a contiguous range of units and each warp a contiguous part of it
// through its own two-slot TMA ring (ring.cuh).  A warp keeps a running top-32
// of its consecutive chunks of one row (a segment) and leaves it with the
// segment's last chunk; the warp whose publish completes a row merges the
// segment lists into the row's top 32; the warp completing a sequence's last
// row truncates every row of the sequence in fp64, takes the accept tests with
// the Philox uniforms and draws the last token from its row's kept tokens in
// index order.  No warp waits for another.
#include "common.cuh"
#include "ring.cuh"
#include "workspace.cuh"

namespace dfl {

constexpr int KT = TRUNC_K;  // keys kept per row: top_k <= 32

// Candidate buffer of one warp: keys pushed by the filter, merged into the
// running list whenever more than TC_FLUSH wait (at most 32 lanes x 8
// elements arrive between two checks) and at the end of every chunk.  The
// count of waiting keys lives in a register of the warp (the same value in
// every lane).
constexpr unsigned TC_FLUSH = 64;
constexpr unsigned TC_CAP = TC_FLUSH + 32 * 8;
struct CandBuf32 {
    uint64_t key[TC_CAP];
    uint64_t out[KT];  // the merged list, placed by rank
};

// The 32 largest of a descending list (one key per lane, 0 = empty) and an
// ascending one: the elementwise maximum holds them as a bitonic sequence,
// which the bitonic merge sorts descending.
__device__ __forceinline__ uint64_t merge_desc_asc(uint64_t desc, uint64_t asc) {
    return warp_merge_desc(desc > asc ? desc : asc);
}

// Merge the n buffered candidates into the running list (one key per lane,
// descending; 0 = empty) up to 32 at a time, by rank: every key of the union
// (keys are distinct) lands at its rank in it, so a batch costs one broadcast
// read, a ballot and two compares per buffered key, and no sort.  Then the
// bound rises to the list's 32nd key; once the list is full its 32nd value
// also raises the row's shared bound (thr: ord32 of a value at least 32 of
// the row's elements reach; pub: what this warp last put there).
// Warp-uniform; n is zero on return.
__device__ __forceinline__ void flush32(CandBuf32& cb, unsigned& n, uint64_t& run,
                                        uint64_t& tkey, float& tv, unsigned* thr,
                                        uint32_t& pub) {
    const int lane = threadIdx.x & 31;
    __syncwarp();  // every lane's pushed keys are visible
    for (unsigned base = 0; base < n; base += 32) {
        const unsigned m = min(32u, n - base);
        const uint64_t c = (unsigned)lane < m ? cb.key[base + lane] : 0ull;
        unsigned rank_list = 0u;  // list keys above this lane's candidate
        unsigned rank_new = 0u;   // batch keys above this lane's candidate
        unsigned above_run = 0u;  // batch keys above this lane's list key
#pragma unroll 4
        for (unsigned j = 0; j < m; ++j) {
            const uint64_t cj = cb.key[base + j];
            const unsigned above = __ballot_sync(FULL, run > cj);
            if ((unsigned)lane == j) rank_list = __popc(above);
            rank_new += cj > c;
            above_run += cj > run;
        }
        cb.out[lane] = 0ull;
        __syncwarp();
        const unsigned pc = rank_list + rank_new;
        if ((unsigned)lane < m && pc < (unsigned)KT) cb.out[pc] = c;
        const unsigned pr = (unsigned)lane + above_run;
        if (run != 0ull && pr < (unsigned)KT) cb.out[pr] = run;
        __syncwarp();
        run = cb.out[lane];
        __syncwarp();  // out is read before the next batch writes it
    }
    n = 0u;
    const uint64_t k32 = shfl64(run, KT - 1);
    if (k32 > tkey) {
        tkey = k32;
        tv = key_value(k32);
    }
    const uint32_t o32 = (uint32_t)(k32 >> 32);
    if (o32 > pub) {
        pub = o32;
        if (lane == 0) atomicMax(thr, o32);
    }
}

// One chunk, one warp: the running top-32 `run` of the row segment updated
// with the chunk's elements.  Pass 1 keeps every vector's packed maximum.
// The bound: the list's 32nd key once it is full; before, the smallest lane
// maximum when every lane holds an element (each lane maximum is an element,
// so at least 32 elements reach it); the row's shared bound when higher
// (`shared`: its value as read one chunk earlier, a valid, looser bound).  No
// element below the bound can be in the row's top 32, so only vectors whose
// maximum reaches it are looked at (one per lane per round: its elements are
// compared with the bound's value and keys built only for those that reach
// it), and the merged row list is the exact top 32 whatever the timing.
template <bool BF16, class View>
__device__ __forceinline__ void top32_chunk(const View& v, CandBuf32& cb, uint64_t& run,
                                            unsigned* thr, uint32_t& pub, uint32_t shared) {
    using C = ChunkT<BF16>;
    const int lane = threadIdx.x & 31, nv = v.nvec();
    uint32_t vm[NVL];
    const float m = chunk_pass1<BF16>(v, vm);
    float tv = -INFINITY;
    uint64_t tkey = shfl64(run, KT - 1);
    if (tkey != 0ull) {
        tv = key_value(tkey);
    } else if (__all_sync(FULL, m != -INFINITY)) {
        uint32_t o = ord32(m);
#pragma unroll
        for (int j = 16; j > 0; j >>= 1) o = min(o, __shfl_xor_sync(FULL, o, j));
        tv = unord32(o);
        tkey = ((uint64_t)o << 32) - 1ull;  // below every key of value tv
        if (o > pub) {  // 32 lane maxima reach it: a bound for the whole row, shared now
            pub = o;
            if (lane == 0) atomicMax(thr, o);
        }
    }
    if (shared != 0u && (((uint64_t)shared << 32) - 1ull) > tkey) {
        tkey = ((uint64_t)shared << 32) - 1ull;
        tv = unord32(shared);
    }
    const uint32_t t2 = (tv == -INFINITY) ? C::NEG_INF_WORD : pack_value<BF16>(tv);
    uint32_t hits = 0;
#pragma unroll
    for (int i = 0; i < NVL; ++i)
        if (32 * i + lane < nv && any_ge<BF16>(vm[i], t2)) hits |= 1u << i;
    if (!__any_sync(FULL, hits != 0u)) return;
    unsigned nbuf = 0u;  // keys waiting in cb (warp-uniform)
    while (__any_sync(FULL, hits != 0u)) {  // one vector per lane per round
        unsigned em = 0u;  // elements of the lane's vector that reach the bound
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        int q = 0;
        if (hits) {
            const int i = __ffs(hits) - 1;
            hits &= hits - 1u;
            q = 32 * i + lane;
            w = v.vec(q);
#pragma unroll
            for (int e = 0; e < C::VW; ++e)
                if (C::elem(w, e) >= tv) em |= 1u << e;
            // elements past the chunk's end read as -inf: they reach only a -inf bound
            const int lim = v.n - q * C::VW;
            if (lim < C::VW) em &= lim > 0 ? (1u << lim) - 1u : 0u;
        }
        // Keys whose value equals the bound's but whose index part is below
        // the list's 32nd key are pushed too: the merge ranks them out.
        // This round's keys appended in lane order: the exclusive prefix of
        // the per-lane counts (at most 8: four bits) from four ballots.
        const unsigned cnt = __popc(em);
        const unsigned below = (1u << lane) - 1u;
        unsigned excl = 0u, total = 0u;
#pragma unroll
        for (int bit = 0; bit < 4; ++bit) {
            const unsigned bb = __ballot_sync(FULL, (cnt >> bit) & 1u);
            excl += (unsigned)__popc(bb & below) << bit;
            total += (unsigned)__popc(bb) << bit;
        }
        unsigned pos = nbuf + excl;
        while (em) {
            const int e = __ffs(em) - 1;
            em &= em - 1u;
            cb.key[pos++] = make_key(C::elem_at(w, e), (uint32_t)v.index(q, e));
        }
        nbuf += total;
        if (nbuf > TC_FLUSH) flush32(cb, nbuf, run, tkey, tv, thr, pub);
    }
    if (nbuf > 0u) flush32(cb, nbuf, run, tkey, tv, thr, pub);
}

static_assert(sizeof(List32) == KT * sizeof(uint64_t), "one segment list per unit");

// The row's top 32 from its segment lists, by the warp whose publish
// completed the row: the chunks' first keys in one round, then the lists
// four at a time, each merged as an ascending list into the descending
// accumulator.  Every lane returns its key of the row list.
__device__ __forceinline__ uint64_t row_merge32(const List32* P, int S) {
    const int lane = threadIdx.x & 31;
    auto ld = [](const uint64_t* p) { return (uint64_t)__ldcg((const unsigned long long*)p); };
    uint64_t acc = 0ull;
    for (int c0 = 0; c0 < S; c0 += 32) {
        const int c = c0 + lane;
        const uint64_t k0 = (c < S) ? ld(&P[c].key[0]) : 0ull;
        unsigned has = __ballot_sync(FULL, k0 != 0ull);
        while (has) {
            constexpr int PF = 4;
            uint64_t kv[PF];
            int nl = 0;
#pragma unroll
            for (int j = 0; j < PF; ++j) {
                kv[j] = 0ull;
                if (has) {
                    const int cc = c0 + __ffs(has) - 1;
                    has &= has - 1u;
                    kv[j] = ld(&P[cc].key[KT - 1 - lane]);  // ascending
                    ++nl;
                }
            }
#pragma unroll
            for (int j = 0; j < PF; ++j)
                if (j < nl) acc = merge_desc_asc(acc, kv[j]);
        }
    }
    return acc;
}

// ---------------------------------------------------------------- the decision
__device__ __forceinline__ double warp_sum_d(double s) {
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) s += __shfl_xor_sync(FULL, s, j);
    return s;
}
__device__ __forceinline__ double warp_scan_d(double x) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 1; k < 32; k <<= 1) {
        const double o = __shfl_up_sync(FULL, x, k);
        if (lane >= k) x += o;
    }
    return x;
}

// One row truncated (lane i holds the row's i-th key): its token and, if it
// is kept, its truncated probability (fp64); 0 and not kept otherwise.
struct TruncLane {
    int32_t tok;
    bool kept;
    double p;
};
__device__ __forceinline__ TruncLane truncate_row(uint64_t key, int kk, double invT,
                                                  double top_p) {
    const int lane = threadIdx.x & 31;
    const bool valid = key != 0ull && lane < kk;
    const double z = valid ? (double)key_value(key) * invT : 0.0;
    const double zmax = __shfl_sync(FULL, z, 0);
    const double e = valid ? exp(z - zmax) : 0.0;
    int kp = kk;
    if (top_p < 1.0) {
        const double sk = warp_sum_d(e);
        const double c = warp_scan_d(e) / sk;
        const unsigned reach = __ballot_sync(FULL, valid && c >= top_p);
        if (reach) kp = __ffs(reach);
    }
    TruncLane t;
    t.kept = valid && lane < kp;
    const double sp = warp_sum_d(t.kept ? e : 0.0);
    t.p = t.kept ? e / sp : 0.0;
    t.tok = valid ? (int32_t)key_index(key) : -1;
    return t;
}
// The truncated probability of token v in a truncated row (0 if not kept).
__device__ __forceinline__ double prob_of(const TruncLane& t, int32_t v) {
    const unsigned hit = __ballot_sync(FULL, t.kept && t.tok == v);
    return hit ? __shfl_sync(FULL, t.p, __ffs(hit) - 1) : 0.0;
}

// The decision of one sequence from its row lists (target rows 0..G at
// L[0..G], draft rows at L[G+1..2G] in softmax mode), one warp.
__device__ __noinline__ void trunc_decide(const uint64_t* __restrict__ L, int G, int kk,
                                          double invT, double top_p, int q_mode,
                                          const int32_t* __restrict__ dtok, uint64_t seed,
                                          uint32_t step, uint32_t sid, int32_t* __restrict__ n_out,
                                          int32_t* __restrict__ out, float* __restrict__ ratio_dbg,
                                          float* __restrict__ u_dbg) {
    const int lane = threadIdx.x & 31;
    const bool soft = q_mode == DFLASH2_Q_SOFTMAX;
    auto ld = [&](int r) { return (uint64_t)__ldcg((const unsigned long long*)L + (int64_t)r * KT + lane); };
    const int32_t dl = (lane < G) ? dtok[lane] : -1;
    int n = G;
    const bool all_ratios = ratio_dbg != nullptr;
    for (int j = 0; j < G; ++j) {
        const uint64_t kt = ld(j);
        const uint64_t kq = soft ? ld(G + 1 + j) : 0ull;
        const int32_t d = __shfl_sync(FULL, dl, j);
        const TruncLane pt = truncate_row(kt, kk, invT, top_p);
        const double p = prob_of(pt, d);
        double r = p;
        if (soft) {
            const double q = prob_of(truncate_row(kq, kk, invT, top_p), d);
            r = (q > 0.0) ? p / q : (p > 0.0 ? INFINITY : 0.0);
        }
        const float u = philox_uniform(seed, step, sid, (uint32_t)j, 0u);
        if (lane == 0) {
            if (ratio_dbg) ratio_dbg[j] = (float)r;
            if (u_dbg) u_dbg[j] = u;
        }
        if (n == G && !((double)u < r)) {
            n = j;
            if (!all_ratios && !u_dbg) break;
        }
    }
    // the draw from row n: its kept tokens in index order
    const TruncLane P = truncate_row(ld(n), kk, invT, top_p);
    const int32_t d_n = (n < G) ? __shfl_sync(FULL, dl, n) : -1;
    double w = P.p;
    if (n < G) {
        if (soft) {
            const TruncLane Q = truncate_row(ld(G + 1 + n), kk, invT, top_p);
            double q = 0.0;
            for (int l = 0; l < 32; ++l) {  // q~_n at this lane's token
                const int32_t qt = __shfl_sync(FULL, Q.tok, l);
                const double qp = __shfl_sync(FULL, Q.p, l);
                const bool qk = __shfl_sync(FULL, Q.kept, l);
                if (qk && qt == P.tok) q = qp;
            }
            w = P.kept ? fmax(0.0, P.p - q) : 0.0;
        } else {
            w = (P.kept && P.tok != d_n) ? P.p : 0.0;
        }
        if (!(warp_sum_d(w) > 0.0)) w = P.p;  // the residual is empty by rounding
    }
    const double R = warp_sum_d(w);
    const double t = (double)philox_uniform(seed, step, sid, (uint32_t)n, 1u) * R;
    // inclusive prefix in index order at this lane's token
    double C = 0.0;
    for (int l = 0; l < 32; ++l) {
        const int32_t ot = __shfl_sync(FULL, P.tok, l);
        const double ow = __shfl_sync(FULL, w, l);
        const bool ok = __shfl_sync(FULL, P.kept, l);
        if (ok && ot <= P.tok) C += ow;
    }
    const bool cross = P.kept && C > t;
    int32_t best = cross ? P.tok : INT32_MAX;
    int32_t last = (P.kept && w > 0.0) ? P.tok : -1;
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) {
        best = min(best, __shfl_xor_sync(FULL, best, j));
        last = max(last, __shfl_xor_sync(FULL, last, j));
    }
    const int32_t pick = (best != INT32_MAX) ? best : last;
    if (lane <= G) out[lane] = (lane < n) ? dl : (lane == n ? pick : -1);
    if (lane == 0) *n_out = n;
}

// ---------------------------------------------------------------- the kernel
// Control words (zero on entry, zero again on exit): per row a counter and a
// shared top-32 bound, per sequence a counter of finished rows.
template <bool BF16, bool TMA>
__global__ void __launch_bounds__(RING_THREADS, 1) verify_trunc_kernel(
    const void* __restrict__ target, const void* __restrict__ draft, int B, int G, int64_t V,
    int S, int rows_per_seq, int64_t units, int kk, double invT, double top_p,
    const int32_t* __restrict__ draft_tok, uint64_t seed, uint32_t step,
    const uint32_t* __restrict__ seq_id, int q_mode, int32_t* __restrict__ n_accept,
    int32_t* __restrict__ out_tok, float* __restrict__ ratio_dbg, float* __restrict__ u_dbg,
    List32* __restrict__ part, uint64_t* __restrict__ rowlist, unsigned* __restrict__ ctl) {
    using Ch = ChunkT<BF16>;
    constexpr int ES = Ch::ES;
    constexpr int LEN = Ch::LEN;
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ __align__(8) uint64_t bars[2 * NCW];
    __shared__ CandBuf32 cbuf[NCW];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t nrows = (int64_t)B * rows_per_seq;
    unsigned* const rowcnt = ctl;
    unsigned* const thr = ctl + nrows;
    unsigned* const seqcnt = ctl + 2 * nrows;
    CandBuf32& cb = cbuf[warp];
    auto rowp = [&](int64_t b, int rr) {
        return (rr <= G) ? (const char*)target + (b * (G + 1) + rr) * V * ES
                         : (const char*)draft + (b * G + (rr - G - 1)) * V * ES;
    };
    int64_t lo, hi;
    warp_range(units, lo, hi);
    const int n = (int)(hi - lo);
    UnitCursor uc, ic;
    uc.init(lo, S, rows_per_seq);
    ic = uc;
    auto src = [&](const UnitCursor& cu, const char*& p, uint32_t& bytes) {
        const int64_t v0 = (int64_t)cu.c * LEN;
        p = rowp(cu.g, cu.r) + v0 * ES;
        bytes = (uint32_t)(min((int64_t)LEN, V - v0) * ES);
    };
    WarpRing r{nullptr, 0u};
    if (TMA) r = warp_ring_start(ring, bars, n, ic, Ch::NEG_INF_WORD, src);
    __syncwarp();
    uint64_t run = 0ull;
    unsigned seg = 0;
    uint32_t pub = 0u;
    // the row's shared bound, read one unit ahead: it only rises while the
    // row is open (and its last unit is still to come), so an older value is
    // a valid, slightly looser bound
    uint32_t thr_now = n > 0 ? *(volatile unsigned*)&thr[uc.g * rows_per_seq + uc.r] : 0u;
    for (int k = 0; k < n; ++k, uc.next()) {
        const int64_t b = uc.g, v0 = (int64_t)uc.c * LEN;
        const int64_t grow = b * rows_per_seq + uc.r;
        const int len = (int)min((int64_t)LEN, V - v0);
        const uint32_t thr_ahead =
            k + 1 < n ? *(volatile unsigned*)&thr[uc.last_of_row() ? grow + 1 : grow] : 0u;
        if (TMA) {
            if (!r.wait(k)) {
                warp_ring_abort(r, k, n);
                return;
            }
            top32_chunk<BF16>(SmemView<BF16>{r.slot(k), v0, len}, cb, run, &thr[grow], pub,
                              thr_now);
            warp_ring_next(r, k, n, ic, Ch::NEG_INF_WORD, src);
        } else {
            top32_chunk<BF16>(GlobalView<BF16>{(const uint8_t*)rowp(b, uc.r), v0, len}, cb, run,
                              &thr[grow], pub, thr_now);
        }
        thr_now = thr_ahead;
        ++seg;
        const bool seg_end = (k + 1 == n) || uc.last_of_row();
        if (!seg_end) {  // no list at this chunk (the entry may hold an earlier call's)
            if (lane == 0) part[grow * S + uc.c].key[0] = 0ull;
            continue;
        }
        part[grow * S + uc.c].key[lane] = run;  // the segment's list (key[0] = 0: empty)
        __syncwarp();
        bool last = false;
        if (lane == 0) last = publish(&rowcnt[grow], seg, (unsigned)S);
        run = 0ull;
        seg = 0;
        pub = 0u;
        if (!__shfl_sync(FULL, last, 0)) continue;
        __syncwarp();  // lane 0's acquire covers the whole warp's reads
        // every chunk of the row is in: its top 32
        const uint64_t acc = row_merge32(part + grow * S, S);
        rowlist[grow * KT + lane] = acc;
        if (lane == 0) {
            rowcnt[grow] = 0u;
            thr[grow] = 0u;
        }
        __syncwarp();
        bool lastrow = false;
        if (lane == 0) lastrow = publish(&seqcnt[b], 1u, (unsigned)rows_per_seq);
        if (!__shfl_sync(FULL, lastrow, 0)) continue;
        __syncwarp();
        // every row of the sequence is in: decide it
        trunc_decide(rowlist + b * rows_per_seq * KT, G, kk, invT, top_p, q_mode,
                     draft_tok + b * G, seed, step, seq_id ? seq_id[b] : (uint32_t)b,
                     &n_accept[b], out_tok + b * (G + 1), ratio_dbg ? ratio_dbg + b * G : nullptr,
                     u_dbg ? u_dbg + b * G : nullptr);
        if (lane == 0) seqcnt[b] = 0u;
    }
}

}  // namespace dfl

using namespace dfl;
using namespace dfl_host;

extern "C" int dflash2_verify_sample_trunc(const void* target, const void* draft, int dtype, int B,
                                           int G, int64_t V, const int32_t* draft_tok,
                                           float inv_temperature, int top_k, float top_p,
                                           uint64_t seed, uint32_t step, const uint32_t* seq_id,
                                           int q_mode, int32_t* n_accept, int32_t* out_tok,
                                           float* ratio_dbg, float* u_dbg, void* ws,
                                           size_t ws_bytes, dflash2_stream_t stream) {
    if (!dtype_ok(dtype)) return DFLASH2_EDTYPE;
    if (B < 0 || G < 1 || G >= DFLASH2_MAX_BLOCK || V < 1 || V > INT32_MAX) return DFLASH2_ESHAPE;
    if (top_k < 1 || top_k > KT) return DFLASH2_ESHAPE;
    if (!finite_pos(inv_temperature) || !finite_pos(top_p) || top_p > 1.0f) return DFLASH2_EINVAL;
    if (q_mode != DFLASH2_Q_SOFTMAX && q_mode != DFLASH2_Q_ONEHOT) return DFLASH2_EINVAL;
    if (B == 0) return DFLASH2_OK;
    if (!target || !draft_tok || !n_accept || !out_tok) return DFLASH2_EINVAL;
    if (q_mode == DFLASH2_Q_SOFTMAX && !draft) return DFLASH2_EINVAL;
    const int es = elem_size(dtype);
    if (!aligned(target, es) || (draft && !aligned(draft, es)) || !aligned(draft_tok, 4) ||
        !aligned(n_accept, 4) || !aligned(out_tok, 4) || (seq_id && !aligned(seq_id, 4)) ||
        (ratio_dbg && !aligned(ratio_dbg, 4)) || (u_dbg && !aligned(u_dbg, 4)))
        return DFLASH2_EALIGN;
    const int64_t S = row_chunks(V, es);
    const int rows_per_seq = (q_mode == DFLASH2_Q_SOFTMAX) ? 2 * G + 1 : G + 1;
    const int64_t units = (int64_t)B * rows_per_seq * S;
    if (units > (int64_t)INT32_MAX) return DFLASH2_ESHAPE;
    const Layout L = trunc_layout(B, G, V, es);
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return DFLASH2_EWORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned* ctl = (unsigned*)((char*)ws + L.counters_off);
    List32* part = (List32*)((char*)ws + L.part_off);
    uint64_t* rowlist = (uint64_t*)((char*)ws + L.part2_off);
    if (!L.self_clean && cudaMemsetAsync(ctl, 0, L.counters_bytes, s) != cudaSuccess)
        return DFLASH2_ECUDA;
    const void* q = (q_mode == DFLASH2_Q_SOFTMAX) ? draft : nullptr;
    const bool tma = aligned(target, 16) && (!q || aligned(q, 16)) && (V * es) % 16 == 0;
    const int kk = (int)((int64_t)top_k < V ? (int64_t)top_k : V);
    const double invT = (double)inv_temperature, tp = (double)top_p;
#define DFL_TRUNC(BF, TM)                                                                        \
    do {                                                                                         \
        auto kern = verify_trunc_kernel<BF, TM>;                                                 \
        const size_t dyn = TM ? (size_t)RING_BYTES : 0;                                          \
        if (ring_prepare(kern, dyn) != DFLASH2_OK) return DFLASH2_ECUDA;                         \
        kern<<<ring_grid(units), RING_THREADS, dyn, s>>>(                                        \
            target, q, B, G, V, (int)S, rows_per_seq, units, kk, invT, tp, draft_tok, seed,      \
            step, seq_id, q_mode, n_accept, out_tok, ratio_dbg, u_dbg, part, rowlist, ctl);      \
    } while (0)
    if (dtype == DFLASH2_BF16) {
        if (tma) DFL_TRUNC(true, true);
        else DFL_TRUNC(true, false);
    } else {
        if (tma) DFL_TRUNC(false, true);
        else DFL_TRUNC(false, false);
    }
#undef DFL_TRUNC
    return launch_status();
}

unsigned dfl_errors_trunc(int clear) {
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_dev_err, sizeof v) != cudaSuccess) return 0xFFFFFFFFu;
    if (clear && v) {
        unsigned z = 0;
        cudaMemcpyToSymbol(g_dev_err, &z, sizeof z);
    }
    return v;
}
