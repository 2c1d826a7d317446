// topk_softmax.cu -- softmax over the vocabulary and the 16 best candidates of
// every drafted position, in one pass over the logits.
//
// Source: "DFlash 2 — 3× plus de tokens sur Qwen3.8-27B, même sortie"
// (tamsi.dev), section "L’idée, sans le papier": the right token lies in the
// drafter's top 16 far more often than at top 1, and the selector picks among
// those 16 per position; "DFlash 2" (myaiexp.com), section "主な機能": the
// path selector keeps the top-16 candidates of each position.
//
// Work unit: (row, chunk of 8 KB of logits).  One CTA per SM streams a
// contiguous range of units, each warp a contiguous part of it brought in by
// its own TMA bulk copies (rows whose start is 16-byte aligned; others are
// read element by element), and each warp reduces whole chunks on its own:
// the chunk maximum M, the sum of exp2(x c - fl(M c)) and the chunk's exact
// top-16, all in a fixed order, so a chunk's partial does not depend on the
// batch or the grid.  A unit's partial is published with one
// acquire-release add; the warp that completes a row (no warp waits) merges
// the chunk lists and softmax partials in chunk order and writes
// idx / prob / logp / logz.  Keys compare (value, -index) exactly, so the
// top-16 set does not depend on how the row was split.
#include <cuda.h>

#include "common.cuh"
#include "ring.cuh"
#include "workspace.cuh"

namespace dfl {

// Candidate buffer of one consumer warp: keys pushed during the candidate
// rounds, merged into the running list whenever more than CAND_FLUSH are
// waiting (at most 32 lanes x 8 elements arrive between two checks) and at
// the end of every chunk.  The count of waiting keys lives in a register of
// the warp (the same value in every lane), not here.
constexpr unsigned CAND_FLUSH = 64;
constexpr unsigned CAND_CAP = CAND_FLUSH + 32 * 8;
struct CandBuf {
    uint64_t key[CAND_CAP];
    uint64_t out[K];  // the merged list, placed by rank
};

// Merge the n buffered candidates into the running list (lanes 0..15 hold
// it, descending; 0 = empty), up to 32 at a time, by rank: every key of the
// union (keys are distinct) lands at its rank in it, so a batch costs one
// broadcast read, two compares and a ballot per buffered key, and no sort.
// Then the threshold rises to the list's 16th key once the list is full; a
// raised value also raises the row's shared bound (thr: ord32 of a value at
// least 16 of the row's elements reach; pub: what this warp last put there).
// Warp-uniform; n is zero on return.
__device__ __forceinline__ void flush_candidates(CandBuf& cb, unsigned& n, uint64_t& run,
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
            const unsigned above = __ballot_sync(FULL, lane < K && run > cj);
            if ((unsigned)lane == j) rank_list = __popc(above);
            rank_new += cj > c;
            above_run += cj > run;
        }
        if (lane < K) cb.out[lane] = 0ull;
        __syncwarp();
        const unsigned pc = rank_list + rank_new;
        if ((unsigned)lane < m && pc < K) cb.out[pc] = c;
        const unsigned pr = (unsigned)lane + above_run;
        if (lane < K && run != 0ull && pr < K) cb.out[pr] = run;
        __syncwarp();
        run = lane < K ? cb.out[lane] : 0ull;
        __syncwarp();  // out is read before the next batch writes it
    }
    n = 0u;
    const uint64_t k16 = shfl64(run, K - 1);
    if (k16 > tkey) {
        tkey = k16;
        tv = key_value(k16);
    }
    const uint32_t o16 = (uint32_t)(k16 >> 32);
    if (o16 > pub) {  // the list is full: its 16th value bounds the row
        pub = o16;
        if (lane == 0) atomicMax(thr, o16);
    }
}

// One chunk, one warp: the chunk maximum M, the sum of exp2((x - M) c) and
// the running top-16 `run` of the row segment (lanes 0..15, descending by
// (value, -index); 0 = empty) updated with the chunk's elements.
//   Pass 1: the packed maximum of every vector of the lane, kept in
//   registers, and the lane maxima.  While the list is not full, T = the 16th
//   largest lane maximum bounds the chunk's own top 16 (at least 16 elements
//   are >= T); once it is full its 16th key is the bound.  The row's shared
//   bound (a value at least 16 of the row's elements reach, raised by every
//   warp whose list fills; `shared` is its value as read one chunk earlier,
//   so the load's latency hides behind a whole chunk) replaces either when
//   higher: no element below it
//   can be in the row's top 16, so the merged result is the same exact set,
//   while a segment's own list may hold fewer than 16 keys.
//   Candidates: only the vectors whose maximum reaches the bound's value are
//   looked at element by element (one per lane per round); keys beating the
//   bound are pushed and merged whenever more than CAND_FLUSH wait, and the
//   bound rises to the list's 16th key at every merge.
//   Pass 2: the exponentials (chunk_expsum_at_mc: the sum against fl(M c),
//   rescaled to the row maximum by the merge).
template <bool BF16, class View>
__device__ __forceinline__ void topk_chunk(const View& v, float c2, CandBuf& cb, float& M_out,
                                           double& S_out, uint64_t& run, unsigned* thr,
                                           uint32_t& pub, uint32_t shared) {
    using C = ChunkT<BF16>;
    const int lane = threadIdx.x & 31, nv = v.nvec();
    uint32_t vm[NVL];
    const float m = chunk_pass1<BF16>(v, vm);
    const float M = warp_max(m);
    float tv = -INFINITY;
    uint64_t tkey = shfl64(run, K - 1);  // the full list's 16th key, or 0
    if (tkey != 0ull) {
        tv = key_value(tkey);
    } else {
        const uint32_t t16 =
            __shfl_sync(FULL, warp_sort_desc(m == -INFINITY ? 0u : ord32(m)), K - 1);
        if (t16 != 0u) {  // else fewer than 16 lanes hold elements: every element qualifies
            tv = unord32(t16);
            tkey = ((uint64_t)t16 << 32) - 1ull;  // below every key of value tv
            // 16 lane maxima of this chunk reach t16: a bound for the whole
            // row, shared at once with the warps on its other chunks
            if (t16 > pub) {
                pub = t16;
                if (lane == 0) atomicMax(thr, t16);
            }
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
    if (__any_sync(FULL, hits != 0u)) {
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
            // the list's 16th key are pushed too: the merge ranks them out.
            const unsigned cnt = __popc(em);
            // this round's keys appended in lane order: the exclusive prefix
            // of the per-lane counts (at most 8: four bits) from four ballots
            const unsigned below = (1u << lane) - 1u;
            unsigned excl = 0u, total = 0u;
#pragma unroll
            for (int bit = 0; bit < 4; ++bit) {
                const unsigned b = __ballot_sync(FULL, (cnt >> bit) & 1u);
                excl += (unsigned)__popc(b & below) << bit;
                total += (unsigned)__popc(b) << bit;
            }
            unsigned pos = nbuf + excl;
            while (em) {
                const int e = __ffs(em) - 1;
                em &= em - 1u;
                cb.key[pos++] = make_key(C::elem_at(w, e), (uint32_t)v.index(q, e));
            }
            nbuf += total;
            if (nbuf > CAND_FLUSH) flush_candidates(cb, nbuf, run, tkey, tv, thr, pub);
        }
        if (nbuf > 0u) flush_candidates(cb, nbuf, run, tkey, tv, thr, pub);
    }
    M_out = M;
    S_out = chunk_expsum_at_mc<BF16>(v, M, c2);  // against fl(M c2); the merge rescales
}

// The row's final merge by one warp, after its last chunk was published:
// the segment lists (bitonic merges in chunk order), the maximum, and the
// fp64 sum of the chunk sums rescaled to it (lane c takes chunks c, c + 32,
// ...; then a fixed butterfly).  Two dependent load rounds for rows of up to
// 64 chunks: every chunk's (max, sum, first key), then the lists, up to
// eight at once; longer rows add a round per further 32 chunks.
__device__ __forceinline__ void topk_row_merge(const TopkPart* P, int S, int64_t row, float inv_t,
                                               float c2, int32_t* __restrict__ idx,
                                               float* __restrict__ prob, float* __restrict__ logp,
                                               float* __restrict__ logz,
                                               float* __restrict__ row_max,
                                               float* __restrict__ row_lse) {
    const int lane = threadIdx.x & 31;
    auto ldkey = [](const uint64_t* p) { return (uint64_t)__ldcg((const unsigned long long*)p); };
    float m0 = -INFINITY, m1 = -INFINITY;  // chunks lane and lane + 32
    double s0 = 0.0, s1 = 0.0;
    uint64_t q0 = 0ull, q1 = 0ull;  // first key of the chunk's list (0: no list)
    if (lane < S) {
        m0 = __ldcg(&P[lane].m);
        s0 = __ldcg(&P[lane].s);
        q0 = ldkey(&P[lane].key[0]);
    }
    if (lane + 32 < S) {
        m1 = __ldcg(&P[lane + 32].m);
        s1 = __ldcg(&P[lane + 32].s);
        q1 = ldkey(&P[lane + 32].key[0]);
    }
    float M = fmaxf(m0, m1);
    for (int c = lane + 64; c < S; c += 32) M = fmaxf(M, __ldcg(&P[c].m));
    M = warp_max(M);
    // a chunk's sum is against fl(mc c2); M c2 is exact in fp64
    const double Mc = (double)M * (double)c2;
    auto rescaled = [&](float mc, double sc) {
        return mc != -INFINITY ? sc * exp2((double)(mc * c2) - Mc) : 0.0;
    };
    double ssum = rescaled(m0, s0);
    ssum += rescaled(m1, s1);
    uint64_t acc = 0ull;
    bool first = true;
    // the lists of the chunks cbase + (set bits of hm), loaded up to eight at
    // once, merged in chunk order
    auto merge_lists = [&](uint64_t hm, int cbase) {
        constexpr int PF = 8;
        while (hm) {
            uint64_t kv[PF];
            int nl = 0;
#pragma unroll
            for (int j = 0; j < PF; ++j) {
                kv[j] = 0ull;
                if (hm) {
                    const int cc = cbase + __ffsll((long long)hm) - 1;
                    hm &= hm - 1ull;
                    kv[j] = ldkey(&P[cc].key[lane < K ? lane : 31 - lane]);
                    ++nl;
                }
            }
#pragma unroll
            for (int j = 0; j < PF; ++j)
                if (j < nl) {
                    if (first) {
                        acc = (lane < K) ? kv[j] : 0ull;
                        first = false;
                    } else {
                        acc = warp_merge_desc(lane < K ? acc : kv[j]);
                    }
                }
        }
    };
    merge_lists(((uint64_t)__ballot_sync(FULL, q1 != 0ull) << 32) | __ballot_sync(FULL, q0 != 0ull),
                0);
    for (int c0 = 64; c0 < S; c0 += 32) {
        const int c = c0 + lane;
        float mc = -INFINITY;
        double sc = 0.0;
        uint64_t k0 = 0ull;
        if (c < S) {
            mc = __ldcg(&P[c].m);
            sc = __ldcg(&P[c].s);
            k0 = ldkey(&P[c].key[0]);
        }
        ssum += rescaled(mc, sc);
        merge_lists(__ballot_sync(FULL, k0 != 0ull), c0);
    }
    ssum = warp_sum(ssum);
    const double lns = log(ssum);
    if (lane < K) {
        const double x = (double)key_value(acc);
        const int64_t o = row * K + lane;
        idx[o] = (int32_t)key_index(acc);
        prob[o] = (float)(exp2((x - (double)M) * (double)c2) / ssum);
        logp[o] = (float)((x - (double)M) * (double)inv_t - lns);
        if (lane == 0) {
            logz[row] = (float)((double)M * (double)inv_t + lns);
            if (row_max) row_max[row] = M;
            if (row_lse) row_lse[row] = (float)lns;
        }
    }
}

// Units (row, chunk): one CTA per SM over a contiguous range, each warp a
// contiguous part of it streamed through its own two ring slots.  Every
// chunk leaves its softmax partial in the workspace; a warp's consecutive
// chunks of one row (a segment) share one running top-16, left with the
// segment's last chunk, and are published together with one acquire-release
// add on the row's counter.  The warp whose add completes the row merges it.
// No warp waits for another.
template <bool BF16, bool TMA>
__global__ void __launch_bounds__(RING_THREADS, 1) topk_softmax_kernel(
    const void* __restrict__ logits, int64_t V, int64_t row_stride, int S, int64_t units,
    float inv_t, float c2, int32_t* __restrict__ idx, float* __restrict__ prob,
    float* __restrict__ logp, float* __restrict__ logz, float* __restrict__ row_max,
    float* __restrict__ row_lse, TopkPart* __restrict__ part, unsigned* __restrict__ counters,
    unsigned* __restrict__ thr) {
    constexpr int ES = BF16 ? 2 : 4;
    constexpr int LEN = chunk_len(ES);
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ __align__(8) uint64_t bars[2 * NCW];
    __shared__ CandBuf cbuf[NCW];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    CandBuf& cb = cbuf[warp];
    int64_t lo, hi;
    warp_range(units, lo, hi);
    const int n = (int)(hi - lo);
    UnitCursor uc, ic;  // the unit being reduced, the next unit to bring in
    uc.init(lo, S, 1);
    ic = uc;
    auto src = [&](const UnitCursor& cu, const char*& p, uint32_t& bytes) {
        const int64_t v0 = (int64_t)cu.c * LEN;
        p = (const char*)logits + (cu.g * row_stride + v0) * ES;
        bytes = (uint32_t)(min((int64_t)LEN, V - v0) * ES);
    };
    WarpRing r{nullptr, 0u};
    if (TMA) r = warp_ring_start(ring, bars, n, ic, ChunkT<BF16>::NEG_INF_WORD, src);
    __syncwarp();
    uint64_t run = 0ull;  // the segment's running top-16
    unsigned seg = 0;     // chunks in the segment so far
    uint32_t pub = 0u;    // the row bound this segment last raised thr to
    // the row's shared bound, read one unit ahead: it only ever rises while
    // the row is open (and its last unit is still to come), so an older value
    // is a valid, slightly looser bound
    uint32_t thr_now = n > 0 ? *(volatile unsigned*)&thr[uc.g] : 0u;
    for (int k = 0; k < n; ++k, uc.next()) {
        const int64_t row = uc.g, v0 = (int64_t)uc.c * LEN;
        const uint32_t thr_ahead =
            k + 1 < n ? *(volatile unsigned*)&thr[uc.last_of_row() ? row + 1 : row] : 0u;
        const int len = (int)min((int64_t)LEN, V - v0);
        float M;
        double Ssum;
        if (TMA) {
            if (!r.wait(k)) {
                warp_ring_abort(r, k, n);
                return;
            }
            topk_chunk<BF16>(SmemView<BF16>{r.slot(k), v0, len}, c2, cb, M, Ssum, run, &thr[row],
                             pub, thr_now);
            warp_ring_next(r, k, n, ic, ChunkT<BF16>::NEG_INF_WORD, src);
        } else {
            topk_chunk<BF16>(
                GlobalView<BF16>{(const uint8_t*)logits + row * row_stride * ES, v0, len}, c2, cb,
                M, Ssum, run, &thr[row], pub, thr_now);
        }
        ++seg;
        const bool seg_end = (k + 1 == n) || uc.last_of_row();
        TopkPart* P = part + row * S + uc.c;
        if (seg_end) {
            if (lane < K) P->key[lane] = run;
        } else if (lane == 0) {
            P->key[0] = 0ull;  // no list here
        }
        if (lane == 0) {
            P->m = M;
            P->s = Ssum;
        }
        if (seg_end) {
            __syncwarp();
            bool last = false;
            if (lane == 0) last = publish(&counters[row], seg, (unsigned)S);
            if (__shfl_sync(FULL, last, 0)) {
                __syncwarp();  // lane 0's acquire covers the whole warp's reads
                topk_row_merge(part + row * S, S, row, inv_t, c2, idx, prob, logp, logz, row_max,
                               row_lse);
                if (lane == 0) {  // the row is done: leave its words zero
                    counters[row] = 0u;
                    thr[row] = 0u;
                }
            }
            run = 0ull;
            seg = 0;
            pub = 0u;
        }
        thr_now = thr_ahead;
    }
}

}  // namespace dfl

using namespace dfl;
using namespace dfl_host;

unsigned dfl_errors_topk(int clear) {
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_dev_err, sizeof v) != cudaSuccess) return 0xFFFFFFFFu;
    if (clear && v) {
        unsigned z = 0;
        cudaMemcpyToSymbol(g_dev_err, &z, sizeof z);
    }
    return v;
}

// The call behind every top-16 entry.  clear_first: zero the counters and
// bounds with one memset after every check has passed (a scratch area whose
// state a previous call may have left behind); otherwise they are zero on
// entry (the workspace contract) unless they do not fit the control area.
static int topk_softmax_impl(const void* logits, int dtype, int64_t rows, int64_t V,
                             int64_t row_stride, float inv_temperature, int32_t* idx, float* prob,
                             float* logp, float* logz, float* row_max, float* row_lse, void* ws,
                             size_t ws_bytes, bool clear_first, dflash2_stream_t stream) {
    if (!dtype_ok(dtype)) return DFLASH2_EDTYPE;
    if (rows < 0 || V < K || V > INT32_MAX || row_stride < V) return DFLASH2_ESHAPE;
    if (!finite_pos(inv_temperature)) return DFLASH2_EINVAL;
    if (rows == 0) return DFLASH2_OK;
    if (!logits || !idx || !prob || !logp || !logz) return DFLASH2_EINVAL;
    const int es = elem_size(dtype);
    if (!aligned(logits, es) || !aligned(idx, 4) || !aligned(prob, 4) || !aligned(logp, 4) ||
        !aligned(logz, 4) || (row_max && !aligned(row_max, 4)) || (row_lse && !aligned(row_lse, 4)))
        return DFLASH2_EALIGN;
    const int64_t S = row_chunks(V, es);
    const int64_t units = rows * S;
    if (units > (int64_t)INT32_MAX) return DFLASH2_ESHAPE;
    const Layout L = topk_layout(rows, V, es);
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return DFLASH2_EWORKSPACE;

    cudaStream_t s = (cudaStream_t)stream;
    unsigned* counters = (unsigned*)((char*)ws + L.counters_off);
    TopkPart* part = (TopkPart*)((char*)ws + L.part_off);
    unsigned* thr = counters + rows;  // the rows' shared top-16 bounds
    if ((clear_first || !L.self_clean) &&
        cudaMemsetAsync(counters, 0, (size_t)rows * 8, s) != cudaSuccess)
        return DFLASH2_ECUDA;

    // TMA bulk copies need 16-byte aligned chunk starts and 16-byte multiples
    const bool tma = aligned(logits, 16) && (row_stride * es) % 16 == 0 && (V * es) % 16 == 0;
    const float c2 = (float)((double)inv_temperature * 1.4426950408889634);
#define DFL_TOPK(BF, TM)                                                                          \
    do {                                                                                          \
        auto kern = topk_softmax_kernel<BF, TM>;                                                  \
        const size_t dyn = TM ? (size_t)RING_BYTES : 0;                                           \
        if (ring_prepare(kern, dyn) != DFLASH2_OK) return DFLASH2_ECUDA;                          \
        kern<<<ring_grid(units), RING_THREADS, dyn, s>>>(logits, V, row_stride, (int)S, units,    \
                                                         inv_temperature, c2, idx, prob, logp,    \
                                                         logz, row_max, row_lse, part, counters, thr); \
    } while (0)
    if (dtype == DFLASH2_BF16) {
        if (tma) DFL_TOPK(true, true);
        else DFL_TOPK(true, false);
    } else {
        if (tma) DFL_TOPK(false, true);
        else DFL_TOPK(false, false);
    }
#undef DFL_TOPK
    return launch_status();
}

extern "C" int dflash2_topk_softmax_ex(const void* logits, int dtype, int64_t rows, int64_t V,
                                       int64_t row_stride, float inv_temperature, int32_t* idx,
                                       float* prob, float* logp, float* logz, float* row_max,
                                       float* row_lse, void* ws, size_t ws_bytes,
                                       dflash2_stream_t stream) {
    return topk_softmax_impl(logits, dtype, rows, V, row_stride, inv_temperature, idx, prob, logp,
                             logz, row_max, row_lse, ws, ws_bytes, false, stream);
}

extern "C" int dflash2_topk_softmax(const void* logits, int dtype, int64_t rows, int64_t V,
                                    int64_t row_stride, float inv_temperature, int32_t* idx,
                                    float* prob, float* logp, float* logz, void* ws,
                                    size_t ws_bytes, dflash2_stream_t stream) {
    return topk_softmax_impl(logits, dtype, rows, V, row_stride, inv_temperature, idx, prob, logp,
                             logz, nullptr, nullptr, ws, ws_bytes, false, stream);
}

// ---------------------------------------------------------------------------
// Allocation-free variant.  Some callers cannot hand us device memory: an
// inference engine that reserved nearly all of the GPU for its own memory
// pools (KV cache, activations) at start-up and does not let a plugin call
// cudaMalloc, or a latency-critical path where cudaMalloc could synchronise
// the device.  For them the scratch (arrival counters and per-chunk partials)
// lives in one fixed array of device memory inside this library, loaded with
// the library on every GPU that uses it and kept until the process exits.
namespace {

constexpr size_t NOALLOC_SCRATCH_BYTES = DFLASH2_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

// Device address of the array in each CUDA context.  The host-side name of
// the array is only a stand-in; the address a kernel can use is looked up
// (cudaGetSymbolAddress) with the context current, once per context.  The
// cache is keyed by the context's unique id (cuCtxGetId), which no later
// context reuses: after cudaDeviceReset, or in another context on the same
// device, the library's module is loaded anew and the address looked up
// again.
constexpr int NOALLOC_MAX_CTX = 64;
struct NoallocEntry {
    unsigned long long ctx_id;
    void* addr;
};
NoallocEntry g_noalloc_cache[NOALLOC_MAX_CTX];
int g_noalloc_used;
std::mutex g_noalloc_mu;

// The two driver calls, resolved through the runtime (the library does not
// link the driver library itself).
typedef CUresult (*PfnCtxGetCurrent)(CUcontext*);
typedef CUresult (*PfnCtxGetId)(CUcontext, unsigned long long*);

bool current_context_id(unsigned long long& id) {
    static PfnCtxGetCurrent get_current = nullptr;
    static PfnCtxGetId get_id = nullptr;
    static std::once_flag resolved;
    std::call_once(resolved, [] {
        void* a = nullptr;
        void* b = nullptr;
        cudaDriverEntryPointQueryResult qa, qb;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
            qa == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
            qb == cudaDriverEntryPointSuccess) {
            get_current = (PfnCtxGetCurrent)a;
            get_id = (PfnCtxGetId)b;
        }
    });
    if (!get_current || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, &id) == CUDA_SUCCESS;
}

void* noalloc_scratch_in_current_context() {
    unsigned long long id = 0;
    if (!current_context_id(id)) {
        // no context current yet: the runtime's symbol lookup creates the
        // device's primary context and makes it current
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        if (!current_context_id(id)) return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    for (int i = 0; i < g_noalloc_used; ++i)
        if (g_noalloc_cache[i].ctx_id == id) return g_noalloc_cache[i].addr;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    const int slot = g_noalloc_used < NOALLOC_MAX_CTX ? g_noalloc_used++ : (int)(id % NOALLOC_MAX_CTX);
    g_noalloc_cache[slot] = NoallocEntry{id, p};
    return p;
}

}  // namespace

extern "C" int dflash2_topk_softmax_noalloc(const void* logits, int dtype, int64_t rows, int64_t V,
                                            int64_t row_stride, float inv_temperature, int32_t* idx,
                                            float* prob, float* logp, float* logz,
                                            dflash2_stream_t stream) {
    if (!dtype_ok(dtype)) return DFLASH2_EDTYPE;
    if (rows < 0 || V < K || V > INT32_MAX || row_stride < V) return DFLASH2_ESHAPE;
    if (rows > 0 && topk_layout(rows, V, elem_size(dtype)).total > NOALLOC_SCRATCH_BYTES)
        return DFLASH2_EWORKSPACE;  // more rows than the built-in scratch holds
    if (rows == 0) return DFLASH2_OK;
    void* scratch = noalloc_scratch_in_current_context();
    if (!scratch) return DFLASH2_ECUDA;
    // every other argument is checked before anything is enqueued; then the
    // array's counters are cleared (whatever an earlier, failed call left)
    return topk_softmax_impl(logits, dtype, rows, V, row_stride, inv_temperature, idx, prob, logp,
                             logz, nullptr, nullptr, scratch, NOALLOC_SCRATCH_BYTES, true, stream);
}
