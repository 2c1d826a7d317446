// topk_softmax.cu -- softmax over the vocabulary and the 16 best candidates of
// every drafted position, in one pass over the logits.
//
// Source: "DFlash 2 — 3× plus de tokens sur Qwen3.8-27B, même sortie"
// (tamsi.dev), section "L’idée, sans le papier": the right token lies in the
// drafter's top 16 far more often than at top 1, and the selector picks among
// those 16 per position; "DFlash 2" (myaiexp.com), section "主な機能": the
// path selector keeps the top-16 candidates of each position.
//
// Work unit: (row, 16384-element chunk).  Persistent CTAs each stream a
// contiguous range of units through a two-slot shared-memory ring filled by
// TMA bulk copies (rows whose start is 16-byte aligned; others are read
// element by element).  Softmax: per chunk, the block max, then the sum of
// exp2((x - M) c) against it, both in a fixed order, so a chunk's partial
// does not depend on the batch or the grid.  Top-16: the block keeps a
// running top-16 of the row segment it streams (its consecutive chunks of one
// row).  The first chunk of a segment takes the exact bounded path (the 16th
// largest per-thread maximum bounds the answer, at most 16 threads contribute
// candidates, one warp sorts them); later chunks only look at elements whose
// key beats the running 16th key, about 16/c of them in the c-th chunk.  The
// segment's list is published with one acquire-release add; the publisher
// that completes a row (no CTA waits) merges the chunk softmax partials in
// chunk order and the segment lists, and writes idx / prob / logp / logz.
// Keys compare (value, -index) exactly, so the top-16 set does not depend on
// how the row was split.
#include "common.cuh"
#include "stream.cuh"
#include "workspace.cuh"

namespace dfl {

struct __align__(16) TopkSmem {
    uint64_t run[K];          // running top-16 of the row segment (descending; 0 = empty)
    uint32_t top[NT / 32][K];
    uint64_t cand[K * EPT];   // candidate keys (capacity 1024)
    uint32_t tie[NT];
    float wmax[NT / 32];
    float wmax2[NT / 32];
    float wsum[NT / 32];
    unsigned ncand, ntie;
    uint32_t thr, vk;
};
constexpr unsigned CAND_CAP = K * EPT;

// Warp 0: merge sm.cand[0..n) into the running list (16 candidates a round).
__device__ __forceinline__ void merge_candidates(TopkSmem& sm, unsigned n) {
    const int lane = threadIdx.x & 31;
    uint64_t acc = (lane < K) ? sm.run[lane] : 0ull;
    for (unsigned base = 0; base < n; base += K) {
        uint64_t v = acc;
        if (lane >= K) v = (base + lane - K < n) ? sm.cand[base + lane - K] : 0ull;
        acc = warp_sort_desc(v);
    }
    if (lane < K) sm.run[lane] = acc;
}

// The chunk's exact top-16 without sorting the chunk: T = the 16th largest
// per-thread maximum bounds it; only threads whose maximum is above T, or
// equal to T with a first index among the lowest (16 - #above) of those, can
// hold a top-16 element (at most 16 threads x 64 candidates); they are merged
// into the running list.  m = this thread's maximum.
template <bool BF16, class C>
__device__ __forceinline__ void chunk_top16_exact(const C& ch, float m, TopkSmem& sm) {
    using R = Row<BF16>;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    __syncthreads();  // everyone has read the count that sent the block here
    const uint32_t my_ord = (m == -INFINITY) ? 0u : ord32(m);
    const uint32_t srt = warp_sort_desc(my_ord);
    if (lane < K) sm.top[warp][lane] = srt;
    if (t == 0) {
        sm.ncand = 0;
        sm.ntie = 0;
    }
    __syncthreads();
    if (warp == 0) {
        uint32_t acc = (lane < K) ? sm.top[0][lane] : 0u;
        for (int w = 1; w < NT / 32; ++w) acc = warp_merge_desc(lane < K ? acc : sm.top[w][31 - lane]);
        if (lane == K - 1) sm.thr = acc;  // 0: fewer than 16 threads hold elements
    }
    __syncthreads();
    const uint32_t thr = sm.thr;
    const bool above = my_ord > thr;
    const bool tie = thr != 0u && my_ord == thr;
    const int n_above = __syncthreads_count(above);
    uint32_t my_first = 0xFFFFFFFFu;
    if (tie) {
        my_first = view_first<BF16>(ch, m);
        sm.tie[atomicAdd(&sm.ntie, 1u)] = my_first;
    }
    __syncthreads();
    if (tie) {
        const unsigned n = sm.ntie;
        unsigned rank = 0;
        for (unsigned j = 0; j < n; ++j) rank += sm.tie[j] < my_first;
        if (rank == (unsigned)(K - n_above - 1)) sm.vk = my_first;
    }
    __syncthreads();
    const float tv = (thr == 0u) ? -INFINITY : unord32(thr);
    const uint32_t vk = (thr == 0u) ? 0u : sm.vk;
    if (above || (tie && my_first <= vk)) {
#pragma unroll
        for (int i = 0; i < R::NV; ++i) {
            const uint4 v4 = ch.vec(i);
#pragma unroll
            for (int e = 0; e < R::VW; ++e) {
                const float x = R::elem(v4, e);
                const uint32_t v = (uint32_t)ch.index_of(i, e);
                if (x > tv || (thr != 0u && x == tv && v <= vk))
                    sm.cand[atomicAdd(&sm.ncand, 1u)] = make_key(x, v);
            }
        }
    }
    __syncthreads();
    if (warp == 0) merge_candidates(sm, sm.ncand);
    __syncthreads();
}

// One unit: the chunk's softmax partial (block max, then the sum of
// exp2(x c - M c) against it, in a fixed order) and the running top-16.
//  - Running list full: elements whose key beats its 16th key are pushed as
//    candidates during the max pass (about 16/c of them in the c-th chunk of
//    a segment); warp 0 merges them while the other warps sum exps.
//  - Running list empty (first chunk of a segment): T' = the smallest of the
//    warps' second-largest thread maxima has at least 16 elements at or above
//    it (two per warp), so the elements >= T' hold the chunk's top-16; they are
//    pushed and merged.
//  - More candidates than the buffer holds (adversarial orders, mass ties):
//    the chunk takes the exact bounded path.
template <bool BF16, class C>
__device__ __forceinline__ void topk_unit(const C& ch, float c2, TopkSmem& sm, float& chunk_m,
                                          float& chunk_s) {
    using R = Row<BF16>;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const uint64_t r16 = sm.run[K - 1];
    const float rv = r16 ? key_value(r16) : INFINITY;
    // pass 1: thread max, and candidates against the running list
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < R::NV; ++i) {
        const uint4 v4 = ch.vec(i);
        const float vm = vec_max<BF16>(v4);
        m = fmaxf(m, vm);
        if (vm >= rv) {
#pragma unroll
            for (int e = 0; e < R::VW; ++e) {
                const float x = R::elem(v4, e);
                if (x >= rv) {
                    const uint64_t key = make_key(x, (uint32_t)ch.index_of(i, e));
                    if (key > r16) {
                        const unsigned slot = atomicAdd(&sm.ncand, 1u);
                        if (slot < CAND_CAP) sm.cand[slot] = key;
                    }
                }
            }
        }
    }
    // warp max and (for seeding) the warp's second-largest thread maximum
    float wm = m;
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) wm = fmaxf(wm, __shfl_xor_sync(FULL, wm, j));
    const unsigned at_max = __ballot_sync(FULL, m == wm);
    float m2 = (lane == __ffs(at_max) - 1) ? -INFINITY : m;
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) m2 = fmaxf(m2, __shfl_xor_sync(FULL, m2, j));
    if (lane == 0) {
        sm.wmax[warp] = wm;
        sm.wmax2[warp] = m2;
    }
    __syncthreads();  // A
    float M = sm.wmax[0];
#pragma unroll
    for (int w = 1; w < NT / 32; ++w) M = fmaxf(M, sm.wmax[w]);
    bool exact = false;
    if (r16 == 0ull) {  // seed the segment's list from this chunk
        float Tp = sm.wmax2[0];
#pragma unroll
        for (int w = 1; w < NT / 32; ++w) Tp = fminf(Tp, sm.wmax2[w]);
        if (m >= Tp && m != -INFINITY) {
#pragma unroll
            for (int i = 0; i < R::NV; ++i) {
                const uint4 v4 = ch.vec(i);
#pragma unroll
                for (int e = 0; e < R::VW; ++e) {
                    const float x = R::elem(v4, e);
                    if (x >= Tp && x != -INFINITY) {
                        const unsigned slot = atomicAdd(&sm.ncand, 1u);
                        if (slot < CAND_CAP) sm.cand[slot] = make_key(x, (uint32_t)ch.index_of(i, e));
                    }
                }
            }
        }
        __syncthreads();  // B (seeding chunks only)
    }
    const unsigned n = sm.ncand;
    if (n > CAND_CAP) {
        exact = true;  // block-uniform
    } else if (n > 0 && warp == 0) {
        merge_candidates(sm, n);  // overlaps the other warps' exp pass
    }
    if (exact) chunk_top16_exact<BF16>(ch, m, sm);

    // pass 2: sum of exp2(x c - M c) (fixed order), each exponent one FMA
    // against mc = fl(M c); the product's rounding error M c - mc (exact in
    // fp32) is taken out of the sum once per chunk below.
    float s = 0.0f;
    const float mc = M * c2;
    if (M != -INFINITY) {
#pragma unroll
        for (int i = 0; i < R::NV; ++i) {
            const uint4 v4 = ch.vec(i);
            float tt[R::VW];
#pragma unroll
            for (int e = 0; e < R::VW; ++e) tt[e] = ex2(fmaf(R::elem(v4, e), c2, -mc));
#pragma unroll
            for (int w = R::VW / 2; w > 0; w >>= 1)
#pragma unroll
                for (int e = 0; e < w; ++e) tt[e] += tt[e + w];
            s += tt[0];
        }
    }
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) s += __shfl_xor_sync(FULL, s, j);
    if (lane == 0) sm.wsum[warp] = s;
    __syncthreads();  // D: sums ready, candidates merged
    float S = 0.0f;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) S += sm.wsum[w];
    chunk_m = M;
    chunk_s = (M != -INFINITY) ? S * ex2(-fmaf(M, c2, -mc)) : S;
    if (t == 0) sm.ncand = 0;  // read by everyone before D; next pushes come after
}

// The row's final merge (warp 0 of the last unit of the row).
__device__ __forceinline__ void topk_row_merge(const TopkPartial* P, int S, int64_t row, float inv_t,
                                               float c2, int32_t* __restrict__ idx,
                                               float* __restrict__ prob, float* __restrict__ logp,
                                               float* __restrict__ logz) {
    const int lane = threadIdx.x & 31;
    auto ldkey = [](const uint64_t* p) { return (uint64_t)__ldcg((const unsigned long long*)p); };
    uint64_t acc = (lane < K) ? ldkey(&P[0].key[lane]) : 0ull;
    for (int c = 1; c < S; ++c) acc = warp_merge_desc(lane < K ? acc : ldkey(&P[c].key[31 - lane]));
    float M = -INFINITY;
    for (int c = lane; c < S; c += 32) M = fmaxf(M, __ldcg(&P[c].m));
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, j));
    double ssum = 0.0;
    if (lane == 0)  // sum in chunk order, fp64
        for (int c = 0; c < S; ++c) {
            const float mc = __ldcg(&P[c].m), sc = __ldcg(&P[c].s);
            if (mc != -INFINITY) ssum += (double)sc * exp2(((double)mc - (double)M) * (double)c2);
        }
    ssum = __shfl_sync(FULL, ssum, 0);
    const double lns = log(ssum);
    if (lane < K) {
        const double x = (double)key_value(acc);
        const int64_t o = row * K + lane;
        idx[o] = (int32_t)key_index(acc);
        prob[o] = (float)(exp2((x - (double)M) * (double)c2) / ssum);
        logp[o] = (float)((x - (double)M) * (double)inv_t - lns);
        if (lane == 0) logz[row] = (float)((double)M * (double)inv_t + lns);
    }
}

template <bool BF16, bool TMA>
__global__ void __launch_bounds__(NT, 3) topk_softmax_kernel(
    const void* __restrict__ logits, int64_t V, int64_t row_stride, int S, int64_t units,
    float inv_t, float c2, int32_t* __restrict__ idx, float* __restrict__ prob,
    float* __restrict__ logp, float* __restrict__ logz, TopkPartial* __restrict__ part,
    unsigned* __restrict__ counters) {
    constexpr int ES = BF16 ? 2 : 4;
    constexpr int SLOT = CHUNK * ES;
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ TopkSmem sm;
    __shared__ __align__(8) uint64_t s_bar[2];
    const int t = threadIdx.x, warp = t >> 5;
    const uint32_t bar0 = smem_u32(&s_bar[0]);

    auto unit_geom = [&](int64_t u, int64_t& row, int64_t& v0, int64_t& vend) {
        row = u / S;
        v0 = (u - row * S) * (int64_t)CHUNK;
        vend = min(V, v0 + (int64_t)CHUNK);
    };
    auto issue = [&](int64_t u, int slot) {
        int64_t row, v0, vend;
        unit_geom(u, row, v0, vend);
        const char* src = (const char*)logits + (row * row_stride + v0) * ES;
        bulk_g2s(smem_u32(ring + slot * SLOT), src, (uint32_t)((vend - v0) * ES), bar0 + 8 * slot);
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
    if (t < K) sm.run[t] = 0ull;
    if (t == 0) sm.ncand = 0;
    int k = 0;
    for (int64_t u = lo; u < hi; ++u, ++k) {
        int64_t row, v0, vend;
        unit_geom(u, row, v0, vend);
        float cm, cs;
        if (TMA) {
            if (t == 0 && u + 1 < hi) issue(u + 1, (k + 1) & 1);
            if (!__syncthreads_and(mbar_wait(bar0 + 8 * (k & 1), (k >> 1) & 1))) {
                if (t == 0) {
                    atomicOr(&g_dev_err, ERR_STREAM);
                    if (u + 1 < hi) mbar_wait(bar0 + 8 * ((k + 1) & 1), ((k + 1) >> 1) & 1);
                }
                return;
            }
            topk_unit<BF16>(SmemChunk<BF16>{ring + (k & 1) * SLOT, v0, vend}, c2, sm, cm, cs);
        } else {
            RegChunk<BF16> ch;
            ch.load((const char*)logits + row * row_stride * ES, v0, vend);
            topk_unit<BF16>(ch, c2, sm, cm, cs);
        }
        ++pending;
        const bool seg_end = (u + 1 == hi) || ((u + 1) / S != row);
        if (t == 0) {  // thread 0 alone stores the partial (published by its release add);
                       // only the last unit of a segment carries the segment's top-16
            uint4* dst = (uint4*)&part[u];
            dst[0] = make_uint4(__float_as_uint(cm), __float_as_uint(cs), 0u, 0u);
            const uint4* kv = (const uint4*)sm.run;
#pragma unroll
            for (int j = 0; j < K / 2; ++j) dst[1 + j] = seg_end ? kv[j] : make_uint4(0, 0, 0, 0);
        }
        if (seg_end) {  // this CTA is done with the row: publish
            if (t == 0) s_last = publish(&counters[row], pending, (unsigned)S);
            __syncthreads();
            if (s_last && warp == 0)
                topk_row_merge(part + row * S, S, row, inv_t, c2, idx, prob, logp, logz);
            pending = 0;
            __syncthreads();
            if (t < K) sm.run[t] = 0ull;  // the next segment starts empty
        }
        __syncthreads();  // ring slot k & 1 is free for the prefetch of iteration k + 1
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

extern "C" int dflash2_topk_softmax(const void* logits, int dtype, int64_t rows, int64_t V,
                                    int64_t row_stride, float inv_temperature, int32_t* idx,
                                    float* prob, float* logp, float* logz, void* ws,
                                    size_t ws_bytes, dflash2_stream_t stream) {
    if (!dtype_ok(dtype)) return DFLASH2_EDTYPE;
    if (rows < 0 || V < K || V > INT32_MAX || row_stride < V) return DFLASH2_ESHAPE;
    if (!finite_pos(inv_temperature)) return DFLASH2_EINVAL;
    if (rows == 0) return DFLASH2_OK;
    if (!logits || !idx || !prob || !logp || !logz) return DFLASH2_EINVAL;
    const int es = elem_size(dtype);
    if (!aligned(logits, es) || !aligned(idx, 4) || !aligned(prob, 4) || !aligned(logp, 4) ||
        !aligned(logz, 4))
        return DFLASH2_EALIGN;
    const int64_t S = n_chunks(V);
    const int64_t units = rows * S;
    if (units > (int64_t)INT32_MAX) return DFLASH2_ESHAPE;
    const Layout L = topk_layout(rows, V);
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return DFLASH2_EWORKSPACE;

    cudaStream_t s = (cudaStream_t)stream;
    unsigned* counters = (unsigned*)((char*)ws + L.counters_off);
    TopkPartial* part = (TopkPartial*)((char*)ws + L.part_off);
    if (cudaMemsetAsync(counters, 0, (size_t)rows * 4, s) != cudaSuccess) return DFLASH2_ECUDA;

    // TMA bulk copies need 16-byte aligned chunk starts and 16-byte multiples
    const bool tma = aligned(logits, 16) && (row_stride * es) % 16 == 0 && (V * es) % 16 == 0;
    const float c2 = (float)((double)inv_temperature * 1.4426950408889634);
#define DFL_TOPK(BF, TM)                                                                          \
    do {                                                                                          \
        auto kern = topk_softmax_kernel<BF, TM>;                                                  \
        const size_t dyn = TM ? 2 * (size_t)CHUNK * (BF ? 2 : 4) : 0;                             \
        if (dyn > 48 * 1024 &&                                                                    \
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn) !=  \
                cudaSuccess)                                                                      \
            return DFLASH2_ECUDA;                                                                 \
        const int grid = persistent_grid(kern, NT, dyn, units);                                   \
        kern<<<grid, NT, dyn, s>>>(logits, V, row_stride, (int)S, units, inv_temperature, c2, idx, \
                                   prob, logp, logz, part, counters);                             \
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

// Device address of the array on each device.  The host-side name of the
// array is only a stand-in; the address a kernel can use is looked up once per
// device, with that device current.
constexpr int NOALLOC_MAX_DEVICES = 64;
void* g_noalloc_addr[NOALLOC_MAX_DEVICES];
std::mutex g_noalloc_mu;

void* noalloc_scratch_on_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= NOALLOC_MAX_DEVICES) return nullptr;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        g_noalloc_addr[dev] = p;
    }
    return g_noalloc_addr[dev];
}

}  // namespace

extern "C" int dflash2_topk_softmax_noalloc(const void* logits, int dtype, int64_t rows, int64_t V,
                                            int64_t row_stride, float inv_temperature, int32_t* idx,
                                            float* prob, float* logp, float* logz,
                                            dflash2_stream_t stream) {
    if (!dtype_ok(dtype)) return DFLASH2_EDTYPE;
    if (rows < 0 || V < K || V > INT32_MAX || row_stride < V) return DFLASH2_ESHAPE;
    if (rows > 0 && topk_layout(rows, V).total > NOALLOC_SCRATCH_BYTES)
        return DFLASH2_EWORKSPACE;  // more rows than the built-in scratch holds
    if (rows == 0) return DFLASH2_OK;
    void* scratch = noalloc_scratch_on_current_device();
    if (!scratch) return DFLASH2_ECUDA;
    return dflash2_topk_softmax(logits, dtype, rows, V, row_stride, inv_temperature, idx, prob, logp,
                                logz, scratch, NOALLOC_SCRATCH_BYTES, stream);
}
