// topk_softmax.cu -- softmax over the vocabulary and the 16 best candidates of
// every drafted position, in one pass over the logits.
//
// Source: "DFlash 2 — 3× plus de tokens sur Qwen3.8-27B, même sortie"
// (tamsi.dev), section "L’idée, sans le papier": the right token lies in the
// drafter's top 16 far more often than at top 1, and the selector picks among
// those 16 per position; "DFlash 2" (myaiexp.com), section "主な機能": the
// path selector keeps the top-16 candidates of each position.
//
// One CTA per (row, 16384-element chunk).  Each thread holds 64 elements
// (eight 128-bit loads in flight for bf16), takes its max and sum-exp, and
// the block merges them in a fixed order.  The chunk's top-16 is exact
// without sorting the chunk: the 16th largest per-thread maximum T bounds
// the answer, only the (at most 16) threads holding keys at or above it
// contribute candidates, and one warp sorts those.  The last CTA of a row
// (arrival ticket, no waiting) merges the row's chunk partials in chunk
// order and writes idx / prob / logp / logz.
#include "common.cuh"
#include "workspace.cuh"

namespace dfl {

template <bool BF16, bool VEC>
__global__ void __launch_bounds__(NT) topk_softmax_kernel(
    const void* __restrict__ logits, int64_t V, int64_t row_stride, int S, float inv_t, float c2,
    int32_t* __restrict__ idx, float* __restrict__ prob, float* __restrict__ logp,
    float* __restrict__ logz, TopkPartial* __restrict__ part, unsigned* __restrict__ counters) {
    using R = Row<BF16>;
    __shared__ uint32_t s_top[NT / 32][K];
    __shared__ uint64_t s_cand[K * EPT];
    __shared__ Lse s_lse[NT / 32];
    __shared__ uint32_t s_tie[NT];
    __shared__ unsigned s_ncand, s_ntie;
    __shared__ uint32_t s_thr, s_vk;
    __shared__ Lse s_chunk;

    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int64_t unit = blockIdx.x;
    const int64_t row = unit / S;
    const int chunk = (int)(unit - row * S);
    const int64_t v0 = (int64_t)chunk * CHUNK;
    const int64_t vend = min(V, v0 + (int64_t)CHUNK);
    const char* rowp = (const char*)logits + row * row_stride * (BF16 ? 2 : 4);

    uint4 r[R::NV];
    R::template load<VEC>(rowp, v0, vend, r);
    const Lse mine = thread_lse<BF16>(r, c2);
    if (t == 0) {
        s_ncand = 0;
        s_ntie = 0;
    }

    // (1) chunk softmax partial and (2) the 16th largest thread maximum, T.
    Lse wl = warp_lse(mine, c2);
    if (lane == 0) s_lse[warp] = wl;
    const uint32_t my_ord = (mine.m == -INFINITY) ? 0u : ord32(mine.m);
    uint32_t srt = warp_sort_desc(my_ord);
    if (lane < K) s_top[warp][lane] = srt;
    __syncthreads();
    if (warp == 0) {
        uint32_t acc = (lane < K) ? s_top[0][lane] : 0u;
        for (int w = 1; w < NT / 32; ++w) acc = warp_merge_desc(lane < K ? acc : s_top[w][31 - lane]);
        if (lane == K - 1) s_thr = acc;  // 0: fewer than 16 threads hold elements
        if (lane == 0) {
            Lse tot = s_lse[0];
            for (int w = 1; w < NT / 32; ++w) tot = lse_merge(tot, s_lse[w], c2);
            s_chunk = tot;
        }
    }
    __syncthreads();

    // (3) Which threads can hold a top-16 element: every thread whose maximum
    // is above T, and, among the threads whose maximum equals T, those whose
    // first index of T is among the lowest (16 - #above).
    const uint32_t thr = s_thr;
    const bool above = my_ord > thr;
    const bool tie = thr != 0u && my_ord == thr;
    const int n_above = __syncthreads_count(above);
    uint32_t my_first = 0xFFFFFFFFu;
    if (tie) {
#pragma unroll
        for (int i = R::NV - 1; i >= 0; --i)
#pragma unroll
            for (int e = R::VW - 1; e >= 0; --e)
                if (R::elem(r[i], e) == mine.m) my_first = (uint32_t)R::index_of(v0, i, e);
        s_tie[atomicAdd(&s_ntie, 1u)] = my_first;
    }
    __syncthreads();
    if (tie) {
        const unsigned n = s_ntie;
        unsigned rank = 0;
        for (unsigned j = 0; j < n; ++j) rank += s_tie[j] < my_first;
        if (rank == (unsigned)(K - n_above - 1)) s_vk = my_first;
    }
    __syncthreads();

    // (4) Candidates: keys at or above (T, vk); at most 16 threads x 64.
    const float tv = (thr == 0u) ? -INFINITY : unord32(thr);
    const uint32_t vk = (thr == 0u) ? 0u : s_vk;
    if (above || (tie && my_first <= vk)) {
#pragma unroll
        for (int i = 0; i < R::NV; ++i)
#pragma unroll
            for (int e = 0; e < R::VW; ++e) {
                const float x = R::elem(r[i], e);
                const uint32_t v = (uint32_t)R::index_of(v0, i, e);
                if (x > tv || (thr != 0u && x == tv && v <= vk))
                    s_cand[atomicAdd(&s_ncand, 1u)] = make_key(x, v);
            }
    }
    __syncthreads();

    // (5) Sort the candidates 16 at a time into a running top-16 (warp 0).
    if (warp == 0) {
        const unsigned n = s_ncand;
        uint64_t acc = 0;
        for (unsigned base = 0; base < n; base += K) {
            uint64_t v = acc;
            if (lane >= K) v = (base + lane - K < n) ? s_cand[base + lane - K] : 0ull;
            acc = warp_sort_desc(v);
        }
        if (lane < K) part[unit].key[lane] = acc;
        if (lane == 0) {
            part[unit].m = s_chunk.m;
            part[unit].s = s_chunk.s;
        }
        __threadfence();
    }

    // (6) The last chunk of the row to finish merges the row.
    if (!arrive_last(&counters[row], (unsigned)S)) return;
    if (warp != 0) return;
    const TopkPartial* P = part + row * S;
    auto ldkey = [](const uint64_t* p) {
        return (uint64_t)__ldcg((const unsigned long long*)p);
    };
    uint64_t acc = (lane < K) ? ldkey(&P[0].key[lane]) : 0ull;
    for (int c = 1; c < S; ++c) acc = warp_merge_desc(lane < K ? acc : ldkey(&P[c].key[31 - lane]));
    // softmax: max over chunks, then the sum in chunk order (fp64)
    float M = -INFINITY;
    for (int c = lane; c < S; c += 32) M = fmaxf(M, __ldcg(&P[c].m));
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, j));
    double ssum = 0.0;
    if (lane == 0)
        for (int c = 0; c < S; ++c) {
            const float mc = __ldcg(&P[c].m), sc = __ldcg(&P[c].s);
            if (mc != -INFINITY) ssum += (double)sc * exp2(((double)mc - (double)M) * (double)c2);
        }
    ssum = __shfl_sync(FULL, ssum, 0);
    const double lns = log(ssum);
    if (lane < K) {
        const double x = (double)key_value(acc);
        const double dz = (x - (double)M) * (double)inv_t;
        const int64_t o = row * K + lane;
        idx[o] = (int32_t)key_index(acc);
        prob[o] = (float)(exp2((x - (double)M) * (double)c2) / ssum);
        logp[o] = (float)(dz - lns);
        if (lane == 0) logz[row] = (float)((double)M * (double)inv_t + lns);
    }
}

}  // namespace dfl

using namespace dfl;
using namespace dfl_host;

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
    if (rows * S > (int64_t)INT32_MAX) return DFLASH2_ESHAPE;
    const Layout L = topk_layout(rows, V);
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return DFLASH2_EWORKSPACE;

    cudaStream_t s = (cudaStream_t)stream;
    unsigned* counters = (unsigned*)((char*)ws + L.counters_off);
    TopkPartial* part = (TopkPartial*)((char*)ws + L.part_off);
    if (cudaMemsetAsync(counters, 0, (size_t)rows * 4, s) != cudaSuccess) return DFLASH2_ECUDA;

    const bool vec = aligned(logits, 16) && (row_stride * es) % 16 == 0;
    const float c2 = (float)((double)inv_temperature * 1.4426950408889634);
    const dim3 grid((unsigned)(rows * S)), block(NT);
    if (dtype == DFLASH2_BF16) {
        if (vec)
            topk_softmax_kernel<true, true><<<grid, block, 0, s>>>(logits, V, row_stride, (int)S,
                inv_temperature, c2, idx, prob, logp, logz, part, counters);
        else
            topk_softmax_kernel<true, false><<<grid, block, 0, s>>>(logits, V, row_stride, (int)S,
                inv_temperature, c2, idx, prob, logp, logz, part, counters);
    } else {
        if (vec)
            topk_softmax_kernel<false, true><<<grid, block, 0, s>>>(logits, V, row_stride, (int)S,
                inv_temperature, c2, idx, prob, logp, logz, part, counters);
        else
            topk_softmax_kernel<false, false><<<grid, block, 0, s>>>(logits, V, row_stride, (int)S,
                inv_temperature, c2, idx, prob, logp, logz, part, counters);
    }
    return launch_status();
}
