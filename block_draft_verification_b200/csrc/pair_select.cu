// pair_select.cu -- bilinear adjacent-pair scores and the exact best path
// through the 16 candidates of every drafted position.
//
// Sources: "DFlash 2 — 3× plus de tokens sur Qwen3.8-27B, même sortie"
// (tamsi.dev), section "L’idée, sans le papier": pick a coherent path through
// candidate lists that are already good, with a small pair selector;
// "DFlash 2" (myaiexp.com), section "主な機能": adjacent candidate pairs are
// scored to keep the block coherent; "Qwen 3.8 27B + DFlash2: 140 Token/Sec?"
// (postsingularityinstitute.com), section "Résumé": candidates are chosen by a
// bilinear attention.  The form fixed here:
//   pair(a, b) = e(a)^T W e(b),
//   score(path) = sum_i logp[i][k_i] + pair(anchor, c[0][k_0])
//               + sum_{i>0} pair(c[i-1][k_{i-1}], c[i][k_i]),
// maximised exactly by the max-sum recursion over positions (ties: the smaller
// rank, at every back-pointer and at the end).
//
// One CTA per (sequence, position i): one TMA bulk copy brings W (fp32,
// 64 KB at d = 128) into shared memory while the threads gather the left
// embeddings (the anchor for i = 0, else the 16 candidates of position i-1)
// and the 16 right ones; then F = E_left W and S_i = F E_right^T from shared
// memory, and S_i goes to the workspace.  The last CTA of the
// sequence (arrival ticket) runs the recursion in one warp, lane k = state k,
// in fp64, and backtracks.
#include "common.cuh"
#include "stream.cuh"
#include "workspace.cuh"

namespace dfl {

template <bool EMB_BF16, int D>
__global__ void __launch_bounds__(NT, 2) pair_select_kernel(
    const int32_t* __restrict__ idx, const float* __restrict__ logp,
    const int32_t* __restrict__ anchor, const void* __restrict__ emb, const float* __restrict__ W,
    int G, int32_t* __restrict__ path_tok, int32_t* __restrict__ path_rank,
    float* __restrict__ path_score, float* __restrict__ scores, unsigned* __restrict__ counters) {
    constexpr int LD = D + 1;  // padded rows: conflict-free column walks
    extern __shared__ __align__(128) float s_w[];  // W [D][D]
    __shared__ float s_left[K][LD], s_right[K][LD], s_f[K][LD];
    __shared__ int32_t s_ltok[K], s_rtok[K];
    __shared__ uint8_t s_back[DFLASH2_MAX_BLOCK][K];
    __shared__ __align__(8) uint64_t s_bar;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int b = blockIdx.x / G, i = blockIdx.x - b * G;
    const int32_t* cand = idx + (int64_t)b * G * K;
    const int nl = (i == 0) ? 1 : K;
    const bool has_left = (i > 0) || (anchor != nullptr);
    float* out = scores + (int64_t)b * (K + (int64_t)K * K * (G - 1)) +
                 (i == 0 ? 0 : K + (int64_t)K * K * (i - 1));

    if (has_left) {
        const uint32_t bar = smem_u32(&s_bar);
        if (t == 0) {
            mbar_init(bar, 1);
            mbar_fence_init();
            bulk_g2s(smem_u32(s_w), W, (uint32_t)(D * D * 4), bar);
        }
        if (t < K) {
            s_rtok[t] = cand[i * K + t];
            if (t < nl) s_ltok[t] = (i == 0) ? anchor[b] : cand[(i - 1) * K + t];
        }
        __syncthreads();
        auto ld_emb = [&](int32_t tok, int j) -> float {
            const int64_t o = (int64_t)tok * D + j;
            if (EMB_BF16)
                return __uint_as_float((uint32_t)__ldg((const unsigned short*)emb + o) << 16);
            return __ldg((const float*)emb + o);
        };
        for (int e = t; e < K * D; e += NT) {
            const int k = e / D, j = e - k * D;
            s_right[k][j] = ld_emb(s_rtok[k], j);
            if (k < nl) s_left[k][j] = ld_emb(s_ltok[k], j);
        }
        const bool ok = __syncthreads_and(mbar_wait(bar, 0));
        if (!ok) {  // W never arrived: flag it, leave this position's scores unset
            if (t == 0) atomicOr(&g_dev_err, ERR_STREAM);
        } else {
            // F = E_left W: thread -> column l, a group of left rows
            constexpr int GROUPS = NT / D;  // 2 for d = 128, 4 for d = 64
            constexpr int RPG = K / GROUPS;  // rows per group
            const int l = t % D, g = t / D;
            float acc[RPG];
#pragma unroll
            for (int q = 0; q < RPG; ++q) acc[q] = 0.0f;
            if (g * RPG < nl) {
#pragma unroll 8
                for (int j = 0; j < D; ++j) {
                    const float w = s_w[j * D + l];
#pragma unroll
                    for (int q = 0; q < RPG; ++q) acc[q] = fmaf(s_left[g * RPG + q][j], w, acc[q]);
                }
            }
#pragma unroll
            for (int q = 0; q < RPG; ++q)
                if (g * RPG + q < nl) s_f[g * RPG + q][l] = acc[q];
            __syncthreads();
            // S[k][k'] = F[k] . E_right[k']
            const int k = t / K, k2 = t % K;
            if (k < nl) {
                float sc = 0.0f;
#pragma unroll 8
                for (int l2 = 0; l2 < D; ++l2) sc = fmaf(s_f[k][l2], s_right[k2][l2], sc);
                out[k * K + k2] = sc;
            }
        }
    } else if (t < K) {
        out[t] = 0.0f;  // no anchor: no term before position 0
    }
    __syncthreads();
    if (t == 0) __threadfence();

    if (!arrive_last(&counters[b], (unsigned)G)) return;
    if (warp != 0) return;

    // Max-sum recursion, lane k = candidate rank k (lanes 16..31 mirror 0..15).
    const float* sc = scores + (int64_t)b * (K + (int64_t)K * K * (G - 1));
    const float* lp = logp + (int64_t)b * G * K;
    const int k = lane & (K - 1);
    double delta = (double)lp[k] + (double)__ldcg(&sc[k]);
    for (int p = 1; p < G; ++p) {
        const float* Sp = sc + K + (int64_t)K * K * (p - 1);
        double best = 0.0;
        int arg = -1;
        for (int kk = 0; kk < K; ++kk) {
            const double dk = __shfl_sync(FULL, delta, kk);
            const double cand_s = dk + (double)__ldcg(&Sp[kk * K + k]);
            if (arg < 0 || cand_s > best) {
                best = cand_s;
                arg = kk;
            }
        }
        delta = (double)lp[p * K + k] + best;
        if (lane < K) s_back[p][k] = (uint8_t)arg;
    }
    // smallest rank with the maximal final score
    double bv = delta;
    int bk = k;
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) {
        const double ov = __shfl_xor_sync(FULL, bv, j);
        const int ok = __shfl_xor_sync(FULL, bk, j);
        if (ov > bv || (ov == bv && ok < bk)) {
            bv = ov;
            bk = ok;
        }
    }
    __syncwarp();
    if (lane == 0) {
        path_score[b] = (float)bv;
        int kk = bk;
        for (int p = G - 1; p >= 0; --p) {
            path_rank[(int64_t)b * G + p] = kk;
            path_tok[(int64_t)b * G + p] = cand[p * K + kk];
            if (p > 0) kk = s_back[p][kk];
        }
    }
}

}  // namespace dfl

using namespace dfl;
using namespace dfl_host;

unsigned dfl_errors_select(int clear) {
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_dev_err, sizeof v) != cudaSuccess) return 0xFFFFFFFFu;
    if (clear && v) {
        unsigned z = 0;
        cudaMemcpyToSymbol(g_dev_err, &z, sizeof z);
    }
    return v;
}

extern "C" int dflash2_pair_select(const int32_t* idx, const float* logp, const int32_t* anchor,
                                   const void* emb, int emb_dtype, int64_t V, int d,
                                   const float* W, int B, int G, int32_t* path_tok,
                                   int32_t* path_rank, float* path_score, void* ws,
                                   size_t ws_bytes, dflash2_stream_t stream) {
    if (!dtype_ok(emb_dtype)) return DFLASH2_EDTYPE;
    if (B < 0 || G < 1 || G >= DFLASH2_MAX_BLOCK || V < K || (d != 64 && d != 128))
        return DFLASH2_ESHAPE;
    if (B == 0) return DFLASH2_OK;
    if (!idx || !logp || !emb || !W || !path_tok || !path_rank || !path_score)
        return DFLASH2_EINVAL;
    if (!aligned(idx, 4) || !aligned(logp, 4) || (anchor && !aligned(anchor, 4)) ||
        !aligned(emb, elem_size(emb_dtype)) || !aligned(W, 16) || !aligned(path_tok, 4) ||
        !aligned(path_rank, 4) || !aligned(path_score, 4))
        return DFLASH2_EALIGN;
    if ((int64_t)B * G > (int64_t)INT32_MAX) return DFLASH2_ESHAPE;
    const Layout L = select_layout(B, G);
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return DFLASH2_EWORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned* counters = (unsigned*)((char*)ws + L.counters_off);
    float* scores = (float*)((char*)ws + L.part_off);
    if (cudaMemsetAsync(counters, 0, (size_t)B * 4, s) != cudaSuccess) return DFLASH2_ECUDA;
    const dim3 grid((unsigned)((int64_t)B * G)), block(NT);
#define DFL_SEL(BF, DD)                                                                          \
    do {                                                                                         \
        auto kern = pair_select_kernel<BF, DD>;                                                  \
        const int dyn = DD * DD * 4;                                                             \
        if (dyn > 48 * 1024 &&                                                                   \
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn) !=      \
                cudaSuccess)                                                                     \
            return DFLASH2_ECUDA;                                                                \
        kern<<<grid, block, dyn, s>>>(idx, logp, anchor, emb, W, G, path_tok, path_rank,         \
                                      path_score, scores, counters);                             \
    } while (0)
    if (emb_dtype == DFLASH2_BF16) {
        if (d == 128) DFL_SEL(true, 128);
        else DFL_SEL(true, 64);
    } else {
        if (d == 128) DFL_SEL(false, 128);
        else DFL_SEL(false, 64);
    }
#undef DFL_SEL
    return launch_status();
}
