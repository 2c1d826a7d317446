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
// and the 16 right ones with 16-byte loads issued together; then
// F = E_left W and S_i = F E_right^T from shared memory, and S_i goes to the
// workspace.  The last CTA of the sequence (arrival ticket) fetches every S_i,
// logp and the candidate ids of the sequence into shared memory in one
// parallel pass, runs the recursion in one warp from there (lane k = state k,
// fp64), backtracks in shared memory and writes the path with one store per
// position.
#include "common.cuh"
#include "stream.cuh"
#include "workspace.cuh"

namespace dfl {

template <bool EMB_BF16, int D>
__global__ void __launch_bounds__(NT, 2) pair_select_kernel(
    const int32_t* __restrict__ idx, const float* __restrict__ logp,
    const int32_t* __restrict__ anchor, const void* __restrict__ emb, const float* __restrict__ W,
    int64_t V, int G, int32_t* __restrict__ path_tok, int32_t* __restrict__ path_rank,
    float* __restrict__ path_score, float* __restrict__ scores, unsigned* __restrict__ counters) {
    constexpr int LD = D + 4;                  // padded rows, still 16-byte aligned
    constexpr int ES = EMB_BF16 ? 2 : 4;
    constexpr int VE = 16 / ES;                // elements per 16-byte vector
    constexpr int RV = D / VE;                 // vectors per embedding row
    constexpr int IPT = (2 * K * RV + NT - 1) / NT;
    // W [D][D] in phase 1; the sequence's pair scores in phase 2
    extern __shared__ __align__(128) float s_dyn[];
    __shared__ __align__(16) float s_leftT[D][K + 4];  // left rows transposed: [column][row]
    __shared__ __align__(16) float s_right[K][LD];
    __shared__ __align__(16) float s_f[K][LD];
    __shared__ int32_t s_tok[2 * K];           // right rows 0..15, left rows 16..
    __shared__ float s_lp[DFLASH2_MAX_BLOCK * K];
    __shared__ int32_t s_cand[DFLASH2_MAX_BLOCK * K];
    __shared__ double s_delta[2][K];
    __shared__ uint8_t s_back[DFLASH2_MAX_BLOCK][K];
    __shared__ int s_path[DFLASH2_MAX_BLOCK];
    __shared__ __align__(8) uint64_t s_bar;
    __shared__ int s_bad;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int b = blockIdx.x / G, i = blockIdx.x - b * G;
    const int32_t* cand = idx + (int64_t)b * G * K;
    const int nl = (i == 0) ? 1 : K;
    const bool has_left = (i > 0) || (anchor != nullptr);
    const int64_t seq_scores = K + (int64_t)K * K * (G - 1);
    float* out = scores + (int64_t)b * seq_scores + (i == 0 ? 0 : K + (int64_t)K * K * (i - 1));

    bool ok = true;
    if (has_left) {
        const uint32_t bar = smem_u32(&s_bar);
        if (t == 0) {
            mbar_init(bar, 1);
            mbar_fence_init();
            bulk_g2s(smem_u32(s_dyn), W, (uint32_t)(D * D * 4), bar);
        }
        if (t < K) s_tok[t] = cand[i * K + t];
        else if (t < K + nl) s_tok[t] = (i == 0) ? anchor[b] : cand[(i - 1) * K + (t - K)];
        __syncthreads();
        // a token id outside [0, V) gets a zero embedding (no load) and is flagged
        if (t < K + nl && (uint32_t)s_tok[t] >= (uint64_t)V) atomicOr(&g_dev_err, ERR_INPUT);
        uint4 v[IPT];
#pragma unroll
        for (int q = 0; q < IPT; ++q) {  // all loads first: one memory round trip
            const int e = t + q * NT, r = e / RV, c = e - r * RV;
            v[q] = make_uint4(0u, 0u, 0u, 0u);
            if (r < K + nl && (uint32_t)s_tok[r] < (uint64_t)V)
                v[q] = __ldg((const uint4*)((const char*)emb + (int64_t)s_tok[r] * (D * ES)) + c);
        }
#pragma unroll
        for (int q = 0; q < IPT; ++q) {
            const int e = t + q * NT, r = e / RV, c = e - r * RV;
            if (r < K + nl) {
                const uint32_t w[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
                float f[VE];
#pragma unroll
                for (int u = 0; u < VE; ++u)
                    f[u] = EMB_BF16 ? __uint_as_float((u & 1) ? (w[u >> 1] & 0xFFFF0000u)
                                                              : (w[u >> 1] << 16))
                                    : __uint_as_float(w[u]);
                if (r < K) {
                    float4* dst = reinterpret_cast<float4*>(&s_right[r][c * VE]);
#pragma unroll
                    for (int u = 0; u < VE / 4; ++u)
                        dst[u] = make_float4(f[4 * u], f[4 * u + 1], f[4 * u + 2], f[4 * u + 3]);
                } else {
#pragma unroll
                    for (int u = 0; u < VE; ++u) s_leftT[c * VE + u][r - K] = f[u];
                }
            }
        }
        ok = __syncthreads_and(mbar_wait(bar, 0));
        if (!ok) {  // W never arrived: flag it, leave this position's scores unset
            if (t == 0) atomicOr(&g_dev_err, ERR_STREAM);
        } else {
            // F = E_left W with K split over the eight warps (warp w: rows
            // j of W in [w D/8, (w+1) D/8)); lane = a quad of 4 columns and
            // RL left rows, so every W element is read from shared memory
            // once.  Each warp's partial F goes to shared memory (over W once
            // every warp is done with it) and the partials are added in warp
            // order.
            constexpr int QUADS = D / 4;             // 32 for d = 128, 16 for d = 64
            constexpr int RL = K * QUADS / 32;       // left rows per lane: 16 or 8
            constexpr int KW = D / (NT / 32);        // rows of W per warp: 16 or 8
            const int cq = lane % QUADS, rg = (lane / QUADS) * RL;
            const float4* w4 = reinterpret_cast<const float4*>(s_dyn);
            float4 acc[RL];
#pragma unroll
            for (int r = 0; r < RL; ++r) acc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
            for (int jj = 0; jj < KW; ++jj) {
                const int j = warp * KW + jj;
                const float4 wj = w4[j * QUADS + cq];
#pragma unroll
                for (int r4 = 0; r4 < RL / 4; ++r4) {
                    const float4 e4 = *reinterpret_cast<const float4*>(&s_leftT[j][rg + 4 * r4]);
                    const float ev[4] = {e4.x, e4.y, e4.z, e4.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        float4& a = acc[4 * r4 + u];
                        a.x = fmaf(ev[u], wj.x, a.x);
                        a.y = fmaf(ev[u], wj.y, a.y);
                        a.z = fmaf(ev[u], wj.z, a.z);
                        a.w = fmaf(ev[u], wj.w, a.w);
                    }
                }
            }
            __syncthreads();  // every warp is done with W
            float4* part = reinterpret_cast<float4*>(s_dyn);  // [warp][row][quad]
#pragma unroll
            for (int r = 0; r < RL; ++r) part[(warp * K + rg + r) * QUADS + cq] = acc[r];
            __syncthreads();
            for (int o = t; o < K * QUADS; o += NT) {  // (row, quad) outputs
                const int r = o / QUADS, qd = o - r * QUADS;
                float4 f = part[r * QUADS + qd];
#pragma unroll
                for (int w = 1; w < NT / 32; ++w) {
                    const float4 g = part[(w * K + r) * QUADS + qd];
                    f.x += g.x;
                    f.y += g.y;
                    f.z += g.z;
                    f.w += g.w;
                }
                *reinterpret_cast<float4*>(&s_f[r][4 * qd]) = f;
            }
            __syncthreads();
            // S[k][k'] = F[k] . E_right[k'] (l ascending)
            const int k = t / K, k2 = t % K;
            if (k < nl) {
                float sc = 0.0f;
#pragma unroll 8
                for (int l2 = 0; l2 < D; l2 += 4) {
                    const float4 f = *reinterpret_cast<const float4*>(&s_f[k][l2]);
                    const float4 r = *reinterpret_cast<const float4*>(&s_right[k2][l2]);
                    sc = fmaf(f.x, r.x, sc);
                    sc = fmaf(f.y, r.y, sc);
                    sc = fmaf(f.z, r.z, sc);
                    sc = fmaf(f.w, r.w, sc);
                }
                out[k * K + k2] = sc;
            }
        }
    } else if (t < K) {
        out[t] = 0.0f;  // no anchor: no term before position 0
    }
    if (t == 0) s_bad = ok ? 0 : 1;
    __syncthreads();
    if (t == 0) __threadfence();

    if (!arrive_last(&counters[b], (unsigned)G)) return;
    if (t == 0) counters[b] = 0u;  // every CTA of the sequence has arrived: leave it zero
    if (s_bad) return;  // this CTA's W copy may still be in flight: leave its smem alone

    // ---- last CTA of the sequence: everything the recursion reads, in one pass
    const float* sc = scores + (int64_t)b * seq_scores;
    float* s_sc = s_dyn;
#pragma unroll 4
    for (int e = t; e < seq_scores; e += NT) s_sc[e] = __ldcg(&sc[e]);
    for (int e = t; e < G * K; e += NT) {
        s_lp[e] = logp[(int64_t)b * G * K + e];
        s_cand[e] = cand[e];
    }
    __syncthreads();
    if (warp != 0) return;

    // Max-sum recursion, lane k = candidate rank k (lanes 16..31 mirror 0..15).
    const int k = lane & (K - 1);
    double delta = (double)s_lp[k] + (double)s_sc[k];
    for (int p = 1; p < G; ++p) {
        if (lane < K) s_delta[(p - 1) & 1][k] = delta;
        __syncwarp();
        const double* dprev = s_delta[(p - 1) & 1];
        const float* Sp = s_sc + K + K * K * (p - 1);
        double best = 0.0;
        int arg = -1;
#pragma unroll
        for (int kk = 0; kk < K; ++kk) {
            const double c_s = dprev[kk] + (double)Sp[kk * K + k];
            if (arg < 0 || c_s > best) {
                best = c_s;
                arg = kk;
            }
        }
        delta = (double)s_lp[p * K + k] + best;
        if (lane < K) s_back[p][k] = (uint8_t)arg;
    }
    // smallest rank with the maximal final score
    double bv = delta;
    int bk = k;
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) {
        const double ov = __shfl_xor_sync(FULL, bv, j);
        const int ok2 = __shfl_xor_sync(FULL, bk, j);
        if (ov > bv || (ov == bv && ok2 < bk)) {
            bv = ov;
            bk = ok2;
        }
    }
    __syncwarp();
    if (lane == 0) {
        path_score[b] = (float)bv;
        int kk = bk;
        for (int p = G - 1; p >= 0; --p) {
            s_path[p] = kk;
            if (p > 0) kk = s_back[p][kk];
        }
    }
    __syncwarp();
    if (lane < G) {
        const int r = s_path[lane];
        path_rank[(int64_t)b * G + lane] = r;
        path_tok[(int64_t)b * G + lane] = s_cand[lane * K + r];
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

int dfl_pair_select_tc(const int32_t* idx, const float* logp, const int32_t* anchor,
                       const void* emb, int64_t V, int d, const float* W, int B, int G,
                       int32_t* path_tok, int32_t* path_rank, float* path_score,
                       cudaStream_t s);

extern "C" int dflash2_pair_select_ex(const int32_t* idx, const float* logp,
                                      const int32_t* anchor, const void* emb, int emb_dtype,
                                      int64_t V, int d, const float* W, int B, int G,
                                      int32_t* path_tok, int32_t* path_rank, float* path_score,
                                      int impl, void* ws, size_t ws_bytes,
                                      dflash2_stream_t stream) {
    if (!dtype_ok(emb_dtype)) return DFLASH2_EDTYPE;
    if (impl < DFLASH2_SELECT_AUTO || impl > DFLASH2_SELECT_TENSOR) return DFLASH2_EINVAL;
    if (impl == DFLASH2_SELECT_TENSOR && emb_dtype != DFLASH2_BF16) return DFLASH2_EDTYPE;
    if (B < 0 || G < 1 || G >= DFLASH2_MAX_BLOCK || V < K || (d != 64 && d != 128))
        return DFLASH2_ESHAPE;
    if (B == 0) return DFLASH2_OK;
    if (!idx || !logp || !emb || !W || !path_tok || !path_rank || !path_score)
        return DFLASH2_EINVAL;
    if (!aligned(idx, 4) || !aligned(logp, 4) || (anchor && !aligned(anchor, 4)) ||
        !aligned(emb, 16) || !aligned(W, 16) || !aligned(path_tok, 4) ||
        !aligned(path_rank, 4) || !aligned(path_score, 4))
        return DFLASH2_EALIGN;
    if ((int64_t)B * G > (int64_t)INT32_MAX) return DFLASH2_ESHAPE;
    const Layout L = select_layout(B, G);
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return DFLASH2_EWORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    // automatic choice: the tensor cores for bf16 tables from DFLASH2_SELECT_TC_MIN_B
    // sequences on (one CTA per sequence: its latency stays flat while the
    // CUDA-core path's grid of B G CTAs grows past one wave), the CUDA cores below
    const bool tensor = impl == DFLASH2_SELECT_TENSOR ||
                        (impl == DFLASH2_SELECT_AUTO && emb_dtype == DFLASH2_BF16 &&
                         B >= DFLASH2_SELECT_TC_MIN_B);
    if (tensor)
        return dfl_pair_select_tc(idx, logp, anchor, emb, V, d, W, B, G, path_tok, path_rank,
                                  path_score, s);
    unsigned* counters = (unsigned*)((char*)ws + L.counters_off);
    float* scores = (float*)((char*)ws + L.part_off);
    if (!L.self_clean && cudaMemsetAsync(counters, 0, (size_t)B * 4, s) != cudaSuccess)
        return DFLASH2_ECUDA;
    const dim3 grid((unsigned)((int64_t)B * G)), block(NT);
#define DFL_SEL(BF, DD)                                                                          \
    do {                                                                                         \
        auto kern = pair_select_kernel<BF, DD>;                                                  \
        const int dyn = (int)(4 * std::max<int64_t>(std::max<int64_t>((int64_t)DD * DD, 8LL * K * DD),    \
                                                    K + (int64_t)K * K * (G - 1)));              \
        /* static + dynamic may pass 48 KB: raise the ceiling to what this call uses */          \
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn) !=      \
            cudaSuccess)                                                                         \
            return DFLASH2_ECUDA;                                                                \
        kern<<<grid, block, dyn, s>>>(idx, logp, anchor, emb, W, V, G, path_tok, path_rank,         \
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

extern "C" int dflash2_pair_select(const int32_t* idx, const float* logp, const int32_t* anchor,
                                   const void* emb, int emb_dtype, int64_t V, int d,
                                   const float* W, int B, int G, int32_t* path_tok,
                                   int32_t* path_rank, float* path_score, void* ws,
                                   size_t ws_bytes, dflash2_stream_t stream) {
    return dflash2_pair_select_ex(idx, logp, anchor, emb, emb_dtype, V, d, W, B, G, path_tok,
                                  path_rank, path_score, DFLASH2_SELECT_AUTO, ws, ws_bytes,
                                  stream);
}
