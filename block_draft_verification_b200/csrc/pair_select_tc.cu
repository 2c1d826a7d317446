// pair_select_tc.cu -- the pair selector with its dense contraction on the
// tensor cores (tcgen05), for bf16 embedding tables.
//
// Sources: "DFlash 2 — 3× plus de tokens sur Qwen3.8-27B, même sortie"
// (tamsi.dev), section "L’idée, sans le papier": pick a coherent path through
// the top-16 candidate lists with a small pair selector; "DFlash 2"
// (myaiexp.com), section "主な機能": adjacent candidate pairs are scored;
// "Qwen 3.8 27B + DFlash2: 140 Token/Sec?" (postsingularityinstitute.com),
// section "Résumé": candidates chosen by a bilinear attention.  The form:
//   pair(a, b) = e(a)^T W e(b),
//   score(path) = sum_i logp[i][k_i] + pair(anchor, c[0][k_0])
//               + sum_{i>0} pair(c[i-1][k_{i-1}], c[i][k_i]),
// maximised exactly by the max-sum recursion (ties: the smaller rank).
//
// One CTA per sequence.  The left rows of the pair scores -- the anchor and
// the 16 candidates of every position but the last -- are gathered into
// windows of 8 slots of 16 rows (128 rows, slot 0 of the first window the
// anchor), and F = E_left W runs as one M = 128, N = d, K = d tcgen05 GEMM per
// window into TMEM.  The embeddings are bf16, so E is exact as an operand; W is
// fp32 and is split into three bf16 planes, W = W1 + W2 + W3 (each plane the
// bf16 rounding of what the previous ones leave; 24 bits in all, W's fp32
// mantissa), accumulated in the same fp32 accumulator: F keeps fp32 accuracy.
// The 16 x 16 blocks S_i = F_i E_i^T run on the tensor cores too: F is split
// the same way into three bf16 planes (exact), and S_all = F E_right^T
// (M = N = 128) accumulates them in a second TMEM region, whose diagonal
// blocks are the S_i; the max-sum recursion runs in one warp from shared
// memory.  Nothing but the path leaves the SM.
#include <cuda_bf16.h>

#include "common.cuh"
#include "stream.cuh"
#include "tc.cuh"
#include "workspace.cuh"

namespace dfl {

constexpr int PT_THREADS = 256;
constexpr int PT_ROWS = 128;   // accumulator rows per window: 8 slots of K rows
constexpr int PT_SLOTS = PT_ROWS / K;

// Byte offset of element (r, k) of a K-major bf16 operand tile of `rows` rows
// in the 128-byte-swizzled layout the descriptors describe: K blocks of 64
// elements, each `rows` x 128 bytes; 8-row groups 1024 bytes apart; the
// 16-byte chunk of a row XORed with the row's index in its group.
__device__ __forceinline__ uint32_t swz_off(int r, int k, int rows) {
    const int kb = k >> 6, c = (k & 63) >> 3;
    return (uint32_t)(kb * rows * 128 + (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4) +
                      ((k & 7) << 1));
}

// Shared memory of one CTA (dynamic, 1024-byte aligned): the three W planes
// (B operand of F, d x d each), the left rows (A operand of F, 128 x d; then,
// one plane at a time, the bf16 planes of F as the A operand of S), the right
// rows (B operand of S, 128 x d), the pair scores of the sequence.
template <int D>
struct PtLayout {
    static constexpr uint32_t W_OFF = 0;
    static constexpr uint32_t W_PLANE = D * D * 2;
    static constexpr uint32_t A_OFF = 3 * W_PLANE;
    static constexpr uint32_t R_OFF = A_OFF + PT_ROWS * D * 2;
    static constexpr uint32_t S_OFF = R_OFF + PT_ROWS * D * 2;
    static size_t bytes(int G) {
        return 1024 + S_OFF + 4 * (size_t)(K + (size_t)K * K * (G > 1 ? G - 1 : 0));
    }
};

template <int D>
__global__ void __launch_bounds__(PT_THREADS, 1) pair_select_tc_kernel(
    const int32_t* __restrict__ idx, const float* __restrict__ logp,
    const int32_t* __restrict__ anchor, const __nv_bfloat16* __restrict__ emb,
    const float* __restrict__ W, int64_t V, int G, int32_t* __restrict__ path_tok,
    int32_t* __restrict__ path_rank, float* __restrict__ path_score) {
    using L = PtLayout<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    float* const s_sc = (float*)(sm + L::S_OFF);  // anchor row [K], then [G-1][K][K]
    __shared__ float s_lp[DFLASH2_MAX_BLOCK * K];
    __shared__ int32_t s_cand[DFLASH2_MAX_BLOCK * K];
    __shared__ double s_delta[2][K];
    __shared__ uint8_t s_back[DFLASH2_MAX_BLOCK][K];
    __shared__ int s_path[DFLASH2_MAX_BLOCK];
    __shared__ __align__(8) uint64_t s_bar;
    __shared__ __align__(8) uint64_t s_wbar;
    __shared__ uint32_t s_tmem;
    __shared__ int s_fail;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int b = blockIdx.x;
    const int32_t* cand = idx + (int64_t)b * G * K;
    const uint32_t bar = smem_u32(&s_bar);
    const int32_t anc = anchor ? anchor[b] : -1;

    const uint32_t wbar = smem_u32(&s_wbar);
    if (t == 0) {
        mbar_init(bar, 1);
        mbar_init(wbar, 1);
        mbar_fence_init();
        s_fail = 0;
        // W (fp32, d x d) into the operand tiles' space (which the gathered
        // rows overwrite only after the split), in 8 KB bulk copies that
        // proceed side by side
        mbar_expect_tx(wbar, (uint32_t)(D * D * 4));
        for (uint32_t off = 0; off < (uint32_t)(D * D * 4); off += 8192u)
            bulk_g2s_nx(smem_u32(sm + L::A_OFF) + off, (const char*)W + off, 8192u, wbar);
    }
    if (warp == 2) {  // 256 TMEM columns: F (d columns at 0), S (128 columns at 128)
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&s_tmem)),
                     "r"(256));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
        tc_fence_before();
    }
    for (int e = t; e < G * K; e += PT_THREADS) {
        s_lp[e] = logp[(int64_t)b * G * K + e];
        s_cand[e] = cand[e];
    }
    if (!anchor && t < K) s_sc[t] = 0.0f;  // no anchor: no term before position 0
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    constexpr int VPR = D / 8;                        // 16-byte vectors per embedding row
    constexpr int NV = 2 * PT_ROWS * VPR / PT_THREADS;  // vectors per thread (both tiles)
    const int nwin = (G + PT_SLOTS - 1) / PT_SLOTS;
    int ncommit = 0;  // commits waited on so far (the barrier's phase)
    for (int wdw = 0; wdw < nwin; ++wdw) {
        // ---- gather: left rows (slot s: the anchor for s = 0, else the
        // candidates of position s - 1) and right rows (the candidates of
        // position s), both slots 8 wdw .. 8 wdw + 7; missing rows are zero.
        // The loads are issued first and held in registers.
        uint4 v[NV];
#pragma unroll
        for (int j = 0; j < NV; ++j) {
            const int e = t + j * PT_THREADS;
            const int tile = e / (PT_ROWS * VPR);  // 0 left, 1 right
            const int rem = e - tile * PT_ROWS * VPR;
            const int r = rem / VPR, c = rem - r * VPR;
            const int s = PT_SLOTS * wdw + (r >> 4), k = r & 15;
            bool need = false;
            int32_t tok = 0;
            if (tile == 0) {
                if (s == 0) {
                    need = anchor && k == 0;
                    tok = anc;
                } else if (s - 1 < G - 1) {  // the last position is never on the left
                    need = true;
                    tok = s_cand[(s - 1) * K + k];
                }
            } else if (s < G) {
                need = true;
                tok = s_cand[s * K + k];
            }
            v[j] = make_uint4(0u, 0u, 0u, 0u);
            if (need) {
                if ((uint32_t)tok < (uint64_t)V)
                    v[j] = __ldg((const uint4*)(emb + (int64_t)tok * D) + c);
                else if (c == 0)
                    atomicOr(&g_dev_err, ERR_INPUT);  // outside [0, V): a zero embedding
            }
        }
        if (wdw == 0) {
            // the three bf16 planes of W as the B operand, B[n][k] = W[k][n]:
            // thread task (n, 8 consecutive k) reads W's column n from the
            // staged copy and writes one 16-byte vector per plane
            const bool wok = mbar_wait(wbar, 0);
            if (!wok && t == 0) {
                atomicOr(&g_dev_err, ERR_STREAM);
                s_fail = 1;
            }
            const float* sw = (const float*)(sm + L::A_OFF);
            for (int task = t; task < D * D / 8 && wok; task += PT_THREADS) {
                const int n = task % D, kc = task / D;
                uint32_t p1[4], p2[4], p3[4];
#pragma unroll
                for (int i = 0; i < 8; i += 2) {
                    float r1[2], r2[2];
                    __nv_bfloat16 b1[2], b2[2], b3[2];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const float w = sw[(8 * kc + i + h) * D + n];
                        b1[h] = __float2bfloat16_rn(w);
                        r1[h] = w - __bfloat162float(b1[h]);
                        b2[h] = __float2bfloat16_rn(r1[h]);
                        r2[h] = r1[h] - __bfloat162float(b2[h]);
                        b3[h] = __float2bfloat16_rn(r2[h]);
                    }
                    p1[i / 2] = (uint32_t)__bfloat16_as_ushort(b1[0]) |
                                ((uint32_t)__bfloat16_as_ushort(b1[1]) << 16);
                    p2[i / 2] = (uint32_t)__bfloat16_as_ushort(b2[0]) |
                                ((uint32_t)__bfloat16_as_ushort(b2[1]) << 16);
                    p3[i / 2] = (uint32_t)__bfloat16_as_ushort(b3[0]) |
                                ((uint32_t)__bfloat16_as_ushort(b3[1]) << 16);
                }
                const uint32_t o = swz_off(n, 8 * kc, D);
                *(uint4*)(sm + L::W_OFF + o) = make_uint4(p1[0], p1[1], p1[2], p1[3]);
                *(uint4*)(sm + L::W_OFF + L::W_PLANE + o) = make_uint4(p2[0], p2[1], p2[2], p2[3]);
                *(uint4*)(sm + L::W_OFF + 2 * L::W_PLANE + o) = make_uint4(p3[0], p3[1], p3[2], p3[3]);
            }
            __syncthreads();  // the staged W is consumed: the tiles may be written
        }
#pragma unroll
        for (int j = 0; j < NV; ++j) {
            const int e = t + j * PT_THREADS;
            const int tile = e / (PT_ROWS * VPR);
            const int rem = e - tile * PT_ROWS * VPR;
            const int r = rem / VPR, c = rem - r * VPR;
            *(uint4*)(sm + (tile == 0 ? L::A_OFF : L::R_OFF) + swz_off(r, 8 * c, PT_ROWS)) = v[j];
        }
        // generic-proxy writes of the operands before the tensor core reads them
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();
        // ---- F = E_left (W1 + W2 + W3): 3 planes x d / 16 MMAs, one commit
        if (s_fail) break;  // W never arrived (uniform: set before the last barrier)
        if (t == 0) {
            tc_fence_after();
            const uint32_t idesc = instr_desc(PT_ROWS, D);
            const uint32_t a0 = smem_u32(sm + L::A_OFF), b0 = smem_u32(sm + L::W_OFF);
#pragma unroll
            for (int p = 0; p < 3; ++p)
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t a = a0 + (ks >> 2) * (PT_ROWS * 128) + (ks & 3) * 32;
                    const uint32_t bb = b0 + p * L::W_PLANE + (ks >> 2) * (D * 128) + (ks & 3) * 32;
                    mma_bf16(tmem, smem_desc(a), smem_desc(bb), idesc, (p | ks) ? 1u : 0u);
                }
            mma_commit(bar);
        }
        bool ok = mbar_wait(bar, (uint32_t)(ncommit++ & 1));
        ok = __syncthreads_and(ok) != 0;  // one verdict for the CTA
        tc_fence_after();
        // ---- S blocks on the tensor cores: F (fp32, TMEM) is split into
        // three bf16 planes F1 + F2 + F3 (24 bits in all: exact), each
        // written over the left-row tile in turn and multiplied by the right
        // rows into one fp32 accumulator, S_all = F E_right^T (128 x 128);
        // its diagonal 16 x 16 blocks are the S_pos.  Thread (quadrant q,
        // half h) splits columns [h d/2, h d/2 + d/2) of F row 32 q + lane.
        const int q = warp & 3, h = warp >> 2;
        const int r = 32 * q + lane;
        constexpr int HC = D / 2;
        float res[HC];
#pragma unroll
        for (int cc = 0; cc < HC / 32; ++cc) {
            float f[32];
            tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(h * HC + 32 * cc), f);
#pragma unroll
            for (int j = 0; j < 32; ++j) res[32 * cc + j] = f[j];
        }
        const uint32_t idesc_s = instr_desc(PT_ROWS, PT_ROWS);
        // With one window W is no longer needed: the three planes go into its
        // space (and the left tile's, when d is small) and meet the right rows
        // in one round; with more, each plane in turn over the left-row tile
        // (W stays for the next window).
        constexpr bool FIT3 = 3 * PT_ROWS * D * 2 <= (int)L::R_OFF;  // W's space and the left tile
        const bool one_round = FIT3 && nwin == 1;
        const int nround = one_round ? 1 : 3;
#pragma unroll 1
        for (int rd = 0; rd < nround && ok; ++rd) {
#pragma unroll
            for (int vv = 0; vv < HC / 8; ++vv) {
#pragma unroll 1
                for (int p = one_round ? 0 : rd; p < (one_round ? 3 : rd + 1); ++p) {
                    uint32_t w4[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const __nv_bfloat16 b0 = __float2bfloat16_rn(res[8 * vv + 2 * i]);
                        const __nv_bfloat16 b1 = __float2bfloat16_rn(res[8 * vv + 2 * i + 1]);
                        res[8 * vv + 2 * i] -= __bfloat162float(b0);
                        res[8 * vv + 2 * i + 1] -= __bfloat162float(b1);
                        w4[i] = (uint32_t)__bfloat16_as_ushort(b0) |
                                ((uint32_t)__bfloat16_as_ushort(b1) << 16);
                    }
                    const uint32_t base = one_round ? L::W_OFF + p * (uint32_t)(PT_ROWS * D * 2) : L::A_OFF;
                    *(uint4*)(sm + base + swz_off(r, h * HC + 8 * vv, PT_ROWS)) =
                        make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc_fence_before();
            __syncthreads();
            if (t == 0) {
                tc_fence_after();
                const uint32_t b0 = smem_u32(sm + L::R_OFF);
                for (int p = 0; p < (one_round ? 3 : 1); ++p) {
                    const uint32_t a0 = smem_u32(sm + (one_round ? L::W_OFF + p * (uint32_t)(PT_ROWS * D * 2) : L::A_OFF));
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t a = a0 + (ks >> 2) * (PT_ROWS * 128) + (ks & 3) * 32;
                        const uint32_t bb = b0 + (ks >> 2) * (PT_ROWS * 128) + (ks & 3) * 32;
                        mma_bf16(tmem + 128u, smem_desc(a), smem_desc(bb), idesc_s,
                                 (rd | p | ks) ? 1u : 0u);
                    }
                }
                mma_commit(bar);
            }
            ok = __syncthreads_and(mbar_wait(bar, (uint32_t)(ncommit++ & 1))) != 0;
            tc_fence_after();
        }
        if (!ok && lane == 0) {
            atomicOr(&g_dev_err, ERR_MMA);
            s_fail = 1;
        }
        // the diagonal blocks: warp q (h = 0) reads S columns 32 q .. 32 q + 31
        // (rows 32 q .. 32 q + 15 need the first 16, the next 16 rows the rest)
        if (h == 0) {
            const int slot = r >> 4, kr = r & 15;
            const int pos = PT_SLOTS * wdw + slot;  // S_pos: left slot pos, right position pos
            const bool valid = ok && pos < G && (pos > 0 || (anchor && kr == 0));
            float sv[32];
            tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + 128u + (uint32_t)(32 * q), sv);
            if (valid) {
                float* dst = (pos == 0) ? s_sc : s_sc + K + (size_t)K * K * (pos - 1) + kr * K;
#pragma unroll
                for (int j = 0; j < K; ++j) dst[j] = (lane < 16) ? sv[j] : sv[16 + j];
            }
        }
        tc_fence_before();
        __syncthreads();  // TMEM and both tiles free for the next window
    }

    // ---- max-sum recursion, one warp, lane k = candidate rank k (lanes
    // 16..31 mirror 0..15)
    if (warp == 0 && !s_fail) {
        const int k = lane & (K - 1);
        double delta = (double)s_lp[k] + (double)s_sc[k];
        for (int p = 1; p < G; ++p) {
            if (lane < K) s_delta[(p - 1) & 1][k] = delta;
            __syncwarp();
            const double* dprev = s_delta[(p - 1) & 1];
            const float* Sp = s_sc + K + K * K * (p - 1);
            // lanes 0..15 take predecessors 0..7, lanes 16..31 predecessors
            // 8..15; the halves meet by one exchange (ties: the smaller rank)
            double best = 0.0;
            int arg = -1;
            const int k0 = (lane >> 4) * (K / 2);
#pragma unroll
            for (int i = 0; i < K / 2; ++i) {
                const int kk = k0 + i;
                const double c_s = dprev[kk] + (double)Sp[kk * K + k];
                if (arg < 0 || c_s > best) {
                    best = c_s;
                    arg = kk;
                }
            }
            {
                const double ob = __shfl_xor_sync(FULL, best, 16);
                const int oa = __shfl_xor_sync(FULL, arg, 16);
                if (ob > best || (ob == best && oa < arg)) {
                    best = ob;
                    arg = oa;
                }
            }
            delta = (double)s_lp[p * K + k] + best;
            if (lane < K) s_back[p][k] = (uint8_t)arg;
        }
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
            const int rr = s_path[lane];
            path_rank[(int64_t)b * G + lane] = rr;
            path_tok[(int64_t)b * G + lane] = s_cand[lane * K + rr];
        }
    }
    if (warp == 2) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256));
    }
}

}  // namespace dfl

using namespace dfl;
using namespace dfl_host;

// Launch of the tensor-core selector (bf16 embeddings, d in {64, 128});
// arguments already checked by the entry point.
int dfl_pair_select_tc(const int32_t* idx, const float* logp, const int32_t* anchor,
                       const void* emb, int64_t V, int d, const float* W, int B, int G,
                       int32_t* path_tok, int32_t* path_rank, float* path_score,
                       cudaStream_t s) {
#define DFL_PTC(DD)                                                                               \
    do {                                                                                          \
        auto kern = pair_select_tc_kernel<DD>;                                                    \
        const size_t dyn = PtLayout<DD>::bytes(G);                                                \
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn) !=  \
            cudaSuccess)                                                                          \
            return DFLASH2_ECUDA;                                                                 \
        kern<<<B, PT_THREADS, dyn, s>>>(idx, logp, anchor, (const __nv_bfloat16*)emb, W, V, G,   \
                                        path_tok, path_rank, path_score);                         \
    } while (0)
    if (d == 128) DFL_PTC(128);
    else DFL_PTC(64);
#undef DFL_PTC
    return launch_status();
}

unsigned dfl_errors_select_tc(int clear) {
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_dev_err, sizeof v) != cudaSuccess) return 0xFFFFFFFFu;
    if (clear && v) {
        unsigned z = 0;
        cudaMemcpyToSymbol(g_dev_err, &z, sizeof z);
    }
    return v;
}
