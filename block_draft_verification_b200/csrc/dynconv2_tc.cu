// dynconv2_tc.cu -- tensor-core (tcgen05 + TMA) path of the two-tap dynamic
// depthwise conv, bf16.
//
// Source: "DFlash 2 — 3× plus de tokens sur Qwen3.8-27B, même sortie"
// (tamsi.dev), section "L’idée, sans le papier" (two-tap conv before/after each
// attention and MLP); "DFlash 2" (myaiexp.com), section "主な機能" (2-tap
// dynamic convolution).  out_t = x_t + a_t * x_t + b_t * x_{t-1}, with
// [a_t; b_t] = W_tap x_t and x_{-1} = x_prev.
//
// The tap projection is the GEMM D[2H x N] = W_tap[2H x H] . X^T[H x N] over
// the N = B*T tokens.  A tile is 64 output channels h0..h0+63 of one chunk of
// up to 256 tokens: its M = 128 accumulator stacks the 64 W_a rows and the 64
// matching W_b rows, so a and b of a channel meet in one accumulator and the
// conv, the residual and the rounding run in the epilogue.
//
// Work is split stream-K: the (tile, 64-wide K block) steps, tile-major, are
// cut into one contiguous run per CTA (one CTA per SM, launched
// cooperatively so all are resident), so every SM streams the same share of
// W_tap whatever the tile count.  A run is a sequence of segments (the part
// of the run inside one tile).  The CTA holding a tile's K block 0 owns the
// tile; a CTA whose run starts inside a tile (at most its first segment)
// writes that segment's fp32 accumulator to the workspace and raises its
// flag.  The owner adds those partials in K order (CTA order) to its own
// accumulator before the epilogue: a fixed summation order for given shapes.
// An owner only ever waits for the FIRST segment of later CTAs, which waits
// for nothing, so no wait chain forms.
//   warp 0   TMA producer: W tile (2 boxes of 64 x 64) + X tile (N x 64) per
//            step into a ring of shared-memory stages (128-byte swizzle)
//   warp 1   MMA issuer: tcgen05.mma (M=128, N, K=16) x 4 per step into one of
//            two TMEM accumulators (segments alternate, so a segment's
//            epilogue overlaps the next segment's MMAs)
//   warp 2   TMEM allocation / release
//   warps 4-7 epilogue: tcgen05.ld of their 32 TMEM lanes; a partial goes to
//            the workspace, an owned tile adds the partials, stages the
//            values in shared memory, then (token, 8-channel) items with
//            16-byte loads of x_t and x_{t-1} and one 16-byte store; warps
//            0-3, idle once the run's MMAs are issued, take half of the run's
//            last owned tile
// Every wait is bounded (one second, stream.cuh); on a timeout the kernel
// records a flag (dflash2_device_errors), stops issuing work, waits (bounded)
// for its tensor-core work in flight, releases TMEM and returns.  Every TMA
// load here fills only the issuing CTA's own shared memory.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "stream.cuh"
#include "tc.cuh"
#include "workspace.cuh"

namespace dfl {

constexpr int TC_BM = 128;          // accumulator rows: 64 a-channels + 64 b-channels
constexpr int TC_CH = 64;           // channels per CTA
constexpr int TC_BK = 64;           // K elements per stage (128 bytes of bf16)
constexpr int TC_MAXN = 256;        // tokens per accumulator
constexpr int TC_THREADS = 256;
constexpr int TC_A_BYTES = TC_BM * TC_BK * 2;  // 16 KB

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(map), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, int c3, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
        "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
        : "memory");
}
constexpr int TC_MAXCTA = 256;  // stream-K CTAs at most (one per SM)

// What the epilogue of an owned tile needs: its accumulator (TMEM column
// base), channels, tokens, and which partials it adds.
struct OwnTile {
    uint32_t tacc;
    int h0, tok0, bi0, q_reg, q_end;
    bool staged, reg_part, first_part;
};

struct TcShape {
    int H, T, ntok, BN, sw, sx, nkb, nh;  // W / X ring stages; nh: channel tiles per token chunk
    int bufcols;                           // TMEM columns per accumulator (power of 2, >= BN)
    int ngroups;                           // 32-column groups per accumulator
    int nctas;                             // stream-K CTAs
    int R;                                 // x_prev rows staged per tile (batches it touches)
    int64_t steps;                         // tiles * nkb
};

__device__ __forceinline__ int64_t run_start(const TcShape& sh, int p) {
    return sh.steps * p / sh.nctas;
}
// One bf16 from shared memory, widened to fp32 (exact).
__device__ __forceinline__ float lds_bf16(uint32_t addr) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
    return __uint_as_float((uint32_t)v << 16);
}
__device__ __forceinline__ void sts_bf16(uint32_t addr, float v) {
    const unsigned short b = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(b) : "memory");
}
__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__global__ void __launch_bounds__(TC_THREADS, 1) dynconv2_tc_kernel(
    const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
    const __grid_constant__ CUtensorMap map_xe, const __grid_constant__ CUtensorMap map_pe,
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ x_prev,
    __nv_bfloat16* __restrict__ out, TcShape sh, float4* __restrict__ partial,
    unsigned* __restrict__ flags, const uint8_t* __restrict__ wpk) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // two rings, 1024-byte aligned for the 128-byte swizzle: W tiles (HBM,
    // deeper) and X tiles (L2), each with its own full / empty barriers
    uint8_t* wring = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int xstage = sh.BN * TC_BK * 2;
    uint8_t* xring = wring + sh.sw * TC_A_BYTES;
    uint8_t* tail = xring + sh.sx * xstage;
    // an owned tile's inputs, row-major 128-byte rows (64 channels):
    // x of its BN tokens, x_prev of the R batches it touches, x of token tok0-1
    uint8_t* s_x = tail;
    uint8_t* s_xp = s_x + sh.BN * 128;
    uint8_t* s_x0 = s_xp + sh.R * 128;
    uint8_t* s_out = s_x0 + 128;  // [2][32 tokens][64 channels] bf16 outputs
    // wfull[SW], wempty[SW], xfull[SX], xempty[SX], tmem_full[2], tmem_empty[2], mma_done,
    // x tile, staged partial, helpers' go
    uint64_t* bars = (uint64_t*)(s_out + 8192);
    uint32_t* s_tmem = (uint32_t*)(bars + 2 * sh.sw + 2 * sh.sx + 8);
    int* s_fail = (int*)(s_tmem + 1);
    OwnTile& s_own = *(OwnTile*)(s_fail + 1);  // the last owned tile, for the helper warps

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int p = blockIdx.x;
    const int64_t s0 = run_start(sh, p), s1 = run_start(sh, p + 1);
    const uint32_t wfull0 = smem_u32(bars), wempty0 = wfull0 + 8 * sh.sw;
    const uint32_t xfull0 = wempty0 + 8 * sh.sw, xempty0 = xfull0 + 8 * sh.sx;
    const uint32_t tfull0 = xempty0 + 8 * sh.sx;
    const uint32_t tempty0 = tfull0 + 16;
    const uint32_t mdone = tfull0 + 32;
    const uint32_t xbar = tfull0 + 40;
    const uint32_t pbar = tfull0 + 48;  // a partial staged in the idle rings
    const uint32_t hbar = tfull0 + 56;  // the last owned tile is ready for the helper warps
    const uint32_t ncols = 2 * (uint32_t)sh.bufcols;

    if (threadIdx.x == 0) {
        for (int i = 0; i < sh.sw; ++i) {
            mbar_init(wfull0 + 8 * i, 1);
            mbar_init(wempty0 + 8 * i, 1);
        }
        for (int i = 0; i < sh.sx; ++i) {
            mbar_init(xfull0 + 8 * i, 1);
            mbar_init(xempty0 + 8 * i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(tfull0 + 8 * i, 1);
            mbar_init(tempty0 + 8 * i, 1);
        }
        mbar_init(mdone, 1);
        mbar_init(xbar, 1);
        mbar_init(pbar, 1);
        mbar_init(hbar, 1);
        mbar_fence_init();
        *s_fail = 0;
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(s_tmem)),
                     "r"(ncols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    // An owned tile's 32-token groups g0 .. g1-1, by a set of four warps
    // (warp w takes TMEM lanes 32 (w mod 4) ..; e: the thread's index in the
    // set): accumulator + partials in K order, the conv and the residual, bf16
    // rounding, 16-byte stores through the set's double-buffered output tile
    // `so` (synchronised by named barrier `bid`).  pp0 / pp1 hold groups g0 and
    // g0 + 1 of the register-prefetched partial, refilled two groups ahead.
    const uint32_t part_bytes = (uint32_t)sh.ngroups * 8 * TC_BM * 16;
    const uint32_t ring_bytes = (uint32_t)sh.sw * TC_A_BYTES + (uint32_t)sh.sx * xstage;
    auto own_groups = [&](const OwnTile& o, int g0, int g1, uint32_t so, int bid,
                          float4 (&pp0)[8], float4 (&pp1)[8]) {
        const int q = warp & 3, e = threadIdx.x & 127, row = 32 * q + lane;
        const uint32_t tacc = o.tacc + ((uint32_t)(32 * q) << 16);
        const float4* sp = (const float4*)wring;
        const float4* partr = partial + (int64_t)o.q_reg * sh.ngroups * 8 * TC_BM;
        auto set_sync = [&]() { asm volatile("bar.sync %0, 128;" ::"r"(bid) : "memory"); };
        // lane l of warp q: channel cl = 16q + (l & 15) of the tile, tokens
        // 16 (l >> 4) .. +15 of each 32-token group; a and b of the channel
        // meet by one exchange between lanes l and l ^ 16
        const int cl = 16 * q + (lane & 15), half = lane >> 4;
        for (int g = g0; g < g1; ++g) {
            float v[32];
            tmem_ld32(tacc + 32 * g, v);
            if (o.staged) {
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float4 w = sp[(g * 8 + c) * TC_BM + row];
                    v[4 * c] += w.x;
                    v[4 * c + 1] += w.y;
                    v[4 * c + 2] += w.z;
                    v[4 * c + 3] += w.w;
                }
            }
            if (o.reg_part) {
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    v[4 * c] += pp0[c].x;
                    v[4 * c + 1] += pp0[c].y;
                    v[4 * c + 2] += pp0[c].z;
                    v[4 * c + 3] += pp0[c].w;
                    pp0[c] = pp1[c];
                }
                if (g + 2 < g1)
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        pp1[c] = __ldcg(&partr[((int64_t)(g + 2) * 8 + c) * TC_BM + row]);
            }
            if (o.first_part) {
                for (int q2 = o.q_reg + 1; q2 < o.q_end; ++q2) {  // further partials, in K order
                    const float4* src = partial + (int64_t)q2 * sh.ngroups * 8 * TC_BM;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const float4 w = __ldcg(&src[((int64_t)g * 8 + c) * TC_BM + row]);
                        v[4 * c] += w.x;
                        v[4 * c + 1] += w.y;
                        v[4 * c + 2] += w.z;
                        v[4 * c + 3] += w.w;
                    }
                }
            }
            float av[16], bv[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                const float recv = __shfl_xor_sync(FULL, half ? v[t] : v[16 + t], 16);
                av[t] = half ? recv : v[t];
                bv[t] = half ? v[16 + t] : recv;
            }
            const int jt0 = 32 * g + 16 * half;
            const int tokf = o.tok0 + jt0, bif = tokf / sh.T;
            // every shared-memory read first (branch-free, so they overlap):
            // x of tokens jt0-1 .. jt0+15, and x_prev of each token's batch
            float xv[17], pv[16];
            xv[0] = jt0 == 0 ? lds_bf16(smem_u32(s_x0) + 2 * cl)
                             : lds_bf16(smem_u32(s_x) + (min(jt0, sh.BN) - 1) * 128 + 2 * cl);
            bool bstart[16];
            {
                int ti = tokf - bif * sh.T, bl = bif - o.bi0;
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const int jt = min(jt0 + t, sh.BN - 1);
                    xv[t + 1] = lds_bf16(smem_u32(s_x) + jt * 128 + 2 * cl);
                    bstart[t] = ti == 0;
                    pv[t] = lds_bf16(smem_u32(s_xp) + min(bl, sh.R - 1) * 128 + 2 * cl);
                    if (++ti == sh.T) {
                        ti = 0;
                        ++bl;
                    }
                }
            }
            // the 16 outputs of this lane into the group's output tile
            // [32 tokens][64 channels] bf16 (double-buffered by group)
            const uint32_t ob = so + (g & 1) * 4096 + (16 * half) * 128 + 2 * cl;
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                const float xc = xv[t + 1], xm = bstart[t] ? pv[t] : xv[t];
                sts_bf16(ob + t * 128, fmaf(bv[t], xm, fmaf(av[t], xc, xc)));
            }
            set_sync();
            // 16-byte rows out: item = (token, 8-channel group)
#pragma unroll
            for (int rep = 0; rep < 2; ++rep) {
                const int it = e + 128 * rep, tl = it >> 3, gg = it & 7;
                const int jt = 32 * g + tl, tok = o.tok0 + jt;
                if (jt < sh.BN && tok < sh.ntok)
                    *(uint4*)(out + (int64_t)tok * sh.H + o.h0 + 8 * gg) =
                        lds_v4(so + (g & 1) * 4096 + tl * 128 + 16 * gg);
            }
        }
    };
    // The run's last segment, if it owns its tile, has nothing after it: the
    // producer, MMA and allocation warps (0-3) then take the second half of
    // its groups, their output tile in the rings behind the staged partial.
    const int64_t last_tile = (s1 - 1) / sh.nkb;
    const uint32_t hso = part_bytes <= ring_bytes ? part_bytes : 0u;
    const bool helpers = s1 > s0 && s0 <= last_tile * sh.nkb && sh.ngroups >= 2 &&
                         hso + 8192u <= ring_bytes;
    const int gh = helpers ? (sh.ngroups + 1) / 2 : sh.ngroups;

    if ((warp == 0 || warp == 3) && lane == 0) {
        // ---------------- TMA producers, the run's steps in order: warp 0
        // the W tiles (HBM), warp 3 the X tiles (L2), each on its own ring
        const bool is_w = warp == 0;
        const int S = is_w ? sh.sw : sh.sx;
        const uint32_t full0 = is_w ? wfull0 : xfull0, empty0 = is_w ? wempty0 : xempty0;
        const uint32_t tx = is_w ? (uint32_t)TC_A_BYTES : (uint32_t)xstage;
        int i = 0;
        const int n = (int)(s1 - s0);
        for (; i < n; ++i) {
            const int st = i % S, r = i / S;
            if (r > 0 && !mbar_wait(empty0 + 8 * st, (r - 1) & 1)) {
                atomicOr(&g_dev_err, ERR_PRODUCER);
                break;
            }
            const int64_t step = s0 + i;
            const int tile = (int)(step / sh.nkb), kb = (int)(step - (int64_t)tile * sh.nkb);
            const int ct = tile / sh.nh, hb = tile - ct * sh.nh;
            mbar_expect_tx(full0 + 8 * st, tx);
            if (is_w && wpk) {
                // packed weights: the stage's 16 KB image, contiguous in memory
                bulk_g2s_nx(smem_u32(wring + st * TC_A_BYTES),
                            wpk + ((int64_t)hb * sh.nkb + kb) * TC_A_BYTES, (uint32_t)TC_A_BYTES,
                            full0 + 8 * st);
            } else if (is_w) {
                // one box of the 4-D view (k, 16 channels, a|b, 16-channel block):
                // accumulator rows 32q .. 32q+15 are a of channels h0+16q ..
                // h0+16q+15, rows 32q+16 .. 32q+31 are b of the same channels
                tma_load_4d(smem_u32(wring + st * TC_A_BYTES), &map_w, kb * TC_BK, 0, 0,
                            hb * TC_CH / 16, full0 + 8 * st);
            } else {
                tma_load_2d(smem_u32(xring + st * xstage), &map_x, kb * TC_BK, ct * TC_MAXN,
                            full0 + 8 * st);
            }
        }
        // drain: the last loads in flight have landed once their stages are
        // consumed (bounded; only a failed MMA thread leaves them pending)
        for (int k = (i > S ? i - S : 0); k < i; ++k) {
            const int st = k % S, r = k / S;
            if (!mbar_wait(empty0 + 8 * st, r & 1)) {
                atomicOr(&g_dev_err, ERR_DRAIN);
                break;
            }
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer: segment j accumulates in buffer j & 1
        const uint32_t idesc = instr_desc(TC_BM, sh.BN);
        int i = 0, j = 0;
        bool ok = true;
        for (int64_t sg = s0; sg < s1 && ok; ++j) {
            const int tile = (int)(sg / sh.nkb);
            const int klo = (int)(sg - (int64_t)tile * sh.nkb);
            const int khi = (int)min((int64_t)sh.nkb, s1 - (int64_t)tile * sh.nkb);
            const int buf = j & 1;
            if (j >= 2 && !mbar_wait(tempty0 + 8 * buf, ((j - 2) >> 1) & 1)) {
                atomicOr(&g_dev_err, ERR_MMA);
                break;
            }
            tc_fence_after();
            const uint32_t d = tmem + (uint32_t)(buf * sh.bufcols);
            for (int kb = klo; kb < khi; ++kb, ++i) {
                const int sw = i % sh.sw, sx = i % sh.sx;
                if (!mbar_wait(wfull0 + 8 * sw, (i / sh.sw) & 1) ||
                    !mbar_wait(xfull0 + 8 * sx, (i / sh.sx) & 1)) {
                    atomicOr(&g_dev_err, ERR_MMA);
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a = smem_u32(wring + sw * TC_A_BYTES);
                const uint32_t b = smem_u32(xring + sx * xstage);
#pragma unroll
                for (int kk = 0; kk < TC_BK / 16; ++kk)
                    mma_bf16(d, smem_desc(a + kk * 32), smem_desc(b + kk * 32), idesc,
                             (kb > klo || kk > 0) ? 1u : 0u);
                mma_commit(wempty0 + 8 * sw);
                mma_commit(xempty0 + 8 * sx);
            }
            if (ok) mma_commit(tfull0 + 8 * buf);
            sg = (int64_t)tile * sh.nkb + khi;
        }
        mma_commit(mdone);  // every MMA this thread issued has completed once this fires
    } else if (warp >= 4) {
        // ---------------- epilogue
        const int q = warp - 4;  // TMEM lanes 32q .. 32q + 31
        const int e = threadIdx.x - 128;
        const int row = 32 * q + lane;
        int j = 0, nown = 0, nstaged = 0;  // segments, owned segments, staged partials
        float4 pp0[8], pp1[8];  // the first partial, two groups ahead of its use
        for (int64_t sg = s0; sg < s1; ++j) {
            const int tile = (int)(sg / sh.nkb);
            const int klo = (int)(sg - (int64_t)tile * sh.nkb);
            const int khi = (int)min((int64_t)sh.nkb, s1 - (int64_t)tile * sh.nkb);
            sg = (int64_t)tile * sh.nkb + khi;
            const int buf = j & 1;
            const int ct = tile / sh.nh, hb = tile - ct * sh.nh;
            const int h0 = hb * TC_CH, tok0 = ct * TC_MAXN, bi0 = tok0 / sh.T;
            // runs that start inside an owned tile hand it partials (CTA order = K order)
            int q_end = p + 1;
            const float4* part1 = partial + (int64_t)(p + 1) * sh.ngroups * 8 * TC_BM;
            // the run's last segment: every load and MMA of this CTA is done by
            // the time its accumulator is, so the first partial can come into
            // the idle rings in one go; the next one is prefetched through
            // registers two groups ahead, any further ones read in place
            const bool will_stage = sg == s1 && part_bytes <= ring_bytes;
            const int q_reg = p + 1 + (will_stage ? 1 : 0);
            const float4* partr = partial + (int64_t)q_reg * sh.ngroups * 8 * TC_BM;
            auto load_part = [&](int g, float4 (&po)[8]) {
#pragma unroll
                for (int c = 0; c < 8; ++c) po[c] = __ldcg(&partr[((int64_t)g * 8 + c) * TC_BM + row]);
            };
            if (klo == 0) {
                // owned tile, while its MMAs run: stage its x rows, the x_prev
                // rows of the batches it touches and x of token tok0 - 1 in
                // shared memory (the previous owned tile's epilogue is done with
                // them), wait for the partials of later runs and request the
                // first two groups of the first one
                if (e == 0 && !*s_fail) {
                    mbar_expect_tx(xbar, (uint32_t)(sh.BN + sh.R) * 128u);
                    tma_load_2d(smem_u32(s_x), &map_xe, h0, tok0, xbar);
                    tma_load_2d(smem_u32(s_xp), &map_pe, h0, tok0 / sh.T, xbar);
                }
                if (e < 8 && tok0 > 0)
                    ((uint4*)s_x0)[e] = *(const uint4*)(x + (int64_t)(tok0 - 1) * sh.H + h0 + 8 * e);
                while (q_end < sh.nctas && run_start(sh, q_end) < (int64_t)(tile + 1) * sh.nkb) ++q_end;
                if (e == 0) {
                    for (int q2 = p + 1; q2 < q_end && !*s_fail; ++q2) {
                        const uint64_t t0 = global_ns();
                        while (ld_acquire(&flags[q2]) == 0u) {
                            if (global_ns() - t0 > WAIT_NS) {
                                atomicOr(&g_dev_err, ERR_EPILOGUE);
                                *s_fail = 1;
                                break;
                            }
                        }
                        if (!*s_fail) flags[q2] = 0u;  // consumed: leave the flag zero
                    }
                    __threadfence();
                }
                epi_sync();
                if (!*s_fail && q_end > q_reg) {
                    load_part(0, pp0);
                    if (sh.ngroups > 1) load_part(1, pp1);
                }
            }
            if (!mbar_wait(tfull0 + 8 * buf, (j >> 1) & 1)) {
                atomicOr(&g_dev_err, ERR_EPILOGUE);
                *s_fail = 1;
            }
            epi_sync();
            if (*s_fail) break;  // uniform over the four warps
            tc_fence_after();
            const uint32_t tacc = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * sh.bufcols);
            if (klo > 0) {
                // a run that starts inside the tile: hand the partial to its owner
                float4* dst = partial + (int64_t)p * sh.ngroups * 8 * TC_BM;
                for (int g = 0; g < sh.ngroups; ++g) {
                    float v[32];
                    tmem_ld32(tacc + 32 * g, v);
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        dst[((int64_t)g * 8 + c) * TC_BM + row] =
                            make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
                }
                tc_fence_before();
                epi_sync();
                if (e == 0) {
                    __threadfence();
                    st_release(&flags[p], 1u);
                    mbar_arrive(tempty0 + 8 * buf);
                }
                continue;
            }
            if (!mbar_wait(xbar, (uint32_t)(nown & 1))) {  // the staged x, x_prev rows
                atomicOr(&g_dev_err, ERR_EPILOGUE);
                *s_fail = 1;
            }
            ++nown;
            const bool first_part = *s_fail == 0 && q_end > p + 1;
            const bool staged = first_part && will_stage;
            const bool reg_part = *s_fail == 0 && q_end > q_reg;
            if (staged) {
                if (e == 0) {  // 32 KB pieces into the rings (free: all MMAs are done)
                    mbar_expect_tx(pbar, part_bytes);
                    for (uint32_t off = 0; off < part_bytes; off += 32768u)
                        bulk_g2s_nx(smem_u32(wring) + off, (const char*)part1 + off,
                                    min(32768u, part_bytes - off), pbar);
                }
                if (!mbar_wait(pbar, (uint32_t)(nstaged & 1))) {
                    atomicOr(&g_dev_err, ERR_EPILOGUE);
                    *s_fail = 1;
                }
                ++nstaged;
            }
            epi_sync();
            if (*s_fail) break;  // uniform over the four warps
            OwnTile o;
            o.tacc = tmem + (uint32_t)(buf * sh.bufcols);
            o.h0 = h0;
            o.tok0 = tok0;
            o.bi0 = bi0;
            o.q_reg = q_reg;
            o.q_end = q_end;
            o.staged = staged;
            o.reg_part = reg_part;
            o.first_part = first_part;
            const bool helped = helpers && sg == s1;
            if (helped && e == 0) {  // hand the second half of the groups to warps 0-3
                s_own = o;
                mbar_arrive(hbar);
            }
            own_groups(o, 0, helped ? gh : sh.ngroups, smem_u32(s_out), 1, pp0, pp1);
            tc_fence_before();
            epi_sync();
            if (e == 0) mbar_arrive(tempty0 + 8 * buf);
        }
    }
    if (warp < 4 && helpers) {
        __syncwarp();  // lane 0 of warps 0, 1 and 3 is back from its role
        if (!mbar_wait(hbar, 0)) {
            if (lane == 0) atomicOr(&g_dev_err, ERR_EPILOGUE);
        } else {
            tc_fence_after();
            const OwnTile o = s_own;
            float4 pp0[8], pp1[8];
            if (o.reg_part) {
                const float4* partr = partial + (int64_t)o.q_reg * sh.ngroups * 8 * TC_BM;
                const int row = 32 * warp + lane;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    pp0[c] = __ldcg(&partr[((int64_t)gh * 8 + c) * TC_BM + row]);
                    if (gh + 1 < sh.ngroups)
                        pp1[c] = __ldcg(&partr[((int64_t)(gh + 1) * 8 + c) * TC_BM + row]);
                }
            }
            own_groups(o, gh, sh.ngroups, smem_u32(wring) + hso, 2, pp0, pp1);
            tc_fence_before();
        }
    }
    __syncthreads();
    if (warp == 2) {
        // every MMA has completed before TMEM goes back (bounded)
        if (!mbar_wait(mdone, 0)) atomicOr(&g_dev_err, ERR_DRAIN);
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols));
    }
}

}  // namespace dfl

// ---------------------------------------------------------------------------
// Host side: tensor maps through the driver entry point (no link-time
// dependency on libcuda), shape planning and launch.
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
    }
    return fn;
}

bool make_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows, uint32_t box_inner,
              uint32_t box_rows, bool swizzle = true) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// W_tap [2H, H] seen as (k, r, ab, blk): row = ab * H + 16 * blk + r; one box
// (64, 16, 2, 4) is a 64-channel tile with a and b rows interleaved in
// 16-row runs, 128-byte swizzle.
bool make_wmap(CUtensorMap* m, const void* w, int H) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const uint64_t rb = (uint64_t)H * 2;  // bytes per W row
    cuuint64_t dims[4] = {(cuuint64_t)H, 16, 2, (cuuint64_t)H / 16};
    cuuint64_t strides[3] = {rb, rb * H, rb * 16};
    cuuint32_t box[4] = {64, 16, 2, 4};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(w), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Stream-K plan of one call: token chunks of up to 256 (the accumulator
// width), 64-channel tiles, 64-wide K blocks; one CTA per SM (at most
// TC_MAXCTA) and never more CTAs than steps.
struct TcPlan {
    int BN, ngroups, bufcols, nh, nkb, nctas;
    int64_t steps;
    size_t flags_bytes, part_bytes;
};
static TcPlan tc_plan(int64_t ntok, int H, int sms) {
    using namespace dfl;
    TcPlan P;
    const int64_t nt = (ntok + TC_MAXN - 1) / TC_MAXN;
    const int64_t chunk_tok = nt > 1 ? TC_MAXN : ntok;
    P.BN = (int)(((chunk_tok + 15) / 16) * 16);
    P.ngroups = (P.BN + 31) / 32;
    P.bufcols = 32;
    while (P.bufcols < P.BN) P.bufcols *= 2;
    P.nh = H / TC_CH;
    P.nkb = H / TC_BK;
    P.steps = nt * P.nh * P.nkb;
    P.nctas = (int)std::min<int64_t>(std::min(sms, TC_MAXCTA), P.steps);
    // flags in the workspace's control area (zero between calls: each owner
    // resets the flags it consumed), partials after it
    P.flags_bytes = dfl::CONTROL_BYTES;
    P.part_bytes = (size_t)P.nctas * P.ngroups * 8 * TC_BM * sizeof(float4);
    return P;
}

// Workspace of the bf16 path, sized for TC_MAXCTA CTAs so that it does not
// depend on the device.
size_t dflash2_dynconv2_tc_workspace(int64_t ntok, int H) {
    const TcPlan P = tc_plan(ntok, H, dfl::TC_MAXCTA);
    return P.flags_bytes + P.part_bytes;
}

// Launches the tensor-core path for bf16 operands (H a multiple of 64,
// 16-byte aligned pointers and a large enough 256-byte aligned workspace,
// checked by the caller).  Returns a dflash2 status.
int dflash2_dynconv2_tc_launch(const void* x, const void* x_prev, const void* w_tap, int B, int T,
                               int H, void* out, void* ws, cudaStream_t s, const void* w_packed) {
    using namespace dfl;
    const int ntok = B * T;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return DFLASH2_ECUDA;
    const TcPlan P = tc_plan(ntok, H, sms);
    CUtensorMap mw, mx;
    // (with packed weights the map is built over the packed buffer, which has
    // the same size, and never used)
    if (!make_wmap(&mw, w_packed ? w_packed : w_tap, H)) return DFLASH2_ECUDA;
    if (!make_map(&mx, x, (uint64_t)H, (uint64_t)ntok, TC_BK, (uint32_t)P.BN)) return DFLASH2_ECUDA;
    // epilogue staging: an owned tile's x rows and the x_prev rows of the
    // (at most R) batches its tokens belong to, 128 bytes per row, unswizzled
    const int R = std::min(B, (P.BN - 1 + T - 1) / T + 1);
    CUtensorMap mxe, mpe;
    if (!make_map(&mxe, x, (uint64_t)H, (uint64_t)ntok, TC_CH, (uint32_t)P.BN, false) ||
        !make_map(&mpe, x_prev, (uint64_t)H, (uint64_t)B, TC_CH, (uint32_t)R, false))
        return DFLASH2_ECUDA;
    // W ring (HBM, ~2 us loaded latency) deeper than the X ring (L2): three X
    // stages (four when they are small), the rest of 227 KB for W, at most 8
    const int xstage = P.BN * TC_BK * 2;
    const int fixed = 1024 + (P.BN + R + 1) * 128 + 8192 + 96 * 8 + 16;
    const int sx = xstage <= 16384 ? 4 : 3;
    int sw = (227 * 1024 - fixed - sx * xstage) / TC_A_BYTES;
    sw = sw > 8 ? 8 : sw;
    if (sw < 2) return DFLASH2_ESHAPE;
    const int smem = fixed + sw * TC_A_BYTES + sx * xstage;
    {
        static std::mutex mu;
        static bool attr_set[64] = {};
        std::lock_guard<std::mutex> g(mu);
        if (dev < 64 && !attr_set[dev]) {
            if (cudaFuncSetAttribute(dynconv2_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     227 * 1024) != cudaSuccess)
                return DFLASH2_ECUDA;
            attr_set[dev] = true;
        }
    }
    unsigned* flags = (unsigned*)ws;
    float4* part = (float4*)((char*)ws + P.flags_bytes);
    TcShape sh{H, T, ntok, P.BN, sw, sx, P.nkb, P.nh, P.bufcols, P.ngroups, P.nctas, R, P.steps};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)P.nctas);
    cfg.blockDim = dim3(TC_THREADS);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    // cooperative: every CTA is resident, so an owner's bounded wait for a
    // later CTA's partial always has a running producer
    cudaLaunchAttribute a[1];
    a[0].id = cudaLaunchAttributeCooperative;
    a[0].val.cooperative = 1;
    cfg.attrs = a;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, dynconv2_tc_kernel, mw, mx, mxe, mpe, (const __nv_bfloat16*)x,
                           (const __nv_bfloat16*)x_prev, (__nv_bfloat16*)out, sh, part,
                           flags, (const uint8_t*)w_packed) != cudaSuccess)
        return DFLASH2_ECUDA;
    return DFLASH2_OK;
}

namespace dfl {
// W_tap [2H, H] bf16 (nn.Linear layout) rewritten as the W stages of the
// tensor-core kernel: block (hb, kb), hb = 64-channel block, kb = 64-wide K
// block, at byte (hb * H/64 + kb) * 16 KB holds the 128 x 64 tile the
// producer's 4-D box brings in -- row 32 q + 16 ab + ch is channel
// 64 hb + 16 q + ch of W_a (ab = 0) or W_b (ab = 1), its 64 K elements in
// 16-byte chunks placed by the 128-byte swizzle (chunk c of row r at chunk
// c ^ (r mod 8)).  One CTA per block, four 16-byte chunks per thread.
__global__ void __launch_bounds__(256) dynconv2_pack_kernel(const uint4* __restrict__ w, int H,
                                                            uint4* __restrict__ packed) {
    const int nkb = H / TC_BK;
    const int blk = blockIdx.x, hb = blk / nkb, kb = blk - hb * nkb;
    const int rowv = H / 8;  // 16-byte vectors per W_tap row
    for (int qi = threadIdx.x; qi < TC_A_BYTES / 16; qi += blockDim.x) {
        const int r = qi >> 3, c = qi & 7;
        const int q = r >> 5, ab = (r >> 4) & 1, ch = r & 15;
        const int64_t g = (int64_t)ab * H + (int64_t)hb * TC_CH + q * 16 + ch;
        packed[(int64_t)blk * (TC_A_BYTES / 16) + r * 8 + (c ^ (r & 7))] =
            __ldg(&w[g * rowv + kb * (TC_BK / 8) + c]);
    }
}
}  // namespace dfl

int dflash2_dynconv2_tc_pack(const void* w_tap, int H, void* packed, cudaStream_t s) {
    using namespace dfl;
    const int blocks = (H / TC_CH) * (H / TC_BK);
    dynconv2_pack_kernel<<<blocks, 256, 0, s>>>((const uint4*)w_tap, H, (uint4*)packed);
    return cudaGetLastError() == cudaSuccess ? DFLASH2_OK : DFLASH2_ECUDA;
}

unsigned dfl_errors_dynconv(int clear) {
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, dfl::g_dev_err, sizeof v) != cudaSuccess) return 0xFFFFFFFFu;
    if (clear && v) {
        unsigned z = 0;
        cudaMemcpyToSymbol(dfl::g_dev_err, &z, sizeof z);
    }
    return v;
}
