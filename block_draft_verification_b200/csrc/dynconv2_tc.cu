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
// the N = B*T tokens.  A CTA owns 64 output channels h0..h0+63: its M = 128
// tile stacks the 64 W_a rows and the 64 matching W_b rows, so a and b of a
// channel meet in one accumulator and the conv, the residual and the rounding
// run in the epilogue straight out of tensor memory.
//   warp 0   TMA producer: W tile (2 boxes of 64 x 64) + X tile (N x 64) per
//            64-wide K block into a ring of shared-memory stages (128-byte
//            swizzle), one mbarrier pair per stage
//   warp 1   MMA issuer: one thread issues tcgen05.mma (M=128, N, K=16) x 4
//            per K block, accumulating in TMEM; tcgen05.commit frees stages
//   warp 2   TMEM allocation / release
//   warps 4-7 epilogue: tcgen05.ld of their 32 TMEM lanes into shared
//            memory, then (token, 8-channel) items: 16-byte loads of x_t and
//            x_{t-1}, conv + residual, one 16-byte bf16 store
// Every mbarrier wait is bounded (one second, stream.cuh); on a timeout the
// kernel records a flag (dflash2_device_errors), stops issuing work, releases
// TMEM and returns.  No TMA load here uses cluster multicast.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "stream.cuh"

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
// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes, 8-row groups 1024 bytes apart (stride byte offset), version 1.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor, kind::f16: fp32 accumulate, bf16 A and B, both
// K-major, N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t instr_desc(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// 32 lanes x 32 consecutive fp32 columns: thread = lane, v[j] = column j.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
}

struct TcShape {
    int H, T, ntok, tok0, BN, stages, nkb;
};

__global__ void __launch_bounds__(TC_THREADS, 1) dynconv2_tc_kernel(
    const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ x_prev,
    __nv_bfloat16* __restrict__ out, TcShape sh) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // stage ring, 1024-byte aligned for the 128-byte swizzle
    uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int stage_bytes = TC_A_BYTES + sh.BN * TC_BK * 2;
    uint8_t* tail = base + sh.stages * stage_bytes;
    float* s_acc = (float*)tail;                                // [128][33] a, b values
    uint64_t* bars = (uint64_t*)(tail + TC_BM * 33 * 4);        // full[S], empty[S], accf
    uint32_t* s_tmem = (uint32_t*)(bars + 2 * sh.stages + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h0 = blockIdx.x * TC_CH;
    const int tok0 = sh.tok0 + blockIdx.y * TC_MAXN;
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + sh.stages);
    const uint32_t accf = smem_u32(bars + 2 * sh.stages);
    const uint32_t ncols = sh.BN <= 32 ? 32 : (sh.BN <= 64 ? 64 : (sh.BN <= 128 ? 128 : 256));

    if (threadIdx.x == 0) {
        for (int s = 0; s < sh.stages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        mbar_init(accf, 1);
        mbar_fence_init();
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

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer
        const uint32_t tx = TC_A_BYTES + sh.BN * TC_BK * 2;
        int kb = 0;
        for (; kb < sh.nkb; ++kb) {
            const int s = kb % sh.stages, r = kb / sh.stages;
            if (r > 0 && !mbar_wait(empty0 + 8 * s, (r - 1) & 1)) {
                atomicOr(&g_dev_err, ERR_PRODUCER);
                break;
            }
            const uint32_t a = smem_u32(base + s * stage_bytes);
            const uint32_t b = a + TC_A_BYTES;
            mbar_expect_tx(full0 + 8 * s, tx);
            // each CTA starts its K walk at its own offset, so the CTAs do
            // not all request the same token tile from L2 at the same time
            const int kp = (kb + blockIdx.x * 7) % sh.nkb;
            tma_load_2d(a, &map_w, kp * TC_BK, h0, full0 + 8 * s);
            tma_load_2d(a + TC_A_BYTES / 2, &map_w, kp * TC_BK, sh.H + h0, full0 + 8 * s);
            tma_load_2d(b, &map_x, kp * TC_BK, tok0, full0 + 8 * s);
        }
        // drain: the last loads in flight have landed once their stages are
        // consumed (bounded; only a failed MMA thread leaves them pending)
        for (int k = (kb > sh.stages ? kb - sh.stages : 0); k < kb; ++k) {
            const int s = k % sh.stages, r = k / sh.stages;
            if (!mbar_wait(empty0 + 8 * s, r & 1)) {
                atomicOr(&g_dev_err, ERR_DRAIN);
                break;
            }
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer
        const uint32_t idesc = instr_desc(TC_BM, sh.BN);
        for (int kb = 0; kb < sh.nkb; ++kb) {
            const int s = kb % sh.stages, r = kb / sh.stages;
            if (!mbar_wait(full0 + 8 * s, r & 1)) {
                atomicOr(&g_dev_err, ERR_MMA);
                break;
            }
            tc_fence_after();
            const uint32_t a = smem_u32(base + s * stage_bytes);
            const uint32_t b = a + TC_A_BYTES;
#pragma unroll
            for (int kk = 0; kk < TC_BK / 16; ++kk)
                mma_bf16(tmem, smem_desc(a + kk * 32), smem_desc(b + kk * 32), idesc,
                         (kb > 0 || kk > 0) ? 1u : 0u);
            mma_commit(empty0 + 8 * s);
        }
        mma_commit(accf);
    } else if (warp >= 4) {
        // ---------------- epilogue: 32 token columns at a time, TMEM -> shared
        // (a in rows 0..63, b in rows 64..127), then each thread takes
        // (token, 8-channel group) items with 16-byte loads of x_t and x_{t-1}
        // and one 16-byte store of the 8 outputs.
        const int q = warp - 4;  // TMEM lanes 32q .. 32q + 31
        const int e = threadIdx.x - 128;
        bool ok = mbar_wait(accf, 0);
        if (!ok) atomicOr(&g_dev_err, ERR_EPILOGUE);
        ok = __all_sync(FULL, ok);  // tcgen05.ld is warp-collective
        tc_fence_after();
        for (int c0 = 0; c0 < sh.BN; c0 += 32) {
            if (ok) {
                float v[32];
                tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
#pragma unroll
                for (int j = 0; j < 32; ++j) s_acc[(32 * q + lane) * 33 + j] = v[j];
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (ok) {
#pragma unroll
                for (int rep = 0; rep < 2; ++rep) {
                    const int it = e + 128 * rep;
                    const int j = it >> 3, g = it & 7;
                    const int tok = tok0 + c0 + j;
                    if (tok < sh.ntok) {
                        const int h = h0 + 8 * g;
                        const int bi = tok / sh.T;
                        const uint4 xv = *(const uint4*)(x + (int64_t)tok * sh.H + h);
                        const uint4 pv = (tok == bi * sh.T)
                                             ? *(const uint4*)(x_prev + (int64_t)bi * sh.H + h)
                                             : *(const uint4*)(x + (int64_t)(tok - 1) * sh.H + h);
                        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                        const uint32_t pw[4] = {pv.x, pv.y, pv.z, pv.w};
                        uint32_t ow[4];
#pragma unroll
                        for (int c = 0; c < 8; c += 2) {
                            float y2[2];
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                const uint32_t xb = (u ? (xw[c >> 1] & 0xFFFF0000u) : (xw[c >> 1] << 16));
                                const uint32_t pb = (u ? (pw[c >> 1] & 0xFFFF0000u) : (pw[c >> 1] << 16));
                                const float xc = __uint_as_float(xb), xp = __uint_as_float(pb);
                                const float a = s_acc[(8 * g + c + u) * 33 + j];
                                const float b = s_acc[(64 + 8 * g + c + u) * 33 + j];
                                y2[u] = fmaf(b, xp, fmaf(a, xc, xc));
                            }
                            const __nv_bfloat162 pr = __floats2bfloat162_rn(y2[0], y2[1]);
                            ow[c >> 1] = *(const uint32_t*)&pr;
                        }
                        *(uint4*)(out + (int64_t)tok * sh.H + h) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                    }
                }
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
        }
        tc_fence_before();
    }
    __syncthreads();
    if (warp == 2) {
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
              uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Launches the tensor-core path for bf16 operands (H a multiple of 64,
// 16-byte aligned pointers, checked by the caller).  Returns a dflash2 status.
int dflash2_dynconv2_tc_launch(const void* x, const void* x_prev, const void* w_tap, int B, int T,
                               int H, void* out, cudaStream_t s) {
    using namespace dfl;
    const int ntok = B * T;
    CUtensorMap mw, mx;
    const int n_chunks_tok = (ntok + TC_MAXN - 1) / TC_MAXN;
    const int chunk_tok = n_chunks_tok > 1 ? TC_MAXN : ntok;
    const int BN = ((chunk_tok + 15) / 16) * 16;
    if (!make_map(&mw, w_tap, (uint64_t)H, (uint64_t)2 * H, TC_BK, TC_CH)) return DFLASH2_ECUDA;
    if (!make_map(&mx, x, (uint64_t)H, (uint64_t)ntok, TC_BK, (uint32_t)BN)) return DFLASH2_ECUDA;
    const int stage_bytes = TC_A_BYTES + BN * TC_BK * 2;
    const int fixed = 1024 + TC_BM * 33 * 4 + 64 * 8 + 16;
    int stages = (227 * 1024 - fixed) / stage_bytes;
    stages = stages > 8 ? 8 : stages;
    if (stages < 2) return DFLASH2_ESHAPE;
    const int smem = fixed + stages * stage_bytes;
    static bool attr_set = false;
    if (!attr_set) {
        if (cudaFuncSetAttribute(dynconv2_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 227 * 1024) != cudaSuccess)
            return DFLASH2_ECUDA;
        attr_set = true;
    }
    TcShape sh{H, T, ntok, 0, BN, stages, H / TC_BK};
    dim3 grid((unsigned)(H / TC_CH), (unsigned)n_chunks_tok);
    dynconv2_tc_kernel<<<grid, TC_THREADS, smem, s>>>(mw, mx, (const __nv_bfloat16*)x,
                                                      (const __nv_bfloat16*)x_prev,
                                                      (__nv_bfloat16*)out, sh);
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
