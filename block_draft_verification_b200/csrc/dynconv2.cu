// dynconv2.cu -- two-tap dynamic depthwise convolution fused with its
// per-token tap projection and the residual add.
//
// Sources: "DFlash 2 — 3× plus de tokens sur Qwen3.8-27B, même sortie"
// (tamsi.dev), section "L’idée, sans le papier": a two-tap convolution in the
// Canon / short-conv style before and after each attention and MLP, to stop
// the end of the block from decaying; "DFlash 2" (myaiexp.com), section
// "主な機能": a 2-tap dynamic convolution.  The form:
//   [a_t; b_t] = W_tap x_t           (W_tap [2H, H], nn.Linear layout)
//   out_t = x_t + a_t * x_t + b_t * x_{t-1},   x_{-1} = x_prev
//
// fp32 operands take the SIMT path here: one warp per (output channel h,
// block of 8 tokens) streams the two weight rows h and H + h with 128-bit
// loads and dots them with the 8 token vectors, fp32 accumulation, then
// applies the conv and residual in the epilogue.  bf16 operands take the
// tensor-core path of dynconv2_tc.cu.
#include <cuda_bf16.h>

#include "common.cuh"

namespace dfl {

constexpr int DC_TOK = 8;  // tokens per warp

template <bool BF16>
__device__ __forceinline__ float ld_elem(const void* p, int64_t i) {
    if (BF16) return __uint_as_float((uint32_t)__ldg((const unsigned short*)p + i) << 16);
    return __ldg((const float*)p + i);
}

template <bool BF16>
__global__ void __launch_bounds__(NT) dynconv2_simt_kernel(const void* __restrict__ x,
                                                           const void* __restrict__ x_prev,
                                                           const void* __restrict__ w, int T, int H,
                                                           int ntok, void* __restrict__ out) {
    using R = Row<BF16>;
    const int lane = threadIdx.x & 31;
    const int64_t gw = (int64_t)blockIdx.x * (NT / 32) + (threadIdx.x >> 5);
    const int ntb = (ntok + DC_TOK - 1) / DC_TOK;
    const int64_t h = gw / ntb;
    const int tb = (int)(gw - h * ntb);
    if (h >= H) return;
    const int tok0 = tb * DC_TOK;
    const int nt = min(DC_TOK, ntok - tok0);
    const char* wa = (const char*)w + h * H * (BF16 ? 2 : 4);
    const char* wb = (const char*)w + ((int64_t)H + h) * H * (BF16 ? 2 : 4);

    float acc_a[DC_TOK], acc_b[DC_TOK];
#pragma unroll
    for (int q = 0; q < DC_TOK; ++q) acc_a[q] = acc_b[q] = 0.0f;
    // H is a multiple of 64: every lane takes whole 16-byte vectors
    for (int k0 = lane * R::VW; k0 < H; k0 += 32 * R::VW) {
        const uint4 va = *(const uint4*)(wa + (int64_t)k0 * (BF16 ? 2 : 4));
        const uint4 vb = *(const uint4*)(wb + (int64_t)k0 * (BF16 ? 2 : 4));
#pragma unroll
        for (int q = 0; q < DC_TOK; ++q) {
            if (q < nt) {
                const uint4 vx = *(const uint4*)((const char*)x +
                                                 ((int64_t)(tok0 + q) * H + k0) * (BF16 ? 2 : 4));
#pragma unroll
                for (int e = 0; e < R::VW; ++e) {
                    const float xv = R::elem(vx, e);
                    acc_a[q] = fmaf(R::elem(va, e), xv, acc_a[q]);
                    acc_b[q] = fmaf(R::elem(vb, e), xv, acc_b[q]);
                }
            }
        }
    }
#pragma unroll
    for (int q = 0; q < DC_TOK; ++q)
#pragma unroll
        for (int j = 16; j > 0; j >>= 1) {
            acc_a[q] += __shfl_xor_sync(FULL, acc_a[q], j);
            acc_b[q] += __shfl_xor_sync(FULL, acc_b[q], j);
        }
    if (lane < nt) {
        float a = 0.0f, bb = 0.0f;
#pragma unroll
        for (int q = 0; q < DC_TOK; ++q)
            if (q == lane) {
                a = acc_a[q];
                bb = acc_b[q];
            }
        const int tok = tok0 + lane;
        const int bi = tok / T, ti = tok - bi * T;
        const float xc = ld_elem<BF16>(x, (int64_t)tok * H + h);
        const float xp = (ti == 0) ? ld_elem<BF16>(x_prev, (int64_t)bi * H + h)
                                   : ld_elem<BF16>(x, (int64_t)(tok - 1) * H + h);
        const float y = fmaf(bb, xp, fmaf(a, xc, xc));
        if (BF16)
            ((__nv_bfloat16*)out)[(int64_t)tok * H + h] = __float2bfloat16_rn(y);
        else
            ((float*)out)[(int64_t)tok * H + h] = y;
    }
}

}  // namespace dfl

using namespace dfl;
using namespace dfl_host;

int dflash2_dynconv2_tc_launch(const void* x, const void* x_prev, const void* w_tap, int B, int T,
                               int H, void* out, void* ws, cudaStream_t s, const void* w_packed);
int dflash2_dynconv2_tc_pack(const void* w_tap, int H, void* packed, cudaStream_t s);
size_t dflash2_dynconv2_tc_workspace(int64_t ntok, int H);

static bool dynconv_shape_ok(int B, int T, int H) {
    return B >= 0 && T >= 0 && H >= 64 && H % 64 == 0 && (int64_t)B * T <= (int64_t)INT32_MAX / 2;
}

extern "C" size_t dflash2_dynconv2_workspace_bytes(int dtype, int B, int T, int H) {
    if (!dtype_ok(dtype) || !dynconv_shape_ok(B, T, H)) return 0;
    if (dtype != DFLASH2_BF16 || (int64_t)B * T == 0) return 0;
    return dflash2_dynconv2_tc_workspace((int64_t)B * T, H);
}

extern "C" int dflash2_dynconv2(const void* x, const void* x_prev, const void* w_tap, int dtype,
                                int B, int T, int H, void* out, void* ws, size_t ws_bytes,
                                dflash2_stream_t stream) {
    if (!dtype_ok(dtype)) return DFLASH2_EDTYPE;
    if (!dynconv_shape_ok(B, T, H)) return DFLASH2_ESHAPE;
    if ((int64_t)B * T == 0) return DFLASH2_OK;
    if (!x || !x_prev || !w_tap || !out) return DFLASH2_EINVAL;
    if (!aligned(x, 16) || !aligned(x_prev, 16) || !aligned(w_tap, 16) || !aligned(out, 16))
        return DFLASH2_EALIGN;
    const int64_t ntok = (int64_t)B * T;
    const int64_t warps = (int64_t)H * ((ntok + DC_TOK - 1) / DC_TOK);
    const int64_t blocks = (warps + NT / 32 - 1) / (NT / 32);
    if (blocks > (int64_t)INT32_MAX) return DFLASH2_ESHAPE;
    const size_t need = dflash2_dynconv2_workspace_bytes(dtype, B, T, H);
    if (need > 0 && (!ws || !aligned(ws, 256) || ws_bytes < need)) return DFLASH2_EWORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    if (dtype == DFLASH2_BF16)  // tensor cores (tcgen05 + TMA), dynconv2_tc.cu
        return dflash2_dynconv2_tc_launch(x, x_prev, w_tap, B, T, H, out, ws, s, nullptr);
    dynconv2_simt_kernel<false><<<(unsigned)blocks, NT, 0, s>>>(x, x_prev, w_tap, T, H, (int)ntok,
                                                                out);
    return launch_status();
}

extern "C" size_t dflash2_dynconv2_packed_bytes(int dtype, int H) {
    if (dtype != DFLASH2_BF16 || !dynconv_shape_ok(0, 0, H)) return 0;
    return (size_t)4 * H * H;
}

extern "C" int dflash2_dynconv2_pack(const void* w_tap, int dtype, int H, void* w_packed,
                                     dflash2_stream_t stream) {
    if (dtype != DFLASH2_BF16) return DFLASH2_EDTYPE;  // the packed form feeds the tensor cores
    if (!dynconv_shape_ok(0, 0, H)) return DFLASH2_ESHAPE;
    if (!w_tap || !w_packed) return DFLASH2_EINVAL;
    if (!aligned(w_tap, 16) || !aligned(w_packed, 256)) return DFLASH2_EALIGN;
    return dflash2_dynconv2_tc_pack(w_tap, H, w_packed, (cudaStream_t)stream);
}

extern "C" int dflash2_dynconv2_packed(const void* x, const void* x_prev, const void* w_packed,
                                       int dtype, int B, int T, int H, void* out, void* ws,
                                       size_t ws_bytes, dflash2_stream_t stream) {
    if (dtype != DFLASH2_BF16) return DFLASH2_EDTYPE;
    if (!dynconv_shape_ok(B, T, H)) return DFLASH2_ESHAPE;
    if ((int64_t)B * T == 0) return DFLASH2_OK;
    if (!x || !x_prev || !w_packed || !out) return DFLASH2_EINVAL;
    if (!aligned(x, 16) || !aligned(x_prev, 16) || !aligned(w_packed, 256) || !aligned(out, 16))
        return DFLASH2_EALIGN;
    const size_t need = dflash2_dynconv2_workspace_bytes(dtype, B, T, H);
    if (!ws || !aligned(ws, 256) || ws_bytes < need) return DFLASH2_EWORKSPACE;
    return dflash2_dynconv2_tc_launch(x, x_prev, nullptr, B, T, H, out, ws, (cudaStream_t)stream,
                                      w_packed);
}
