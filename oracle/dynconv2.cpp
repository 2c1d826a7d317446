/*
 * dynconv2.cpp -- the two-tap dynamic depthwise convolution with its per-token
 * tap projection and the residual add.
 * TEST INFRASTRUCTURE ONLY (see oracle.h).
 *
 * Source: [tamsi] "L’idée, sans le papier" -- a two-tap convolution (Canon /
 * short-conv style) before and after each attention and MLP counters suffix
 * decay; [myaiexp] "主な機能" -- a 2-tap dynamic convolution.  The pages give
 * no formula; the form here is the plainest dynamic two-tap depthwise conv:
 *
 *   a_t = W_a x_t,  b_t = W_b x_t      (W_tap = [W_a; W_b], shape [2H, H],
 *                                       row h of W_a is row h of W_tap, row h
 *                                       of W_b is row H + h)
 *   y_t = a_t * x_t + b_t * x_{t-1}    (elementwise; x_{-1} = x_prev)
 *   out_t = x_t + y_t
 * No bias and no gate; a_t and b_t stay unrounded until the output.
 * Layouts: x [B, T, H], x_prev [B, H], w_tap [2H, H], out [B, T, H].
 */
#include "oracle_util.h"

extern "C" int orc_dynconv2(const void* x, const void* x_prev, const void* w_tap, int dtype,
                            int B, int T, int H, double* out) {
    if (!x || !x_prev || !w_tap || !out || !orc_dtype_ok(dtype) || B < 0 || T < 0 || H < 1)
        return -1;
    for (int b = 0; b < B; ++b) {
        for (int t = 0; t < T; ++t) {
            int64_t xt = ((int64_t)b * T + t) * H;
            for (int h = 0; h < H; ++h) {
                double a = 0.0, bb = 0.0;
                for (int k = 0; k < H; ++k) {
                    double xk = orc_load(x, dtype, xt + k);
                    a += orc_load(w_tap, dtype, (int64_t)h * H + k) * xk;
                    bb += orc_load(w_tap, dtype, ((int64_t)H + h) * H + k) * xk;
                }
                double xcur = orc_load(x, dtype, xt + h);
                double xprev = (t == 0) ? orc_load(x_prev, dtype, (int64_t)b * H + h)
                                        : orc_load(x, dtype, xt - H + h);
                out[xt + h] = xcur + a * xcur + bb * xprev;
            }
        }
    }
    return 0;
}
