/*
 * topk_softmax.cpp -- per drafted position: the vocab-wide softmax of the
 * drafter logits and the 16 best candidates.
 * TEST INFRASTRUCTURE ONLY (see oracle.h).
 *
 * Source: [tamsi] "L’idée, sans le papier" -- the right token sits in the
 * drafter's top 16 far more often than at top 1, and the selector chooses
 * among those 16 per position; [myaiexp] "主な機能" -- the path selector keeps
 * the top-16 candidates of each position.
 *
 * For each row r (row pointer = logits + r * row_stride):
 *   z_v    = x_v * inv_temperature                      (double)
 *   m      = max_v z_v
 *   logz   = m + log(sum_v exp(z_v - m))                (ascending v)
 *   order  = all v sorted by (x_v descending, v ascending); x is compared as
 *            a value, so -0 and +0 are equal and fall back to the index
 *   idx[k] = order[k] for k < 16
 *   prob_k = exp(z_idx[k] - logz),  logp_k = z_idx[k] - logz
 */
#include <math.h>

#include <algorithm>
#include <vector>

#include "oracle_util.h"

extern "C" int orc_topk_softmax(const void* logits, int dtype, int64_t rows, int64_t V,
                                int64_t row_stride, double inv_temperature, int32_t* idx,
                                double* prob, double* logp, double* logz) {
    if (!logits || !orc_dtype_ok(dtype) || rows < 0 || V < ORC_K || row_stride < V ||
        !(inv_temperature > 0.0))
        return -1;
    std::vector<double> x((size_t)V), z((size_t)V);
    std::vector<int32_t> order((size_t)V);
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t v = 0; v < V; ++v) {
            x[v] = orc_load(logits, dtype, r * row_stride + v);
            z[v] = x[v] * inv_temperature;
        }
        double m = z[0];
        for (int64_t v = 1; v < V; ++v) m = std::max(m, z[v]);
        double s = 0.0;
        for (int64_t v = 0; v < V; ++v) s += exp(z[v] - m);
        double lz = m + log(s);

        for (int64_t v = 0; v < V; ++v) order[v] = (int32_t)v;
        /* stable sort by value, descending: equal values keep ascending index */
        std::stable_sort(order.begin(), order.end(),
                         [&](int32_t a, int32_t b) { return x[a] > x[b]; });
        for (int k = 0; k < ORC_K; ++k) {
            int32_t v = order[k];
            idx[r * ORC_K + k] = v;
            logp[r * ORC_K + k] = z[v] - lz;
            prob[r * ORC_K + k] = exp(z[v] - lz);
        }
        logz[r] = lz;
    }
    return 0;
}
