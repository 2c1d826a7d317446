// workspace.cuh -- layout of the caller-provided workspace of each call.
//
// The first CONTROL_BYTES of every workspace hold the calls' arrival counters
// (and dynconv's flags); partial results start after them, so no call's
// partials ever land on another call's counters.  A call whose counters fit
// the control area relies on them being zero and leaves them zero when it
// completes (its finishers reset what they used): a workspace is zeroed once,
// when it is allocated.  A call with more counters than fit (shapes far beyond
// the bench's) clears its own with one cudaMemsetAsync instead.  All regions
// start on 256-byte boundaries.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "common.cuh"
#include "ring.cuh"

namespace dfl {

// Partial result of one (row, chunk) unit of dflash2_topk_softmax: the
// chunk maximum m, the chunk's sum of exp2(x c - fl(m c)) and its top-16
// keys.
struct TopkPart {
    float m;
    float pad;
    double s;
    uint64_t key[K];
};

// Per-sequence state handed from the verify_sample scan to its draw:
// p_v = exp2((x_v - mt) * c - l2t) on the target row used, likewise q, and
// dl = logZ_t - logZ_q (natural log) for the residual.
struct SampleInfo {
    float mt, l2t;    // target row max and log2 of its sum-exp
    float mq, l2q;    // draft row (mode 0 only)
    float dl;         // logZ_t - logZ_q (mode 0 only)
    float u_res;      // u' of the draw
    int32_t n;        // accepted count = row the draw uses
    int32_t mode;     // 0 = residual max(0, p - q), 1 = p without d_n, 2 = p
    int32_t d;        // the rejected drafted token (mode 1)
    int32_t pad;
};

struct Layout {
    bool self_clean;  // counters in the control area: zero on entry, reset by the call
    size_t counters_off, counters_bytes;
    size_t part_off, part_bytes;
    size_t part2_off, part2_bytes;
    size_t info_off, info_bytes;
    size_t total;
};

inline size_t align256(size_t x) { return (x + 255) / 256 * 256; }

constexpr size_t CONTROL_BYTES = 65536;

// True when a call's counters fit the control area (self-cleaning, no memset).
inline bool counters_in_control(size_t counters) { return counters <= CONTROL_BYTES; }

inline Layout make_layout(size_t counters, size_t part, size_t part2 = 0, size_t info = 0) {
    Layout L;
    L.self_clean = counters_in_control(counters);
    L.counters_off = 0;
    L.counters_bytes = align256(counters);
    L.part_off = L.counters_bytes > CONTROL_BYTES ? L.counters_bytes : CONTROL_BYTES;
    L.part_bytes = align256(part);
    L.part2_off = L.part_off + L.part_bytes;
    L.part2_bytes = align256(part2);
    L.info_off = L.part2_off + L.part2_bytes;
    L.info_bytes = align256(info);
    L.total = L.info_off + L.info_bytes;
    return L;
}

// Layouts for an element size es (2 for bf16, 4 for fp32; a workspace sized
// with es = 4 serves both, its chunks being the shorter).
inline Layout topk_layout(int64_t rows, int64_t V, int es) {
    const int64_t S = row_chunks(V, es);  // counters [rows], then the rows' top-16 bounds [rows]
    return make_layout((size_t)rows * 8, (size_t)(rows * S) * sizeof(TopkPart));
}
inline Layout greedy_layout(int B, int G, int64_t V, int es) {
    const int64_t S = row_chunks(V, es);
    return make_layout((size_t)B * 4, (size_t)((int64_t)B * (G + 1) * S) * sizeof(uint64_t));
}
// Greedy with early exit: per sequence a counter and a skip word.
inline Layout greedy_ee_layout(int B, int G, int64_t V, int es) {
    const int64_t S = row_chunks(V, es);
    return make_layout((size_t)B * 8, (size_t)((int64_t)B * (G + 1) * S) * sizeof(uint64_t));
}
// Sampling: the control words (two queue words, a line each; scan and draw
// counters [B] each; the finish queue, a line per position), the scan's
// per-unit partials, the draw's per-unit lane prefixes (32 per chunk of the
// drawn row, and 32 of scratch) and the per-sequence hand-over to the draw.
constexpr int CTL_LINE = 32;  // words in a 128-byte line
__host__ __device__ inline size_t sample_fin_off(int B) {
    return (2 * (size_t)CTL_LINE + 2 * (size_t)B + CTL_LINE - 1) / CTL_LINE * CTL_LINE;
}
inline size_t sample_ctl_words(int B) { return sample_fin_off(B) + (size_t)B * CTL_LINE; }
inline Layout sample_layout(int B, int G, int64_t V, int es) {
    const int64_t S = row_chunks(V, es);
    // the draw's units are half chunks: 2 S + 1 per row is enough
    return make_layout(sample_ctl_words(B) * 4, (size_t)((int64_t)B * (2 * G + 1) * S) * sizeof(LseD),
                       (size_t)((int64_t)B * (2 * S + 1) + 1) * 32 * sizeof(double),
                       (size_t)B * sizeof(SampleInfo));
}
// Truncated sampling verify: control words (per row a counter and a shared
// top-32 bound, per sequence a counter of finished rows; rows = B (2G+1), the
// softmax-q count, which also covers one-hot q), the segment lists per
// (row, chunk) and the rows' top-32 lists.
constexpr int TRUNC_K = 32;
struct List32 {  // a running top-32 left at a segment's last chunk (key[0] = 0: none)
    uint64_t key[TRUNC_K];
};
inline Layout trunc_layout(int B, int G, int64_t V, int es) {
    const int64_t rows = (int64_t)B * (2 * G + 1);
    const int64_t S = row_chunks(V, es);
    return make_layout((size_t)(2 * rows + B) * 4, (size_t)(rows * S) * sizeof(List32),
                       (size_t)rows * TRUNC_K * sizeof(uint64_t));
}
inline Layout select_layout(int B, int G) {
    return make_layout((size_t)B * 4, (size_t)B * (K + (size_t)K * K * (G - 1)) * sizeof(float));
}

}  // namespace dfl
