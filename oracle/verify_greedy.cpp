/*
 * verify_greedy.cpp -- greedy lossless verification of one drafted block.
 * TEST INFRASTRUCTURE ONLY (see oracle.h).
 *
 * Source: [tamsi] "Les chiffres qui comptent sur Qwen3.8-27B" -- greedy
 * decoding gives exactly the target's output; [latenode] "Un drafter que
 * adivina el bloque entero de una vez" -- the large model checks the proposed
 * tokens in one pass and what survives is kept; "El desacuerdo empieza..." --
 * acceptance length is tokens completed per verify step.
 *
 * Target rows j = 0..G (row j scores the token at drafted position j; row G
 * is the position after the block).  For each sequence:
 *   t_j = argmax_v target[j][v], lowest v among equal maxima
 *   n   = first j < G with draft_tok[j] != t_j, or G if there is none
 *   out = draft_tok[0..n-1], then t_n (the correction, or the bonus token when
 *         n = G), then -1 up to G+1 entries.
 * Tokens completed this step = n + 1.
 */
#include "oracle_util.h"

extern "C" int orc_verify_greedy(const void* target, int dtype, int B, int G, int64_t V,
                                 const int32_t* draft_tok, int32_t* n_accept, int32_t* out_tok) {
    if (!target || !draft_tok || !orc_dtype_ok(dtype) || B < 0 || G < 1 || V < 1) return -1;
    for (int b = 0; b < B; ++b) {
        int32_t t[64 + 1];
        if (G > 64) return -1;
        for (int j = 0; j <= G; ++j) {
            int64_t base = ((int64_t)b * (G + 1) + j) * V;
            int64_t best = 0;
            double bv = orc_load(target, dtype, base);
            for (int64_t v = 1; v < V; ++v) {
                double x = orc_load(target, dtype, base + v);
                if (x > bv) {
                    bv = x;
                    best = v;
                }
            }
            t[j] = (int32_t)best;
        }
        int n = 0;
        while (n < G && draft_tok[(int64_t)b * G + n] == t[n]) ++n;
        n_accept[b] = n;
        int32_t* o = out_tok + (int64_t)b * (G + 1);
        for (int j = 0; j <= G; ++j) o[j] = -1;
        for (int j = 0; j < n; ++j) o[j] = draft_tok[(int64_t)b * G + j];
        o[n] = t[n];
    }
    return 0;
}
