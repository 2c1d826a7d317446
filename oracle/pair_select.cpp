/*
 * pair_select.cpp -- the bilinear adjacent-pair score and the exact best path
 * through the 16 candidates of each drafted position.
 * TEST INFRASTRUCTURE ONLY (see oracle.h).
 *
 * Source: [tamsi] "L’idée, sans le papier" -- the problem is choosing a
 * coherent path through candidate lists that are already good, done by a
 * small pair selector; [myaiexp] "主な機能" -- adjacent candidate pairs are
 * scored so the block stays coherent; [psi] "Résumé" -- candidates are chosen
 * with a bilinear attention.  The pages give the selector only in outline;
 * the form used here is the bilinear score e(a)^T W e(b) between a candidate
 * a at one position and a candidate b at the next, added to the drafter
 * log-probabilities, maximised over whole paths.
 *
 * Positions 0..G-1 are the drafted positions; c[i][k] = idx[b][i][k] is the
 * k-th candidate (rank k) of position i.  The anchor (last accepted token)
 * precedes position 0 as a single known state; with no anchor its term is
 * absent.
 *   score(path) = sum_i logp[i][k_i] + [anchor] pair(anchor, c[0][k_0])
 *               + sum_{i>0} pair(c[i-1][k_{i-1}], c[i][k_i])
 * The best path is found by the max-sum recursion over positions:
 *   delta[0][k]  = logp[0][k] + [anchor] pair(anchor, c[0][k])
 *   delta[i][k'] = logp[i][k'] + max_k (delta[i-1][k] + pair(c[i-1][k], c[i][k']))
 * On equal scores the smaller rank wins, both for the back-pointer and for
 * the final state, which returns the optimal path whose rank vector, read
 * from the last position backwards, is smallest.
 */
#include <vector>

#include "oracle_util.h"

extern "C" double orc_pair(const void* emb, int emb_dtype, int d, const float* W, int32_t a,
                           int32_t b) {
    double s = 0.0;
    for (int j = 0; j < d; ++j) {
        double ea = orc_load(emb, emb_dtype, (int64_t)a * d + j);
        for (int l = 0; l < d; ++l) {
            double eb = orc_load(emb, emb_dtype, (int64_t)b * d + l);
            s += ea * (double)W[(int64_t)j * d + l] * eb;
        }
    }
    return s;
}

static int check_args(const int32_t* idx, const float* logp, const void* emb, int emb_dtype,
                      int64_t V, int d, const float* W, int B, int G) {
    if (!idx || !logp || !emb || !W || !orc_dtype_ok(emb_dtype) || V < ORC_K || d < 1 ||
        B < 0 || G < 1)
        return -1;
    return 0;
}

extern "C" int orc_pair_select(const int32_t* idx, const float* logp, const int32_t* anchor,
                               const void* emb, int emb_dtype, int64_t V, int d, const float* W,
                               int B, int G, int32_t* path_tok, int32_t* path_rank,
                               double* path_score) {
    if (check_args(idx, logp, emb, emb_dtype, V, d, W, B, G)) return -1;
    const int K = ORC_K;
    std::vector<double> delta((size_t)G * K);
    std::vector<int> back((size_t)G * K, 0);
    for (int b = 0; b < B; ++b) {
        const int32_t* c = idx + (int64_t)b * G * K;
        const float* lp = logp + (int64_t)b * G * K;
        for (int k = 0; k < K; ++k) {
            double a = 0.0;
            if (anchor) a = orc_pair(emb, emb_dtype, d, W, anchor[b], c[k]);
            delta[k] = (double)lp[k] + a;
        }
        for (int i = 1; i < G; ++i) {
            for (int k2 = 0; k2 < K; ++k2) {
                double best = 0.0;
                int arg = -1;
                for (int k = 0; k < K; ++k) {
                    double cand = delta[(i - 1) * K + k] +
                                  orc_pair(emb, emb_dtype, d, W, c[(i - 1) * K + k], c[i * K + k2]);
                    if (arg < 0 || cand > best) {
                        best = cand;
                        arg = k;
                    }
                }
                delta[i * K + k2] = (double)lp[i * K + k2] + best;
                back[i * K + k2] = arg;
            }
        }
        int kstar = 0;
        for (int k = 1; k < K; ++k)
            if (delta[(G - 1) * K + k] > delta[(G - 1) * K + kstar]) kstar = k;
        path_score[b] = delta[(G - 1) * K + kstar];
        int k = kstar;
        for (int i = G - 1; i >= 0; --i) {
            path_rank[(int64_t)b * G + i] = k;
            path_tok[(int64_t)b * G + i] = c[i * K + k];
            if (i > 0) k = back[i * K + k];
        }
    }
    return 0;
}

extern "C" int orc_path_rescore(const int32_t* idx, const float* logp, const int32_t* anchor,
                                const void* emb, int emb_dtype, int64_t V, int d, const float* W,
                                int B, int G, const int32_t* path_rank, double* score) {
    if (check_args(idx, logp, emb, emb_dtype, V, d, W, B, G) || !path_rank) return -1;
    const int K = ORC_K;
    for (int b = 0; b < B; ++b) {
        const int32_t* c = idx + (int64_t)b * G * K;
        const float* lp = logp + (int64_t)b * G * K;
        const int32_t* rk = path_rank + (int64_t)b * G;
        for (int i = 0; i < G; ++i)
            if (rk[i] < 0 || rk[i] >= K) return -1;
        double s = 0.0;
        for (int i = 0; i < G; ++i) s += (double)lp[i * K + rk[i]];
        if (anchor) s += orc_pair(emb, emb_dtype, d, W, anchor[b], c[rk[0]]);
        for (int i = 1; i < G; ++i)
            s += orc_pair(emb, emb_dtype, d, W, c[(i - 1) * K + rk[i - 1]], c[i * K + rk[i]]);
        score[b] = s;
    }
    return 0;
}
