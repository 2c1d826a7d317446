/*
 * verify_sample_trunc.cpp -- sampling-mode verification of distributions
 * truncated by top-k and top-p, the sampling settings a serving stack applies.
 * TEST INFRASTRUCTURE ONLY (see oracle.h).
 *
 * Source: [latenode] "DFlash2 speculative decoding", section "Preguntas
 * frecuentes": the recommended sampling for the Qwen targets is temperature
 * 1.0, top-p 0.95, top-k 20.  The pages do not say how truncation meets the
 * verification; the reading here: the distribution a token is sampled from is
 * the truncated one, so the verification keeps the truncated target
 * distribution p~ exactly, against the drafter's truncated distribution q~.
 *
 * Truncation of a row (z = x * invT, pi = softmax(z)):
 *   1. order the tokens by (z descending, index ascending);
 *   2. top-k: keep the first min(k, V) of them (k <= 0: all);
 *   3. top-p: renormalise pi over the kept tokens and keep the shortest
 *      prefix, in the same order, whose cumulative sum reaches top_p
 *      (cumsum >= top_p; at least one token; top_p >= 1: all);
 *   4. p~ = pi on the kept tokens, renormalised to sum 1.
 * The top-p decision's margin (the distance from top_p to the cumulative sum
 * on either side of the cut) is reported, so a caller can tell a float
 * near-tie at the cut.
 *
 * Verification, with p~_j, q~_j the truncated rows:
 *   r_j = p~_j(d_j) / q~_j(d_j)  (q_mode SOFTMAX; q~(d) = 0 < p~(d) gives
 *   r = +inf, both 0 give r = 0), or r_j = p~_j(d_j) (q_mode ONEHOT);
 *   accept iff u_j < r_j, stop at the first rejection, n = accepted count;
 *   n < G: draw from w = max(0, p~_n - q~_n) (ONEHOT: p~_n with d_n removed),
 *   from p~_n if that sums to zero; n = G: draw the bonus from p~_G.
 *   The draw takes t = u' * R and returns the smallest index whose inclusive
 *   prefix (index order) exceeds t, the last index with mass if none.
 */
#include <math.h>

#include <algorithm>
#include <numeric>
#include <vector>

#include "oracle_util.h"

namespace {

struct Truncated {
    std::vector<int64_t> idx;  // kept tokens, ascending
    std::vector<double> p;     // their renormalised probabilities
    double margin;             // top-p cut margin (+inf if no cut was made)
};

Truncated truncate_row(const void* base, int dtype, int64_t off, int64_t V, double invT,
                       int top_k, double top_p) {
    std::vector<double> z((size_t)V);
    double m = -INFINITY;
    for (int64_t v = 0; v < V; ++v) {
        z[v] = orc_load(base, dtype, off + v) * invT;
        m = std::max(m, z[v]);
    }
    std::vector<int64_t> ord((size_t)V);
    std::iota(ord.begin(), ord.end(), (int64_t)0);
    const int64_t kk = (top_k > 0 && (int64_t)top_k < V) ? (int64_t)top_k : V;
    std::partial_sort(ord.begin(), ord.begin() + kk, ord.end(), [&](int64_t a, int64_t b) {
        return z[a] > z[b] || (z[a] == z[b] && a < b);
    });
    std::vector<double> e((size_t)kk);
    double sk = 0.0;
    for (int64_t i = 0; i < kk; ++i) {
        e[i] = exp(z[ord[i]] - m);
        sk += e[i];
    }
    int64_t kp = kk;
    double margin = INFINITY;
    if (top_p < 1.0) {
        double c = 0.0;
        for (int64_t i = 0; i < kk; ++i) {
            const double before = c;
            c += e[i] / sk;
            if (c >= top_p) {
                kp = i + 1;
                margin = std::min(c - top_p, top_p - before);
                break;
            }
        }
    }
    double sp = 0.0;
    for (int64_t i = 0; i < kp; ++i) sp += e[i];
    std::vector<int64_t> sel(ord.begin(), ord.begin() + kp);
    std::sort(sel.begin(), sel.end());
    Truncated T;
    T.margin = margin;
    T.idx = sel;
    T.p.resize(sel.size());
    for (size_t i = 0; i < sel.size(); ++i) T.p[i] = exp(z[sel[i]] - m) / sp;
    return T;
}

double prob_of(const Truncated& T, int64_t v) {
    auto it = std::lower_bound(T.idx.begin(), T.idx.end(), v);
    if (it == T.idx.end() || *it != v) return 0.0;
    return T.p[(size_t)(it - T.idx.begin())];
}

}  // namespace

extern "C" int orc_verify_sample_trunc_u(const void* target, const void* draft, int dtype, int B,
                                         int G, int64_t V, const int32_t* draft_tok,
                                         double inv_temperature, int top_k, double top_p,
                                         int q_mode, const double* u_acc, const double* u_res,
                                         int32_t* n_accept, int32_t* out_tok, double* ratio,
                                         double* margin_acc, double* margin_res,
                                         double* margin_trunc) {
    if (!target || !draft_tok || !orc_dtype_ok(dtype) || B < 0 || G < 1 || V < 1 ||
        !(inv_temperature > 0.0) || !u_acc || !u_res || !(top_p > 0.0))
        return -1;
    if (q_mode != ORC_Q_SOFTMAX && q_mode != ORC_Q_ONEHOT) return -1;
    if (q_mode == ORC_Q_SOFTMAX && !draft) return -1;
    const double invT = inv_temperature;
    for (int b = 0; b < B; ++b) {
        const int32_t* d = draft_tok + (int64_t)b * G;
        std::vector<Truncated> pt((size_t)G + 1), qt;
        double mtr = INFINITY;
        for (int j = 0; j <= G; ++j) {
            pt[j] = truncate_row(target, dtype, ((int64_t)b * (G + 1) + j) * V, V, invT, top_k,
                                 top_p);
        }
        if (q_mode == ORC_Q_SOFTMAX) {
            qt.resize((size_t)G);
            for (int j = 0; j < G; ++j)
                qt[j] = truncate_row(draft, dtype, ((int64_t)b * G + j) * V, V, invT, top_k, top_p);
        }
        std::vector<double> r((size_t)G);
        for (int j = 0; j < G; ++j) {
            const double p = prob_of(pt[j], d[j]);
            if (q_mode == ORC_Q_SOFTMAX) {
                const double q = prob_of(qt[j], d[j]);
                r[j] = (q > 0.0) ? p / q : (p > 0.0 ? INFINITY : 0.0);
            } else {
                r[j] = p;
            }
            if (ratio) ratio[(int64_t)b * G + j] = r[j];
        }
        int n = 0;
        double macc = INFINITY;
        while (n < G) {
            const double u = u_acc[(int64_t)b * G + n];
            macc = std::min(macc, fabs(u - r[n]));
            mtr = std::min(mtr, pt[n].margin);
            if (q_mode == ORC_Q_SOFTMAX) mtr = std::min(mtr, qt[n].margin);
            if (u < r[n]) ++n;
            else break;
        }
        mtr = std::min(mtr, pt[n].margin);
        /* the draw: weights on the kept tokens of p~_n, in index order */
        const Truncated& P = pt[n];
        std::vector<double> w(P.p);
        if (n < G) {
            for (size_t i = 0; i < w.size(); ++i) {
                if (q_mode == ORC_Q_SOFTMAX) w[i] = std::max(0.0, w[i] - prob_of(qt[n], P.idx[i]));
                else if (P.idx[i] == d[n]) w[i] = 0.0;
            }
            if (q_mode == ORC_Q_SOFTMAX) mtr = std::min(mtr, qt[n].margin);
            double R0 = 0.0;
            for (double x : w) R0 += x;
            if (!(R0 > 0.0)) w = P.p;
        }
        double R = 0.0;
        for (double x : w) R += x;
        const double t = u_res[(int64_t)b * (G + 1) + n] * R;
        int64_t pick = -1;
        double before = 0.0, after = 0.0, C = 0.0;
        for (size_t i = 0; i < w.size(); ++i) {
            const double prev = C;
            C += w[i];
            if (C > t) {
                pick = P.idx[i];
                before = prev;
                after = C;
                break;
            }
        }
        if (pick < 0) {
            for (size_t i = w.size(); i-- > 0;)
                if (w[i] > 0.0) {
                    pick = P.idx[i];
                    break;
                }
            before = after = C;
        }
        n_accept[b] = n;
        int32_t* o = out_tok + (int64_t)b * (G + 1);
        for (int j = 0; j <= G; ++j) o[j] = -1;
        for (int j = 0; j < n; ++j) o[j] = d[j];
        o[n] = (int32_t)pick;
        if (margin_acc) margin_acc[b] = macc;
        if (margin_res) margin_res[b] = std::min(fabs(t - before), fabs(after - t)) / R;
        if (margin_trunc) margin_trunc[b] = mtr;
    }
    return 0;
}

extern "C" int orc_verify_sample_trunc(const void* target, const void* draft, int dtype, int B,
                                       int G, int64_t V, const int32_t* draft_tok,
                                       double inv_temperature, int top_k, double top_p,
                                       uint64_t seed, uint32_t step, const uint32_t* seq_id,
                                       int q_mode, int32_t* n_accept, int32_t* out_tok,
                                       double* ratio, double* u, double* margin_acc,
                                       double* margin_res, double* margin_trunc) {
    if (B < 0 || G < 1) return -1;
    std::vector<double> ua((size_t)B * G), ur((size_t)B * (G + 1));
    for (int b = 0; b < B; ++b) {
        const uint32_t sid = seq_id ? seq_id[b] : (uint32_t)b;
        for (int j = 0; j < G; ++j) ua[(size_t)b * G + j] = orc_uniform(seed, step, sid, j, 0);
        for (int j = 0; j <= G; ++j)
            ur[(size_t)b * (G + 1) + j] = orc_uniform(seed, step, sid, j, 1);
    }
    if (u)
        for (size_t i = 0; i < ua.size(); ++i) u[i] = ua[i];
    return orc_verify_sample_trunc_u(target, draft, dtype, B, G, V, draft_tok, inv_temperature,
                                     top_k, top_p, q_mode, ua.data(), ur.data(), n_accept, out_tok,
                                     ratio, margin_acc, margin_res, margin_trunc);
}
