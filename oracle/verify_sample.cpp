/*
 * verify_sample.cpp -- sampling-mode lossless verification by rejection
 * sampling, with the residual resample and the bonus draw.
 * TEST INFRASTRUCTURE ONLY (see oracle.h).
 *
 * Source: [tamsi] "Les chiffres qui comptent sur Qwen3.8-27B" -- sampling via
 * rejection sampling keeps the same distribution; [latenode] "Un drafter que
 * adivina el bloque entero de una vez" and "Preguntas frecuentes" -- sampling
 * preserves the target distribution.  The pages name the method but print no
 * rule; the rule here is the standard speculative rejection sampler:
 *
 * With p_j = softmax(target[j] * invT) and q_j = softmax(draft[j] * invT):
 *   for j = 0, 1, ...: r_j = p_j(d_j) / q_j(d_j) = exp(lp_j - lq_j),
 *       lp_j = z^t_j[d_j] - logZ^t_j,  lq_j = z^q_j[d_j] - logZ^q_j;
 *       accept d_j iff u_j < r_j (strict, so r_j >= 1 always accepts);
 *       stop at the first rejection; n = number accepted.
 *   if n < G: draw from w = max(0, p_n - q_n) normalised (the residual);
 *   if n = G: draw the bonus token from p_G.
 * q_mode ONEHOT (q is a point mass on the drafted token, the reading for a
 * deterministic selector): lq_j = 0 and the residual is p_n with d_n removed.
 * If the residual mass R is zero (possible only through rounding when p and
 * q agree), the draw falls back to p_n.
 *
 * The draw: t = u' * R with R = sum_v w_v; the token is the smallest v whose
 * inclusive prefix sum C_v exceeds t; if rounding leaves none, the last v
 * with w_v > 0.  Uniforms: u_j (purpose 0, position j) and u' (purpose 1,
 * position n) from the Philox stream of philox.cpp.
 *
 * Diagnostics: ratio[b][j] = r_j for every j < G; margin_acc[b] = the
 * smallest |u_j - r_j| over the decisions taken; margin_res[b] = the distance
 * from t to the nearer end of the chosen token's interval, divided by R.
 */
#include <math.h>

#include <algorithm>
#include <vector>

#include "oracle_util.h"

namespace {

/* z = row * invT and logZ = log(sum_v exp(z_v)) computed as max + log-sum. */
double row_logz(const void* base, int dtype, int64_t off, int64_t V, double invT) {
    double m = orc_load(base, dtype, off) * invT;
    for (int64_t v = 1; v < V; ++v) m = std::max(m, orc_load(base, dtype, off + v) * invT);
    double s = 0.0;
    for (int64_t v = 0; v < V; ++v) s += exp(orc_load(base, dtype, off + v) * invT - m);
    return m + log(s);
}

}  // namespace

extern "C" int orc_verify_sample_u(const void* target, const void* draft, int dtype, int B,
                                   int G, int64_t V, const int32_t* draft_tok,
                                   double inv_temperature, int q_mode, const double* u_acc,
                                   const double* u_res, int32_t* n_accept, int32_t* out_tok,
                                   double* ratio, double* margin_acc, double* margin_res) {
    if (!target || !draft_tok || !orc_dtype_ok(dtype) || B < 0 || G < 1 || V < 1 ||
        !(inv_temperature > 0.0) || !u_acc || !u_res)
        return -1;
    if (q_mode != ORC_Q_SOFTMAX && q_mode != ORC_Q_ONEHOT) return -1;
    if (q_mode == ORC_Q_SOFTMAX && !draft) return -1;
    const double invT = inv_temperature;
    std::vector<double> w((size_t)V);
    std::vector<double> r((size_t)G), lzt((size_t)G + 1), lzq((size_t)G);
    for (int b = 0; b < B; ++b) {
        const int32_t* d = draft_tok + (int64_t)b * G;
        for (int j = 0; j <= G; ++j)
            lzt[j] = row_logz(target, dtype, ((int64_t)b * (G + 1) + j) * V, V, invT);
        for (int j = 0; j < G; ++j) {
            int64_t toff = ((int64_t)b * (G + 1) + j) * V;
            double lp = orc_load(target, dtype, toff + d[j]) * invT - lzt[j];
            double lq = 0.0;
            if (q_mode == ORC_Q_SOFTMAX) {
                int64_t qoff = ((int64_t)b * G + j) * V;
                lzq[j] = row_logz(draft, dtype, qoff, V, invT);
                lq = orc_load(draft, dtype, qoff + d[j]) * invT - lzq[j];
            }
            r[j] = exp(lp - lq);
            if (ratio) ratio[(int64_t)b * G + j] = r[j];
        }

        /* accept / reject, stopping at the first rejection */
        int n = 0;
        double macc = INFINITY;
        while (n < G) {
            double u = u_acc[(int64_t)b * G + n];
            macc = std::min(macc, fabs(u - r[n]));
            if (u < r[n]) ++n;
            else break;
        }

        /* the distribution the last token is drawn from */
        int64_t toff = ((int64_t)b * (G + 1) + n) * V;
        for (int64_t v = 0; v < V; ++v) w[v] = exp(orc_load(target, dtype, toff + v) * invT - lzt[n]);
        if (n < G) {
            if (q_mode == ORC_Q_SOFTMAX) {
                int64_t qoff = ((int64_t)b * G + n) * V;
                for (int64_t v = 0; v < V; ++v) {
                    double q = exp(orc_load(draft, dtype, qoff + v) * invT - lzq[n]);
                    w[v] = std::max(0.0, w[v] - q);
                }
            } else {
                w[d[n]] = 0.0;
            }
            double R = 0.0;
            for (int64_t v = 0; v < V; ++v) R += w[v];
            if (!(R > 0.0)) /* residual empty by rounding: fall back to p_n */
                for (int64_t v = 0; v < V; ++v)
                    w[v] = exp(orc_load(target, dtype, toff + v) * invT - lzt[n]);
        }
        double R = 0.0;
        for (int64_t v = 0; v < V; ++v) R += w[v];
        double t = u_res[(int64_t)b * (G + 1) + n] * R;

        int64_t pick = -1;
        double before = 0.0, after = 0.0, C = 0.0;
        for (int64_t v = 0; v < V; ++v) {
            double prev = C;
            C += w[v];
            if (C > t) {
                pick = v;
                before = prev;
                after = C;
                break;
            }
        }
        if (pick < 0) { /* rounding left t at or above the total */
            for (int64_t v = V - 1; v >= 0; --v)
                if (w[v] > 0.0) {
                    pick = v;
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
    }
    return 0;
}

extern "C" int orc_verify_sample(const void* target, const void* draft, int dtype, int B, int G,
                                 int64_t V, const int32_t* draft_tok, double inv_temperature,
                                 uint64_t seed, uint32_t step, const uint32_t* seq_id, int q_mode,
                                 int32_t* n_accept, int32_t* out_tok, double* ratio, double* u,
                                 double* margin_acc, double* margin_res) {
    if (B < 0 || G < 1) return -1;
    std::vector<double> ua((size_t)B * G), ur((size_t)B * (G + 1));
    for (int b = 0; b < B; ++b) {
        uint32_t sid = seq_id ? seq_id[b] : (uint32_t)b;
        for (int j = 0; j < G; ++j) ua[(size_t)b * G + j] = orc_uniform(seed, step, sid, j, 0);
        for (int j = 0; j <= G; ++j)
            ur[(size_t)b * (G + 1) + j] = orc_uniform(seed, step, sid, j, 1);
    }
    if (u)
        for (size_t i = 0; i < ua.size(); ++i) u[i] = ua[i];
    return orc_verify_sample_u(target, draft, dtype, B, G, V, draft_tok, inv_temperature, q_mode,
                               ua.data(), ur.data(), n_accept, out_tok, ratio, margin_acc,
                               margin_res);
}
