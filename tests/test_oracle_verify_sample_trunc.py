"""Pins of the oracle's verification of top-k / top-p truncated distributions
(oracle/verify_sample_trunc.cpp): truncation switched off reduces to the
plain sampling oracle; top-1 truncation reduces to the greedy verify; the
truncated probabilities of a hand-worked row in closed form; and the exact
marginal of the first emitted token equals the truncated target (the
lossless property), measured by bisection on the oracle's own decisions."""
import math

import numpy as np
import pytest

pytestmark = pytest.mark.filterwarnings("ignore")


def truncated_np(x, inv_t, top_k, top_p):
    """Independent restatement (numpy): order by (z desc, index asc), top-k,
    then the shortest prefix whose renormalised cumulative sum reaches top_p;
    renormalise.  Returns a dense vector."""
    z = np.asarray(x, np.float64) * inv_t
    V = len(z)
    order = np.lexsort((np.arange(V), -z))
    kk = top_k if 0 < top_k < V else V
    keep = order[:kk]
    e = np.exp(z[keep] - z.max())
    if top_p < 1.0:
        c = np.cumsum(e / e.sum())
        kp = int(np.argmax(c >= top_p)) + 1 if np.any(c >= top_p) else kk
        keep, e = keep[:kp], e[:kp]
    out = np.zeros(V)
    out[keep] = e / e.sum()
    return out


def test_no_truncation_is_the_plain_verify(orc):
    rng = np.random.default_rng(71)
    B, G, V = 64, 3, 50
    for dt in ("f32", "bf16"):
        t = (rng.standard_normal((B, G + 1, V)) * 1.5).astype(np.float32)
        q = (t[:, :G] + rng.standard_normal((B, G, V)) * 0.7).astype(np.float32)
        if dt == "bf16":
            import synth
            t, q = synth.to_bf16_bits(t), synth.to_bf16_bits(q)
        d = rng.integers(0, V, (B, G)).astype(np.int32)
        ua, ur = rng.random((B, G)), rng.random((B, G + 1))
        for mode, qq in ((0, q), (1, None)):
            n, out, ratio, ma, mr, mt = orc.verify_sample_trunc_u(t, qq, d, ua, ur, 0.8, 0, 1.0,
                                                                  mode)
            on, oout, oratio, oma, omr = orc.verify_sample_u(t, qq, d, ua, ur, 0.8, mode)
            np.testing.assert_allclose(ratio, oratio, rtol=1e-12, atol=1e-300)
            assert np.all(np.isinf(mt))
            same = (n == on) & np.all(out == oout, axis=1)
            assert np.all(same | (oma < 1e-9) | (omr < 1e-9)), np.where(~same)


@pytest.mark.parametrize("mode", [0, 1])
def test_top1_truncation_is_the_greedy_verify(orc, mode):
    """top-k = 1: p~ and q~ are point masses on the rows' argmaxes; on the
    drafter's top-1 path (softmax mode) or any path (one-hot mode) the
    verification accepts exactly the matching prefix and emits the target's
    argmax, whatever the uniforms."""
    rng = np.random.default_rng(72 + mode)
    B, G, V = 128, 4, 40
    t = (rng.standard_normal((B, G + 1, V)) * 2.0).astype(np.float32)
    q = (t[:, :G] + rng.standard_normal((B, G, V)) * 0.8).astype(np.float32)
    d = np.argmax(q, axis=2).astype(np.int32) if mode == 0 else \
        rng.integers(0, V, (B, G)).astype(np.int32)
    for seed in range(3):
        ua, ur = np.random.default_rng(seed).random((B, G)), np.random.default_rng(9 + seed).random((B, G + 1))
        n, out, _, _, _, _ = orc.verify_sample_trunc_u(t, q if mode == 0 else None, d, ua, ur, 1.0,
                                                       1, 0.95, mode)
        gn, gout = orc.verify_greedy(t, d)
        np.testing.assert_array_equal(n, gn)
        np.testing.assert_array_equal(out, gout)


def test_truncation_closed_form(orc):
    """Row x = (2, 1, 1, 0, -1), invT = 1; the one-hot ratio r_0 = p~(d_0)
    reads the truncated row.  top-k 3, top-p 0.75: kept {0, 1} (tokens 1 and 2
    tie; the lower index goes first), p~ = (e/(e+1), 1/(e+1)).  top-k 3,
    top-p 0.8: kept {0, 1, 2}, p~ = (e/(e+2), 1/(e+2), 1/(e+2)).  top-k 2:
    {0, 1} again.  No truncation: softmax."""
    e = math.e
    x = np.array([2.0, 1.0, 1.0, 0.0, -1.0], np.float32)
    t = np.tile(x, (5, 2, 1))                     # B = 5 sequences, G = 1
    d = np.arange(5, dtype=np.int32)[:, None]     # sequence b drafts token b
    ua, ur = np.zeros((5, 1)), np.zeros((5, 2))
    cases = [((3, 0.75), [e / (e + 1), 1 / (e + 1), 0, 0, 0]),
             ((3, 0.8), [e / (e + 2), 1 / (e + 2), 1 / (e + 2), 0, 0]),
             ((2, 1.0), [e / (e + 1), 1 / (e + 1), 0, 0, 0])]
    soft = np.exp(x.astype(np.float64)) / np.exp(x.astype(np.float64)).sum()
    cases.append(((0, 1.0), list(soft)))
    for (k, p), want in cases:
        _, _, ratio, _, _, mt = orc.verify_sample_trunc_u(t, None, d, ua, ur, 1.0, k, p, 1)
        np.testing.assert_allclose(ratio[:, 0], want, rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(ratio[:, 0], truncated_np(x, 1.0, k, p), rtol=1e-12,
                                   atol=1e-15)
    # the cut's margin: top-p 0.75 cuts after e/(e+2) + 1/(e+2) = (e+1)/(e+2)
    _, _, _, _, _, mt = orc.verify_sample_trunc_u(t, None, d, ua, ur, 1.0, 3, 0.75, 1)
    want = min((e + 1) / (e + 2) - 0.75, 0.75 - e / (e + 2))
    np.testing.assert_allclose(mt, want, rtol=1e-12)


def draw_measures(orc, t, q, x, u_acc, inv_t, k, p, mode, grid=2048, iters=48):
    """Measure (over u_res in [0, 1)) of every first token the oracle emits for
    one sequence, with drafted token x at position 0 and the accept uniform
    fixed: the pick is a step function of u_res (inverse CDF in index order),
    so its steps are found on a grid and their ends refined by bisection."""
    G = t.shape[0] - 1

    def picks(us):
        m = len(us)
        tt = np.broadcast_to(t, (m,) + t.shape).copy()
        qq = None if q is None else np.broadcast_to(q, (m,) + q.shape).copy()
        d = np.zeros((m, G), np.int32)
        d[:, 0] = x
        ua = np.full((m, G), u_acc)
        ur = np.zeros((m, G + 1))
        ur[:, 0] = us
        ur[:, 1:] = us[:, None]
        n, out, _, _, _, _ = orc.verify_sample_trunc_u(tt, qq, d, ua, ur, inv_t, k, p, mode)
        return out[:, 0]

    us = (np.arange(grid) + 0.5) / grid
    pk = picks(us)
    bounds = [0.0]
    for i in np.nonzero(pk[1:] != pk[:-1])[0]:
        lo, hi = us[i], us[i + 1]
        a, b0 = pk[i], pk[i + 1]
        for _ in range(iters):
            mid = 0.5 * (lo + hi)
            if picks(np.array([mid]))[0] == a:
                lo = mid
            else:
                hi = mid
        bounds.append(0.5 * (lo + hi))
    bounds.append(1.0)
    tokens = [pk[0]] + [pk[i + 1] for i in np.nonzero(pk[1:] != pk[:-1])[0]]
    meas = {}
    for tok, a, b0 in zip(tokens, bounds[:-1], bounds[1:]):
        meas[int(tok)] = meas.get(int(tok), 0.0) + (b0 - a)
    return meas


@pytest.mark.parametrize("k,p", [(5, 0.9), (3, 1.0), (0, 0.6)])
def test_first_token_marginal_is_the_truncated_target(orc, k, p):
    """Lossless w.r.t. the truncated target: P(first token = y) = p~_0(y),
    exactly, for the one-hot rule with every drafted token x (kept or not) and
    for the softmax rule with x drawn from q~_0.  Accept probabilities come
    from the ratio the oracle reports (u_acc below or above it), draw measures
    from bisection on u_res."""
    rng = np.random.default_rng(100 + k)
    V, G, inv_t = 12, 2, 0.9
    t = (rng.standard_normal((G + 1, V)) * 1.3).astype(np.float32)
    q = (t[:G] + rng.standard_normal((G, V)) * 0.6).astype(np.float32)
    pt = truncated_np(t[0], inv_t, k, p)
    qt = truncated_np(q[0], inv_t, k, p)
    def first_token_marginal(x, mode):
        d = np.zeros((1, G), np.int32)
        d[0, 0] = x
        qq = None if mode == 1 else q
        _, _, ratio, _, _, _ = orc.verify_sample_trunc_u(
            t[None], None if qq is None else qq[None], d, np.zeros((1, G)), np.zeros((1, G + 1)),
            inv_t, k, p, mode)
        r = ratio[0, 0]
        a = min(1.0, r)
        marg = np.zeros(V)
        marg[x] += a
        if a < 1.0:  # u_acc = r rejects (the rule is u < r): the residual draw
            for y, m in draw_measures(orc, t, qq, x, max(r, 0.0), inv_t, k, p, mode).items():
                marg[y] += (1.0 - a) * m
        return marg

    for x in range(V):  # one-hot rule: the marginal is p~_0 for every drafted token
        np.testing.assert_allclose(first_token_marginal(x, 1), pt, atol=1e-9, err_msg=str(x))
    marg = np.zeros(V)  # softmax rule: x drawn from q~_0
    for x in range(V):
        if qt[x] > 0:
            marg += qt[x] * first_token_marginal(x, 0)
    np.testing.assert_allclose(marg, pt, atol=1e-9)
