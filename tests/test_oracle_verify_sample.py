"""Pins of the oracle's sampling-mode verify (tamsi page, "Les chiffres qui
comptent sur Qwen3.8-27B": rejection sampling keeps the target's distribution;
latenode page, "Preguntas frecuentes": sampling preserves the distribution).

1. Hand-worked cases (tests/golden/sample_cases.json).
2. The exact identity, on the oracle's own decisions: for V <= 8 the measure
   of the uniforms u (accept) and u' (draw) that lead to each outcome is found
   by bisection on the oracle, so P(first emitted token = y) is computed
   without sampling and must equal p(y) to 1e-12 -- with the drafted token
   x ~ q (softmax mode) and for every fixed x (one-hot mode).
3. Chi-square over 10^6 oracle cycles on the oracle's Philox stream, the
   drafted tokens drawn from q with the test-only purpose-2 uniforms.
4. Special cases: p = q always accepts; p(d) = 0 always rejects and never
   emits d; one-hot with p(d) = 1 accepts.
"""
import json
import os

import numpy as np
import pytest
from scipy import stats
from scipy.special import softmax

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "sample_cases.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


@pytest.mark.parametrize("mode", ["softmax", "onehot"])
def test_golden_cases(orc, mode):
    g = _golden()
    tgt = np.array(g["target_logits"], np.float32)[None]
    drf = np.array(g["draft_logits"], np.float32)[None]
    cases = g["cases"] if mode == "softmax" else g["onehot_cases"]
    qm = orc.Q_SOFTMAX if mode == "softmax" else orc.Q_ONEHOT
    for c in cases:
        n, out, ratio, _, _ = orc.verify_sample_u(
            tgt, drf if mode == "softmax" else None, np.array([[c["d"]]], np.int32),
            np.array([[c["u"]]]), np.array([c["u_res"]]), 1.0, qm)
        assert n[0] == c["n"], c
        np.testing.assert_array_equal(out[0], c["out"])
        assert ratio[0, 0] == pytest.approx(c["ratio"], rel=1e-6)


# ----------------------------------------------------------------- exact identity
def _run(orc, tgt, drf, d, u_acc, u_res, qm, invT):
    """One oracle call over a batch of identical logits with per-row uniforms."""
    B = len(d)
    T = np.broadcast_to(tgt, (B,) + tgt.shape).copy()
    Q = None if drf is None else np.broadcast_to(drf, (B,) + drf.shape).copy()
    n, out, _, _, _ = orc.verify_sample_u(T, Q, np.asarray(d, np.int32).reshape(B, -1),
                                          np.asarray(u_acc, np.float64).reshape(B, -1),
                                          np.asarray(u_res, np.float64).reshape(B, -1), invT, qm)
    return n, out


def _accept_measure(orc, tgt, drf, qm, invT, V):
    """For each drafted token x: the length of {u in [0,1): accepted}."""
    lo, hi = np.zeros(V), np.ones(V)
    # the accepted set is [0, r): bisect for its right end
    for _ in range(56):
        mid = (lo + hi) / 2
        n, _ = _run(orc, tgt, drf, np.arange(V), mid, np.full((V, 2), 0.5), qm, invT)
        acc = n == 1
        lo = np.where(acc, mid, lo)
        hi = np.where(acc, hi, mid)
    n0, _ = _run(orc, tgt, drf, np.arange(V), np.zeros(V), np.full((V, 2), 0.5), qm, invT)
    return np.where(n0 == 1, hi, 0.0)


def _draw_measure(orc, tgt, drf, qm, invT, V, x, row):
    """Length of {u' in [0,1): the draw at ``row`` (0 = residual after rejecting x,
    1 = bonus after accepting x) returns y}, for each y."""
    # the draw is an inverse CDF, monotone in u': find where it first exceeds y
    u_acc = 1.0 - 2.0 ** -40 if row == 0 else 0.0
    lo, hi = np.zeros(V), np.ones(V)
    for _ in range(56):
        mid = (lo + hi) / 2
        ur = np.zeros((V, 2))
        ur[:, row] = mid
        _, out = _run(orc, tgt, drf, np.full(V, x), np.full(V, u_acc), ur, qm, invT)
        above = out[:, row] > np.arange(V)
        hi = np.where(above, mid, hi)
        lo = np.where(above, lo, mid)
    ends = np.minimum(hi, 1.0)
    ends[-1] = 1.0
    return np.diff(np.concatenate([[0.0], ends]))


@pytest.mark.parametrize("V", [2, 5, 8])
@pytest.mark.parametrize("invT", [1.0, 0.6])
def test_exact_marginal_softmax_mode(orc, V, invT):
    rng = np.random.default_rng(100 + V)
    tgt = (rng.standard_normal((2, V)) * 1.5).astype(np.float32)
    drf = (tgt[:1] + rng.standard_normal((1, V))).astype(np.float32)
    p = softmax(tgt[0].astype(np.float64) * invT)
    p1 = softmax(tgt[1].astype(np.float64) * invT)
    q = softmax(drf[0].astype(np.float64) * invT)
    a = _accept_measure(orc, tgt, drf, orc.Q_SOFTMAX, invT, V)
    np.testing.assert_allclose(a, np.minimum(1.0, p / q), rtol=0, atol=1e-12)
    marg = np.zeros(V)
    for x in range(V):
        marg[x] += q[x] * a[x]
        if a[x] < 1.0:
            marg += q[x] * (1.0 - a[x]) * _draw_measure(orc, tgt, drf, orc.Q_SOFTMAX, invT, V, x, 0)
    np.testing.assert_allclose(marg, p, rtol=0, atol=1e-12)
    # the bonus row after a full accept is drawn from p_G
    np.testing.assert_allclose(_draw_measure(orc, tgt, drf, orc.Q_SOFTMAX, invT, V, 0, 1), p1,
                               rtol=0, atol=1e-12)


@pytest.mark.parametrize("V", [3, 8])
def test_exact_marginal_onehot_mode_every_fixed_draft(orc, V):
    rng = np.random.default_rng(200 + V)
    tgt = (rng.standard_normal((2, V)) * 2).astype(np.float32)
    p = softmax(tgt[0].astype(np.float64))
    a = _accept_measure(orc, tgt, None, orc.Q_ONEHOT, 1.0, V)
    np.testing.assert_allclose(a, p, rtol=0, atol=1e-12)
    for x in range(V):
        marg = (1.0 - a[x]) * _draw_measure(orc, tgt, None, orc.Q_ONEHOT, 1.0, V, x, 0)
        marg[x] += a[x]
        np.testing.assert_allclose(marg, p, rtol=0, atol=1e-12)


# ----------------------------------------------------------------- chi-square
@pytest.mark.slow
def test_chi_square_one_million_cycles(orc):
    V, G, N, chunk = 8, 2, 1_000_000, 100_000
    rng = np.random.default_rng(9)
    tgt = (rng.standard_normal((G + 1, V)) * 1.5).astype(np.float32)
    drf = (tgt[:G] + rng.standard_normal((G, V)) * 0.8).astype(np.float32)
    p = softmax(tgt.astype(np.float64), axis=1)
    q = softmax(drf.astype(np.float64), axis=1)
    seed, step = 1234, 77
    first, second, bonus = np.zeros(V), np.zeros(V), np.zeros(V)
    for s0 in range(0, N, chunk):
        sid = np.arange(s0, s0 + chunk, dtype=np.uint32)
        d = np.stack([np.searchsorted(np.cumsum(q[j]), orc.uniforms(seed, step, sid, j, 2),
                                      side="right").clip(0, V - 1) for j in range(G)], axis=1)
        T = np.broadcast_to(tgt, (chunk, G + 1, V)).copy()
        Q = np.broadcast_to(drf, (chunk, G, V)).copy()
        n, out, _, _, _, _ = orc.verify_sample(T, Q, d, seed, step, sid)
        first += np.bincount(out[:, 0], minlength=V)
        second += np.bincount(out[n >= 1, 1], minlength=V)
        bonus += np.bincount(out[n == G, G], minlength=V)
    for counts, dist in ((first, p[0]), (second, p[1]), (bonus, p[2])):
        assert stats.chisquare(counts, dist * counts.sum())[1] > 1e-3
    assert counts.sum() > 1000


# ----------------------------------------------------------------- special cases
def test_p_equals_q_always_accepts(orc):
    rng = np.random.default_rng(11)
    B, G, V = 500, 3, 50
    tgt = rng.standard_normal((B, G + 1, V)).astype(np.float32)
    drf = tgt[:, :G].copy()
    d = rng.integers(0, V, (B, G)).astype(np.int32)
    n, out, ratio, u, _, _ = orc.verify_sample(tgt, drf, d, 5, 1)
    assert np.all(n == G)
    np.testing.assert_array_equal(ratio, 1.0)
    np.testing.assert_array_equal(out[:, :G], d)
    assert np.all(out[:, G] >= 0)


def test_zero_target_probability_always_rejects(orc):
    rng = np.random.default_rng(12)
    B, G, V = 400, 2, 30
    tgt = rng.standard_normal((B, G + 1, V)).astype(np.float32)
    drf = rng.standard_normal((B, G, V)).astype(np.float32)
    d = rng.integers(0, V, (B, G)).astype(np.int32)
    tgt[np.arange(B), 0, d[:, 0]] = -1000.0          # p(d_0) underflows to 0
    n, out, ratio, _, _, _ = orc.verify_sample(tgt, drf, d, 3, 9)
    assert np.all(n == 0)
    assert np.all(ratio[:, 0] == 0.0)
    assert np.all(out[:, 0] != d[:, 0])
    n, out, _, _, _, _ = orc.verify_sample(tgt, None, d, 3, 9, q_mode=orc.Q_ONEHOT)
    assert np.all(n == 0) and np.all(out[:, 0] != d[:, 0])


def test_onehot_certain_token_accepts(orc):
    B, G, V = 64, 4, 20
    rng = np.random.default_rng(13)
    d = rng.integers(0, V, (B, G)).astype(np.int32)
    tgt = np.zeros((B, G + 1, V), np.float32)
    for j in range(G):
        tgt[np.arange(B), j, d[:, j]] = 1000.0          # p(d_j) = 1
    n, out, ratio, _, _, _ = orc.verify_sample(tgt, None, d, 1, 1, q_mode=orc.Q_ONEHOT)
    assert np.all(n == G)
    np.testing.assert_array_equal(ratio, 1.0)


def test_uniforms_are_the_philox_stream(orc):
    """verify_sample's uniforms are the (step, seq_id, position, purpose 0) draws."""
    B, G, V = 3, 5, 16
    rng = np.random.default_rng(14)
    tgt = rng.standard_normal((B, G + 1, V)).astype(np.float32)
    drf = rng.standard_normal((B, G, V)).astype(np.float32)
    sid = np.array([7, 100, 3], np.uint32)
    d = rng.integers(0, V, (B, G)).astype(np.int32)
    *_, u, _, _ = orc.verify_sample(tgt, drf, d, 42, 6, sid)
    for j in range(G):
        np.testing.assert_array_equal(u[:, j], orc.uniforms(42, 6, sid, j, 0))
