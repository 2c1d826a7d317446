"""Pins of the oracle's greedy verify (tamsi page, "Les chiffres qui comptent
sur Qwen3.8-27B": greedy output equals the target exactly; latenode page, "El
desacuerdo empieza en las propias tablas del proveedor": acceptance length =
tokens completed per verify step).

Hand-worked cases live in tests/golden/greedy_cases.json.  The acceptance
length law is pinned to its closed form: if each drafted token equals the
target's choice independently with probability pi, then
P(n >= k) = pi^k and E[n + 1] = sum_{k=0..G} pi^k = (1 - pi^(G+1)) / (1 - pi);
for G = 7 and pi = 0.848 that is the pages' mean of 4.8.
"""
import json
import os

import numpy as np
import pytest
from scipy import stats

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "greedy_cases.json")


def _cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _cases(), ids=lambda c: c["name"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_golden_cases(orc, case, dtype):
    tgt = np.array(case["target"], np.float32)
    if dtype == "bf16":
        bits = synth.to_bf16_bits(tgt)
        assert np.array_equal(synth.bf16_bits_to_f32(bits), tgt)  # values exact in bf16
        tgt = bits
    n, out = orc.verify_greedy(tgt, np.array(case["draft_tok"], np.int32))
    np.testing.assert_array_equal(n, case["n"])
    np.testing.assert_array_equal(out, case["out"])
    np.testing.assert_array_equal(n + 1, case["accept_len"])


def _iid_match_batch(rng, B, G, V, pi):
    tgt = rng.standard_normal((B, G + 1, V)).astype(np.float32)
    amax = tgt.argmax(axis=2)
    hit = rng.random((B, G)) < pi
    wrong = (amax[:, :G] + rng.integers(1, V, (B, G))) % V
    draft = np.where(hit, amax[:, :G], wrong).astype(np.int32)
    return tgt, draft, amax


def test_acceptance_length_closed_form(orc):
    rng = np.random.default_rng(7)
    B, G, V, pi = 40000, 7, 8, 0.848
    tgt, draft, amax = _iid_match_batch(rng, B, G, V, pi)
    n, out = orc.verify_greedy(tgt, draft)
    L = n + 1
    mean = (1 - pi ** (G + 1)) / (1 - pi)
    assert mean == pytest.approx(4.8, abs=0.03)
    assert abs(L.mean() - mean) < 4 * L.std() / np.sqrt(B)
    # the whole law: P(n = k) = pi^k (1 - pi) for k < G, pi^G for k = G
    expect = np.array([pi ** k * (1 - pi) for k in range(G)] + [pi ** G]) * B
    counts = np.bincount(n, minlength=G + 1)
    assert stats.chisquare(counts, expect)[1] > 1e-3
    # emitted tokens: the accepted prefix, then the target's own choice
    for b in range(200):
        k = n[b]
        np.testing.assert_array_equal(out[b, :k], draft[b, :k])
        assert out[b, k] == amax[b, k]
        np.testing.assert_array_equal(out[b, k + 1:], -1)
