"""Pins of the oracle's softmax + top-16 (tamsi page, "L’idée, sans le papier";
myaiexp page, "主な機能": the selector keeps the 16 best candidates of each
position).

The ordering is pinned to numpy's lexsort (a library sort on the same key),
the probabilities to scipy's logsumexp and to closed forms, and the special
cases to what the definition fixes.
"""
import numpy as np
import pytest
from scipy.special import logsumexp

import synth


def _lib_top16(x):
    """Indices sorted by value descending, index ascending on ties (numpy lexsort)."""
    x = x.astype(np.float64)
    v = np.arange(x.size)
    return np.lexsort((v, -x))[:16]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("invT", [1.0, 0.7, 1.9])
def test_random_rows_match_library_sort_and_logsumexp(orc, dtype, invT):
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((5, 4096)) * 2.0).astype(np.float32)
    if dtype == "bf16":
        store = synth.to_bf16_bits(x)            # many exact ties after rounding
        xv = synth.bf16_bits_to_f32(store)
    else:
        store, xv = x, x
    idx, prob, logp, logz = orc.topk_softmax(store, invT)
    for r in range(5):
        np.testing.assert_array_equal(idx[r], _lib_top16(xv[r]))
        z = xv[r].astype(np.float64) * invT
        lz = logsumexp(z)
        assert abs(logz[r] - lz) < 1e-12 * max(1.0, abs(lz))
        np.testing.assert_allclose(logp[r], z[idx[r]] - lz, rtol=0, atol=1e-12)
        np.testing.assert_allclose(prob[r], np.exp(z[idx[r]] - lz), rtol=1e-12)
    if dtype == "bf16":
        # the rounded rows really do hold ties inside the top 16
        assert any(len(set(xv[r][idx[r]])) < 16 for r in range(5))


def test_probabilities_sum_to_one_when_all_kept(orc):
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((3, 16)) * 4).astype(np.float32)
    _, prob, _, _ = orc.topk_softmax(x, 1.3)
    np.testing.assert_allclose(prob.sum(axis=1), 1.0, rtol=0, atol=1e-12)


@pytest.mark.parametrize("invT", [1.0, 2.0, 0.5])
def test_closed_form_log_ramp(orc, invT):
    """x_v = ln(v + 1): p_v = (v + 1)^invT / sum_u (u + 1)^invT."""
    V = 64
    x = np.log(np.arange(1, V + 1, dtype=np.float64)).astype(np.float32)
    idx, prob, logp, logz = orc.topk_softmax(x[None], invT)
    np.testing.assert_array_equal(idx[0], np.arange(V - 1, V - 17, -1))
    w = np.exp(invT * x.astype(np.float64))
    np.testing.assert_allclose(prob[0], w[idx[0]] / w.sum(), rtol=1e-12)
    np.testing.assert_allclose(logz[0], np.log(w.sum()), rtol=1e-13)


def test_uniform_row(orc):
    V = 1000
    idx, prob, logp, logz = orc.topk_softmax(np.full((1, V), 0.25, np.float32))
    np.testing.assert_array_equal(idx[0], np.arange(16))
    np.testing.assert_allclose(prob[0], 1.0 / V, rtol=1e-13)
    np.testing.assert_allclose(logz[0], 0.25 + np.log(V), rtol=1e-13)


def test_seventeen_equal_maxima_keep_lowest_sixteen(orc):
    V = 300
    x = np.zeros((1, V), np.float32)
    pos = np.sort(np.random.default_rng(3).choice(V, 17, replace=False))
    x[0, pos] = 5.0
    idx, _, _, _ = orc.topk_softmax(x)
    np.testing.assert_array_equal(idx[0], pos[:16])


def test_signed_zeros_are_equal(orc):
    x = np.full((1, 40), -1.0, np.float32)
    x[0, [3, 7, 9, 20]] = [-0.0, 0.0, -0.0, 0.0]
    idx, _, _, _ = orc.topk_softmax(x)
    np.testing.assert_array_equal(idx[0, :4], [3, 7, 9, 20])
    np.testing.assert_array_equal(idx[0, 4:], [0, 1, 2, 4, 5, 6, 8, 10, 11, 12, 13, 14])


def test_single_spike(orc):
    x = np.zeros((1, 5000), np.float32)
    x[0, 4321] = 50.0
    idx, prob, logp, _ = orc.topk_softmax(x)
    assert idx[0, 0] == 4321
    assert 1.0 - prob[0, 0] < 5000 * np.exp(-50.0) * 1.01
    np.testing.assert_allclose(prob[0, 1:], np.exp(-50.0) * prob[0, 0], rtol=1e-12)


def test_row_stride(orc):
    rng = np.random.default_rng(6)
    wide = (rng.standard_normal((6, 900)) * 2).astype(np.float32)
    a = orc.topk_softmax(wide[:, 100:800])
    b = orc.topk_softmax(np.ascontiguousarray(wide[:, 100:800]))
    for u, v in zip(a, b):
        np.testing.assert_array_equal(u, v)


def test_bf16_widening(orc):
    """bf16 bits widen exactly: the bf16 row gives the same answer as the fp32
    row holding the widened values."""
    rng = np.random.default_rng(4)
    bits = synth.to_bf16_bits((rng.standard_normal((4, 777)) * 3).astype(np.float32))
    f32 = synth.bf16_bits_to_f32(bits)
    a = orc.topk_softmax(bits, 1.1)
    b = orc.topk_softmax(f32, 1.1)
    for u, v in zip(a, b):
        np.testing.assert_array_equal(u, v)
