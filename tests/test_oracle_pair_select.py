"""Pins of the oracle's bilinear pair selector and exact best path (tamsi page,
"L’idée, sans le papier": choose a coherent path through the top-16 lists;
myaiexp page, "主な機能": adjacent candidate pairs are scored; PSI page,
"Résumé": candidates chosen by a bilinear attention).

The recursion is pinned to brute-force enumeration of all 16^L paths (L <= 4)
with pair scores from a numpy matrix product, including the tie rule; the
bilinear form's orientation by a one-hot construction; special cases by what
the definition fixes.
"""
import itertools

import numpy as np
import pytest

import synth


def _problem(seed, B, G, V=64, d=8, dtype=np.float32, ties=False):
    rng = np.random.default_rng(seed)
    idx = np.stack([np.stack([rng.choice(V, 16, replace=False) for _ in range(G)])
                    for _ in range(B)]).astype(np.int32)
    if ties:
        logp = np.full((B, G, 16), -2.0, np.float32)
    else:
        logp = np.sort(rng.standard_normal((B, G, 16)).astype(np.float32) - 3, axis=2)[:, :, ::-1]
    emb = (rng.standard_normal((V, d)) / np.sqrt(d)).astype(np.float32)
    W = (rng.standard_normal((d, d)) / np.sqrt(d)).astype(np.float32)
    anchor = rng.integers(0, V, B).astype(np.int32)
    return idx, np.ascontiguousarray(logp), anchor, emb, W


def _brute(idx, logp, anchor, emb, W):
    """Score of every rank vector (k_0..k_{G-1}) by enumeration; pair scores by matmul."""
    e = emb.astype(np.float64) if emb.dtype == np.float32 else \
        synth.bf16_bits_to_f32(emb).astype(np.float64)
    P = e @ W.astype(np.float64) @ e.T                   # P[a, b] = e_a^T W e_b
    G = idx.shape[0]
    best, best_path = None, None
    scores = {}
    for ranks in itertools.product(range(16), repeat=G):
        s = sum(float(logp[i, k]) for i, k in enumerate(ranks))
        if anchor is not None:
            s += P[anchor, idx[0, ranks[0]]]
        for i in range(1, G):
            s += P[idx[i - 1, ranks[i - 1]], idx[i, ranks[i]]]
        scores[ranks] = s
        if best is None or s > best:
            best = s
    return best, scores


@pytest.mark.parametrize("G", [1, 2, 3, 4])
@pytest.mark.parametrize("with_anchor", [True, False])
def test_matches_brute_force(orc, G, with_anchor):
    idx, logp, anchor, emb, W = _problem(10 + G, 2, G)
    W = W * 8  # make the pair term decide often
    a = anchor if with_anchor else None
    tok, rank, score = orc.pair_select(idx, logp, a, emb, W)
    for b in range(2):
        best, scores = _brute(idx[b], logp[b], None if a is None else a[b], emb, W)
        assert abs(score[b] - best) < 1e-9
        # unique optimum in random data: the returned path is it
        optimal = [r for r, s in scores.items() if s > best - 1e-9]
        assert len(optimal) == 1
        assert tuple(rank[b]) == optimal[0]
        np.testing.assert_array_equal(tok[b], idx[b][np.arange(G), rank[b]])


def test_exact_ties_choose_reverse_lexicographic_smallest(orc):
    """All logp equal and a pair term of a few exactly-representable levels: the
    oracle's tie rule returns the optimal path whose rank vector is smallest
    when compared from the last position backwards."""
    G, V, d = 3, 40, 2
    rng = np.random.default_rng(3)
    idx = np.stack([rng.choice(V, 16, replace=False) for _ in range(G)]).astype(np.int32)[None]
    logp = np.full((1, G, 16), -1.0, np.float32)
    emb = np.zeros((V, d), np.float32)
    emb[:, 0] = rng.integers(0, 2, V)           # one-hot-ish integer embeddings
    emb[:, 1] = 1 - emb[:, 0]
    W = np.array([[1.0, 0.0], [0.0, 0.0]], np.float32)   # pair = 1 iff both have e_0
    tok, rank, score = orc.pair_select(idx, logp, None, emb, W)
    best, scores = _brute(idx[0], logp[0], None, emb, W)
    assert score[0] == best
    optimal = [r for r, s in scores.items() if s == best]
    assert len(optimal) > 1
    expect = min(optimal, key=lambda r: tuple(reversed(r)))
    assert tuple(rank[0]) == expect


def test_zero_W_picks_top1(orc):
    idx, logp, anchor, emb, W = _problem(4, 3, 7)
    tok, rank, score = orc.pair_select(idx, logp, anchor, emb, np.zeros_like(W))
    np.testing.assert_array_equal(rank, 0)
    np.testing.assert_allclose(score, logp[:, :, 0].astype(np.float64).sum(axis=1), rtol=1e-12)


def test_zero_W_equal_logp_picks_rank0(orc):
    idx, logp, anchor, emb, W = _problem(5, 2, 5, ties=True)
    _, rank, _ = orc.pair_select(idx, logp, anchor, emb, np.zeros_like(W))
    np.testing.assert_array_equal(rank, 0)


def test_bilinear_orientation_anchor(orc):
    """pair(a, b) = e_a^T W e_b, not e_b^T W e_a: with e_anchor = u0, a candidate
    with e = u1 and W[0][1] = 10 the anchor term lifts that candidate."""
    V, d = 32, 2
    emb = np.zeros((V, d), np.float32)
    emb[0] = [1, 0]                 # anchor token
    emb[5] = [1, 0]                 # rank-0 candidate
    emb[9] = [0, 1]                 # rank-1 candidate
    idx = np.array([[[5, 9] + list(range(10, 24))]], np.int32)
    logp = np.array([[[-1.0, -1.5] + [-9.0] * 14]], np.float32)
    W = np.array([[0.0, 10.0], [0.0, 0.0]], np.float32)
    tok, rank, score = orc.pair_select(idx, logp, np.array([0], np.int32), emb, W)
    assert rank[0, 0] == 1 and tok[0, 0] == 9
    assert score[0] == pytest.approx(-1.5 + 10.0, abs=1e-12)
    # the transposed weight makes the anchor term vanish for token 9
    tok, rank, score = orc.pair_select(idx, logp, np.array([0], np.int32), emb, W.T.copy())
    assert rank[0, 0] == 0
    # without the anchor the term is absent
    tok, rank, score = orc.pair_select(idx, logp, None, emb, W)
    assert rank[0, 0] == 0 and score[0] == pytest.approx(-1.0, abs=1e-12)


def test_huge_entry_forces_a_pair_between_positions(orc):
    """W[0][1] huge, e(c[2][7]) = u0 and e(c[3][4]) = u1: the best path must use
    rank 7 at position 2 and rank 4 at position 3; the orientation matters."""
    d, G = 2, 5
    rng = np.random.default_rng(8)
    V = 2 + 16 * G  # every candidate token distinct across positions
    idx = rng.permutation(np.arange(2, V)).reshape(1, G, 16).astype(np.int32)
    emb = np.zeros((V, d), np.float32)
    emb[idx[0, 2, 7]] = [1, 0]
    emb[idx[0, 3, 4]] = [0, 1]
    logp = np.sort(rng.standard_normal((1, G, 16)).astype(np.float32) - 3, axis=2)[:, :, ::-1].copy()
    W = np.array([[0.0, 1000.0], [0.0, 0.0]], np.float32)
    _, rank, _ = orc.pair_select(idx, logp, None, emb, W)
    assert rank[0, 2] == 7 and rank[0, 3] == 4
    np.testing.assert_array_equal(np.delete(rank[0], [2, 3]), 0)
    _, rank, _ = orc.pair_select(idx, logp, None, emb, W.T.copy())
    np.testing.assert_array_equal(rank[0], 0)


def test_rescore_equals_path_score_and_bf16(orc):
    w = synth.WORKLOADS["tiny"]
    idx, logp, anchor, emb, W = _problem(12, 2, 7, V=300, d=16)
    bits = synth.to_bf16_bits(emb)
    for e in (emb, bits):
        tok, rank, score = orc.pair_select(idx, logp, anchor, e, W)
        re = orc.path_rescore(idx, logp, anchor, e, W, rank)
        np.testing.assert_allclose(re, score, rtol=1e-13, atol=1e-13)
        # and any other path scores no higher
        other = rank.copy()
        other[:, 3] = (other[:, 3] + 1) % 16
        assert np.all(orc.path_rescore(idx, logp, anchor, e, W, other) <= score + 1e-12)
    assert w.G == 7
