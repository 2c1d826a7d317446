"""GPU parity of dflash2_verify_greedy and dflash2_verify_sample against the
CPU oracle (tamsi page, "Les chiffres qui comptent sur Qwen3.8-27B": greedy is
exactly the target, rejection sampling keeps its distribution; latenode page,
"El desacuerdo...": acceptance length = tokens completed per verify step).

Greedy: n_accept and out_tok bit-exact.  Sampling: the Philox uniforms are
bit-identical; ratios within 1e-5 relative; n_accept and out_tok bit-exact
except counted near-ties (accept |u - r| < 1e-6, draw margin < 1e-6 * R)."""
import json
import os

import numpy as np
import pytest
import torch

import block_draft_verification_b200 as dfl
import synth
from parity import (ACCEPT_BAND, count_compared, DRAW_BAND, RTOL_F32, NearTies, assert_close, gpu, need_cuda,
                    to_dev, to_host)

pytestmark = gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "greedy_cases.json")


def drafted_tokens(orc, w, b, rng, mode):
    """Drafted tokens for a batch: the oracle's own selected path ('path'),
    or the target argmax corrupted at a random position ('cut'), which spreads
    n_accept over 0..G."""
    G = w.G
    B = b.target.shape[0]
    if mode == "path":
        sel = synth.gen_selector(w)
        idx, _, logp, _ = orc.topk_softmax(b.draft.reshape(-1, b.draft.shape[-1]), w.inv_temperature)
        tok, _, _ = orc.pair_select(idx.reshape(B, G, 16), logp.astype(np.float32).reshape(B, G, 16),
                                    b.anchor, sel.emb, sel.W)
        return tok
    t = b.target.astype(np.float64) if b.target.dtype == np.float32 else \
        synth.bf16_bits_to_f32(b.target).astype(np.float64)
    amax = t.argmax(axis=2)[:, :G].astype(np.int32)
    cut = rng.integers(0, G + 1, B)
    for i in range(B):
        if cut[i] < G:
            amax[i, cut[i]] = (amax[i, cut[i]] + 1 + rng.integers(0, 100)) % t.shape[2]
    return amax


# ------------------------------------------------------------------ greedy
def check_greedy(orc, target, draft_tok):
    """Both greedy entries (the full verify and the early-exit one) against
    the oracle: bit-exact n_accept and out_tok."""
    need_cuda()
    on, oout = orc.verify_greedy(target, draft_tok)
    for early in (False, True):
        n, out = dfl.verify_greedy(to_dev(target), to_dev(draft_tok), early_exit=early)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(to_host(n), on)
        np.testing.assert_array_equal(to_host(out), oout)
    return on


def test_greedy_golden_cases(orc):
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        t = np.array(c["target"], np.float32)
        d = np.array(c["draft_tok"], np.int32)
        for arr in (t, synth.to_bf16_bits(t)):
            n = check_greedy(orc, arr, d)
            np.testing.assert_array_equal(n, c["n"])


@pytest.mark.parametrize("name", ["tiny", "b1", "b8", "b32", "ctx16"])
@pytest.mark.parametrize("mode", ["path", "cut"])
def test_greedy_workloads(orc, name, mode):
    w = synth.WORKLOADS[name]
    if mode == "path" and name == "b32":
        pytest.skip("the oracle path of 32 sequences is covered by the cycle test")
    b = synth.gen_batch(w)
    d = drafted_tokens(orc, w, b, np.random.default_rng(1), mode)
    n = check_greedy(orc, b.target, d)
    if mode == "cut":
        assert len(set(n.tolist())) > 1 or len(n) == 1


@pytest.mark.parametrize("V", [1, 2, 7, 16385, 40001])
def test_greedy_ragged(orc, V):
    rng = np.random.default_rng(V)
    B, G = 6, 5
    t = rng.integers(-4, 5, (B, G + 1, V)).astype(np.float32)   # ties everywhere
    d = t.argmax(axis=2)[:, :G].astype(np.int32)
    d[::2, 2] = (d[::2, 2] + 1) % V
    check_greedy(orc, t, d)
    check_greedy(orc, synth.to_bf16_bits(t), d)


def test_greedy_early_exit_every_mismatch_row(orc):
    """The first mismatch at every row 0..G (and none), many sequences per
    row, a workspace shared by consecutive calls: the early exit skips the
    rows after it and still returns the full verify's results."""
    rng = np.random.default_rng(12)
    B, G, V = 64, 7, 20000
    t = (rng.standard_normal((B, G + 1, V)) * 3).astype(np.float32)
    d = t.argmax(axis=2)[:, :G].astype(np.int32)
    cut = np.arange(B) % (G + 1)
    for i in range(B):
        if cut[i] < G:
            d[i, cut[i]] = (d[i, cut[i]] + 1 + i) % V
            d[i, cut[i] + 1:] = rng.integers(0, V, G - cut[i] - 1)
    ws = dfl.Workspace(torch.device("cuda"))
    on, oout = orc.verify_greedy(t, d)
    np.testing.assert_array_equal(on, np.minimum(cut, G))
    for arr in (t, synth.to_bf16_bits(t), t):
        n, out = dfl.verify_greedy(to_dev(arr), to_dev(d), ws=ws, early_exit=True)
        torch.cuda.synchronize()
        o2 = orc.verify_greedy(arr, d)
        np.testing.assert_array_equal(to_host(n), o2[0])
        np.testing.assert_array_equal(to_host(out), o2[1])
    assert dfl.device_errors() == 0


def test_greedy_max_block(orc):
    rng = np.random.default_rng(2)
    B, G, V = 3, 31, 5000
    t = (rng.standard_normal((B, G + 1, V)) * 3).astype(np.float32)
    d = t.argmax(axis=2)[:, :G].astype(np.int32)
    d[1, 30] = (d[1, 30] + 1) % V
    n = check_greedy(orc, synth.to_bf16_bits(t), d)
    assert n[0] == G or n[0] < G


# ------------------------------------------------------------------ sampling
def draft_stats(orc, draft, invT):
    """The drafter normalisers the fused cycle reuses: the row maximum (exact)
    and ln sum exp((x - max) invT) in fp64 (scipy's logsumexp; any V, also
    below the 16 candidates the top-16 needs), each rounded to float as
    dflash2_topk_softmax_ex writes them."""
    from scipy.special import logsumexp
    B, G, V = draft.shape
    rows = draft.reshape(-1, V)
    x = (synth.bf16_bits_to_f32(rows) if rows.dtype == np.uint16 else rows).astype(np.float64)
    mx = x.max(axis=1)
    lse = logsumexp((x - mx[:, None]) * invT, axis=1)
    return mx.astype(np.float32).reshape(B, G), lse.astype(np.float32).reshape(B, G)


def check_sample(orc, target, draft, draft_tok, seed, step, seq_id=None, invT=1.0, q_mode=0,
                 ties=None, fused=False):
    """fused: the drafter normalisers are given (dflash2_verify_sample_ex) and
    the draft rows are read only at the drafted tokens and the drawn row; the
    oracle is the same."""
    need_cuda()
    ties = ties if ties is not None else NearTies()
    stats = None
    if fused and draft is not None:
        stats = tuple(to_dev(a) for a in draft_stats(orc, draft, invT))
    n, out, ratio, u = dfl.verify_sample(to_dev(target), None if draft is None else to_dev(draft),
                                         to_dev(draft_tok), seed, step,
                                         None if seq_id is None else to_dev(seq_id.view(np.int32)),
                                         invT, q_mode, debug=True, draft_stats=stats)
    torch.cuda.synchronize()
    n, out, ratio, u = to_host(n), to_host(out), to_host(ratio), to_host(u)
    on, oout, oratio, ou, macc, mres = orc.verify_sample(target, draft, draft_tok, seed, step,
                                                         seq_id, invT, q_mode)
    np.testing.assert_array_equal(u.astype(np.float64), ou)       # Philox: bit-identical
    assert_close(ratio, oratio, RTOL_F32, "ratio")
    count_compared("accept", len(n))
    count_compared("draw", len(n))
    for b in range(len(n)):
        if n[b] != on[b]:
            assert macc[b] < ACCEPT_BAND, (b, n[b], on[b], macc[b])
            ties.add("accept")
        elif not np.array_equal(out[b], oout[b]):
            assert mres[b] < DRAW_BAND, (b, out[b], oout[b], mres[b])
            np.testing.assert_array_equal(out[b, :n[b]], oout[b, :n[b]])
            ties.add("draw")
    return on, ties


@pytest.mark.parametrize("name", ["tiny", "b8", "b32", "ctx16"])
@pytest.mark.parametrize("q_mode,fused", [(0, False), (1, False), (0, True)])
def test_sample_workloads(orc, name, q_mode, fused):
    w = synth.WORKLOADS[name]
    B = min(w.B, 8) if name == "b32" else w.B
    b = synth.gen_batch(w, B=B)
    d = drafted_tokens(orc, w, b, np.random.default_rng(3), "cut")
    ties = NearTies()
    for step in range(3):
        check_sample(orc, b.target, b.draft if q_mode == 0 else None, d, w.seed, step, b.seq_id,
                     w.inv_temperature, q_mode, ties, fused)
    print("near-ties:", ties.report())


@pytest.mark.parametrize("fused", [False, True])
def test_sample_b32_full_batch_sampled(orc, fused):
    """The bench's launch (B=32); the oracle checks all 32 sequences once."""
    w = synth.WORKLOADS["b32"]
    b = synth.gen_batch(w)
    d = drafted_tokens(orc, w, b, np.random.default_rng(4), "cut")
    check_sample(orc, b.target, b.draft, d, 7, 11, b.seq_id, fused=fused)


@pytest.mark.parametrize("V", [2, 8, 100, 16385, 33000])
@pytest.mark.parametrize("invT", [1.0, 0.5, 1.7])
def test_sample_small_vocab_many_sequences(orc, V, invT):
    """Many sequences over small vocabularies: rejections, residual draws and
    bonus draws all occur; seq_id far from b."""
    rng = np.random.default_rng(V)
    B, G = 64, 3
    t = (rng.standard_normal((B, G + 1, V)) * 1.5).astype(np.float32)
    q = (t[:, :G] + rng.standard_normal((B, G, V))).astype(np.float32)
    d = rng.integers(0, V, (B, G)).astype(np.int32)
    sid = (np.arange(B, dtype=np.uint32) * 7919 + 12345).astype(np.uint32)
    ties = NearTies()
    on, _ = check_sample(orc, t, q, d, 99, 5, sid, invT, 0, ties)
    check_sample(orc, t, None, d, 99, 5, sid, invT, 1, ties)
    check_sample(orc, synth.to_bf16_bits(t), synth.to_bf16_bits(q), d, 99, 6, sid, invT, 0, ties)
    check_sample(orc, t, q, d, 99, 7, sid, invT, 0, ties, fused=True)
    check_sample(orc, synth.to_bf16_bits(t), synth.to_bf16_bits(q), d, 99, 8, sid, invT, 0, ties,
                 fused=True)
    print("near-ties:", ties.report())


def test_sample_special_cases(orc):
    rng = np.random.default_rng(5)
    B, G, V = 32, 4, 300
    t = rng.standard_normal((B, G + 1, V)).astype(np.float32)
    d = rng.integers(0, V, (B, G)).astype(np.int32)
    for fused in (False, True):
        on, _ = check_sample(orc, t, t[:, :G].copy(), d, 1, 1, fused=fused)  # p = q: accept all
        assert np.all(on == G)
        t2 = t.copy()
        t2[np.arange(B), 0, d[:, 0]] = -1000.0                   # p(d_0) = 0: reject at 0
        on, _ = check_sample(orc, t2, t[:, :G].copy(), d, 1, 2, fused=fused)
        assert np.all(on == 0)
    t3 = np.zeros((B, G + 1, V), np.float32)
    for j in range(G):
        t3[np.arange(B), j, d[:, j]] = 1000.0                    # one-hot, p(d) = 1: accept
    on, _ = check_sample(orc, t3, None, d, 1, 3, q_mode=1)
    assert np.all(on == G)


def test_sample_large_magnitude_logits(orc):
    """Logits offset by +-700: ratios and draws must not pick up the rounding
    error of max * c in the exponent reference."""
    rng = np.random.default_rng(41)
    B, G, V = 16, 5, 20000
    off = np.where(np.arange(B) % 2 == 0, 700.0, -700.0)[:, None, None]
    t = (rng.standard_normal((B, G + 1, V)) * 1.5 + off).astype(np.float32)
    q = (t[:, :G] + rng.standard_normal((B, G, V)) * 0.3).astype(np.float32)
    d = np.argmax(q, axis=2).astype(np.int32)
    ties = NearTies()
    check_sample(orc, t, q, d, 3, 1, None, 1.0, 0, ties)
    check_sample(orc, t, None, d, 3, 2, None, 1.0, 1, ties)
    check_sample(orc, t, q, d, 3, 1, None, 1.0, 0, ties, fused=True)
    print("near-ties:", ties.report())


def test_sample_batch_invariance(orc):
    need_cuda()
    w = synth.WORKLOADS["b8"]
    b = synth.gen_batch(w)
    d = drafted_tokens(orc, w, b, np.random.default_rng(6), "cut")
    T, Q, D = to_dev(b.target), to_dev(b.draft), to_dev(d)
    sid = to_dev(b.seq_id.view(np.int32))
    full = [to_host(x) for x in dfl.verify_sample(T, Q, D, 3, 4, sid, debug=True)]
    one = [to_host(x) for x in dfl.verify_sample(T[2:3].contiguous(), Q[2:3].contiguous(),
                                                 D[2:3].contiguous(), 3, 4, sid[2:3].contiguous(),
                                                 debug=True)]
    for a, o in zip(full, one):
        np.testing.assert_array_equal(a[2:3], o)


def test_sample_fused_batch_invariance(orc):
    """The fused cycle: a sequence's outputs do not depend on its batch."""
    need_cuda()
    w = synth.WORKLOADS["b8"]
    b = synth.gen_batch(w)
    d = drafted_tokens(orc, w, b, np.random.default_rng(6), "cut")
    T, Q, D = to_dev(b.target), to_dev(b.draft), to_dev(d)
    sid = to_dev(b.seq_id.view(np.int32))
    mx, lse = (to_dev(a) for a in draft_stats(orc, b.draft, w.inv_temperature))
    full = [to_host(x) for x in dfl.verify_sample(T, Q, D, 3, 4, sid, debug=True,
                                                 draft_stats=(mx, lse))]
    one = [to_host(x) for x in dfl.verify_sample(T[2:3].contiguous(), Q[2:3].contiguous(),
                                                 D[2:3].contiguous(), 3, 4, sid[2:3].contiguous(),
                                                 debug=True,
                                                 draft_stats=(mx[2:3].contiguous(),
                                                              lse[2:3].contiguous()))]
    for a, o in zip(full, one):
        np.testing.assert_array_equal(a[2:3], o)


def test_fused_cycle_matches_topk_stats(orc):
    """End to end: the statistics come from dflash2_topk_softmax_ex on the
    GPU (not the oracle) and feed dflash2_verify_sample_ex; the oracle's
    unfused verify decides."""
    need_cuda()
    w = synth.WORKLOADS["b8"]
    b = synth.gen_batch(w)
    d = drafted_tokens(orc, w, b, np.random.default_rng(8), "cut")
    B, G, V = b.draft.shape
    Q = to_dev(b.draft)
    _, _, _, _, mx, lse = dfl.topk_softmax(Q.view(B * G, V), w.inv_temperature, stats=True)
    n, out, ratio, u = dfl.verify_sample(to_dev(b.target), Q, to_dev(d), w.seed, 9,
                                         to_dev(b.seq_id.view(np.int32)), w.inv_temperature,
                                         debug=True, draft_stats=(mx.view(B, G), lse.view(B, G)))
    torch.cuda.synchronize()
    on, oout, oratio, ou, macc, mres = orc.verify_sample(b.target, b.draft, d, w.seed, 9, b.seq_id,
                                                         w.inv_temperature, 0)
    assert_close(to_host(ratio), oratio, RTOL_F32, "ratio")
    n, out = to_host(n), to_host(out)
    for s in range(B):
        if n[s] != on[s]:
            assert macc[s] < ACCEPT_BAND
        elif not np.array_equal(out[s], oout[s]):
            assert mres[s] < DRAW_BAND


def test_sample_fallback_when_residual_empty(orc):
    """A rejected row whose residual max(0, p - q) is empty makes the draw use
    p_n (the reading for an empty residual).  Made here on purpose through the
    fused entry: p_0 is a spike; the draft row equals the target row except a
    large logit at the drafted token d_0 (q(d_0) ~ 5e-5, p(d_0) ~ 0: row 0
    rejects), and the given normaliser is 1 too small, so q = e q_true covers
    p everywhere (q(spike) ~ e > p(spike) = 1): the residual is empty and the
    draw must return the spike's token."""
    need_cuda()
    rng = np.random.default_rng(17)
    B, G, V = 6, 2, 25000                       # three draw chunks per row
    t = rng.standard_normal((B, G + 1, V)).astype(np.float32)
    spike = rng.integers(0, V, B)
    t[np.arange(B), 0, spike] = 1000.0          # p_0 is one-hot at the spike
    d = np.zeros((B, G), np.int32)
    d[:, 0] = (spike + 1) % V                   # p_0(d_0) ~ exp(-1000): reject at 0
    d[:, 1] = spike
    q = t[:, :G].copy()
    q[np.arange(B), 0, d[:, 0]] = 990.0
    mx, lse = draft_stats(orc, q, 1.0)
    n, out = dfl.verify_sample(to_dev(t), to_dev(q), to_dev(d), 5, 1,
                               draft_stats=(to_dev(mx), to_dev(lse - 1.0)))[:2]
    torch.cuda.synchronize()
    n, out = to_host(n), to_host(out)
    np.testing.assert_array_equal(n, np.zeros(B, np.int32))
    np.testing.assert_array_equal(out[:, 0], spike.astype(np.int32))
    assert np.all(out[:, 1:] == -1)


@pytest.mark.parametrize("fused", [False, True])
def test_sample_many_sequences_memset_control(orc, fused):
    """More sequences than the 64 KB control area holds (B = 2,048: the finish
    queue alone needs 256 KB), so the call clears its control words with a
    memset; every V is one draw unit.  Two calls on one workspace: the second
    must not see the first's queue."""
    need_cuda()
    rng = np.random.default_rng(2048)
    B, G, V = 2048, 3, 64
    t = (rng.standard_normal((B, G + 1, V)) * 2.0).astype(np.float32)
    q = (t[:, :G] + rng.standard_normal((B, G, V)) * 0.5).astype(np.float32)
    d = np.argmax(q, axis=2).astype(np.int32)
    ws = dfl.Workspace(torch.device("cuda"))
    stats = tuple(to_dev(a) for a in draft_stats(orc, q, 1.0)) if fused else None
    ties = NearTies()
    for step in (0, 1):
        n, out = dfl.verify_sample(to_dev(t), to_dev(q), to_dev(d), 77, step, None, 1.0,
                                   ws=ws, draft_stats=stats)[:2]
        torch.cuda.synchronize()
        n, out = to_host(n), to_host(out)
        on, oout, _, _, macc, mres = orc.verify_sample(t, q, d, 77, step, None, 1.0, 0)
        count_compared("accept", B)
        count_compared("draw", B)
        for s in range(B):
            if n[s] != on[s]:
                assert macc[s] < ACCEPT_BAND, (s, n[s], on[s])
                ties.add("accept")
            elif not np.array_equal(out[s], oout[s]):
                assert mres[s] < DRAW_BAND, (s, out[s], oout[s])
                ties.add("draw")
    assert dfl.device_errors() == 0
    print("near-ties:", ties.report())
