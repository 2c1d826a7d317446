"""GPU parity of dflash2_verify_sample_trunc, the sampling verify of top-k /
top-p truncated distributions (latenode page, "Preguntas frecuentes": the Qwen
targets are sampled at temperature 1.0, top-p 0.95, top-k 20), against the
CPU oracle's orc_verify_sample_trunc on the same inputs and Philox uniforms.

Bit-exact on n_accept and out_tok, except counted near-ties: an accept test
with |u - r| < 1e-6, a draw within 1e-6 R of its interval's end, and a top-p
cut whose cumulative sum is within 1e-9 of top_p (the oracle reports each
margin; the kernel sums in another order).  The uniforms are bit-identical;
the ratios agree within 1e-5 relative (both +inf where q~(d) = 0 < p~(d))."""
import numpy as np
import pytest
import torch

import block_draft_verification_b200 as dfl
import synth
from parity import (ACCEPT_BAND, DRAW_BAND, NearTies, count_compared, gpu, need_cuda, to_dev,
                    to_host)

pytestmark = gpu
TRUNC_BAND = 1e-9


def check_trunc(orc, target, draft, d, seed, step, seq_id=None, invT=1.0, top_k=20, top_p=0.95,
                q_mode=0, ties=None, ws=None):
    need_cuda()
    ties = ties if ties is not None else NearTies()
    top_p = float(np.float32(top_p))  # the value the kernel compares (the ABI takes a float)
    sid = None if seq_id is None else to_dev(np.asarray(seq_id, np.uint32).view(np.int32))
    n, out, ratio, u = dfl.verify_sample_trunc(
        to_dev(target), None if (draft is None or q_mode == 1) else to_dev(draft), to_dev(d),
        seed, step, sid, invT, top_k, top_p, q_mode, debug=True, ws=ws)
    torch.cuda.synchronize()
    assert dfl.device_errors() == 0
    n, out, ratio, u = to_host(n), to_host(out), to_host(ratio), to_host(u)
    on, oout, oratio, ou, macc, mres, mtr = orc.verify_sample_trunc(
        target, None if q_mode == 1 else draft, d, seed, step, seq_id, invT, top_k, top_p, q_mode)
    np.testing.assert_array_equal(u.astype(np.float64), ou)
    B = len(n)
    count_compared("accept", B)
    count_compared("draw", B)
    count_compared("trunc", B)
    o32 = oratio.astype(np.float32).astype(np.float64)   # +inf beyond the float range, as the kernel
    g = ratio.astype(np.float64)
    for b in range(B):
        if mtr[b] < TRUNC_BAND:
            ties.add("trunc")
            continue
        inf_o, inf_g = np.isinf(o32[b]), np.isinf(g[b])
        assert np.array_equal(inf_o, inf_g), (b, g[b], oratio[b])
        fin = ~inf_o
        err = np.abs(g[b][fin] - oratio[b][fin])
        assert np.all(err <= 1e-5 * np.abs(oratio[b][fin]) + 1e-30), (b, g[b], oratio[b])
        if n[b] != on[b]:
            assert macc[b] < ACCEPT_BAND, (b, n[b], on[b], macc[b])
            ties.add("accept")
        elif not np.array_equal(out[b], oout[b]):
            assert mres[b] < DRAW_BAND, (b, out[b], oout[b], mres[b])
            np.testing.assert_array_equal(out[b, :n[b]], oout[b, :n[b]])
            ties.add("draw")
    return on, ties


def drafted(w, b, rng):
    """The drafter's own top-1 tokens, corrupted at a random position, so
    acceptance spreads over 0..G."""
    q = b.draft
    x = synth.bf16_bits_to_f32(q) if q.dtype == np.uint16 else q
    d = x.argmax(axis=2).astype(np.int32)
    B, G = d.shape
    cut = rng.integers(0, G + 1, B)
    for i in range(B):
        if cut[i] < G:
            d[i, cut[i]] = rng.integers(0, x.shape[2])
    return d


@pytest.mark.parametrize("name", ["tiny", "b8", "ctx16", "b32"])
@pytest.mark.parametrize("q_mode", [0, 1])
def test_trunc_workloads(orc, name, q_mode):
    """The pages' setting (top-k 20, top-p 0.95, T = 1) on every workload; the
    concurrency-32 batch in full (the launch the benchmark times)."""
    w = synth.WORKLOADS[name]
    b = synth.gen_batch(w)
    d = drafted(w, b, np.random.default_rng(5))
    ties = NearTies()
    for step in range(2 if name == "b32" else 3):
        check_trunc(orc, b.target, b.draft, d, w.seed, step, b.seq_id, w.inv_temperature, 20,
                    0.95, q_mode, ties)
    print(name, "near-ties:", ties.report())


@pytest.mark.parametrize("V", [8, 20, 33, 100, 5000, 40001])
@pytest.mark.parametrize("top_k,top_p", [(1, 0.95), (5, 0.5), (20, 0.95), (32, 0.9),
                                         (32, 1.0), (7, 1.0)])
def test_trunc_small_vocab_many_sequences(orc, V, top_k, top_p):
    """Many sequences over small and ragged vocabularies (V below the 32 keys,
    below and above top_k, not a multiple of a chunk): rejections, residual
    and bonus draws, top-k beyond V, top-p off."""
    rng = np.random.default_rng(V * 100 + top_k)
    B, G = 48, 3
    t = (rng.standard_normal((B, G + 1, V)) * 1.5).astype(np.float32)
    q = (t[:, :G] + rng.standard_normal((B, G, V)) * 0.7).astype(np.float32)
    d = np.argmax(q, axis=2).astype(np.int32)
    d[::3, 1] = rng.integers(0, V, len(d[::3]))
    sid = (np.arange(B, dtype=np.uint32) * 7919 + 12345).astype(np.uint32)
    ties = NearTies()
    for q_mode in (0, 1):
        check_trunc(orc, t, q, d, 99, 5, sid, 1.0, top_k, top_p, q_mode, ties)
        check_trunc(orc, synth.to_bf16_bits(t), synth.to_bf16_bits(q), d, 99, 6, sid, 0.7,
                    top_k, top_p, q_mode, ties)
    print("near-ties:", ties.report())


def test_trunc_ties_and_temperature(orc):
    """Equal logits across the top-k boundary (index order decides), integer
    logits, and a temperature that sharpens the rows."""
    rng = np.random.default_rng(17)
    B, G, V = 32, 4, 3000
    t = rng.integers(-3, 4, (B, G + 1, V)).astype(np.float32)
    q = rng.integers(-3, 4, (B, G, V)).astype(np.float32)
    d = rng.integers(0, 64, (B, G)).astype(np.int32)
    ties = NearTies()
    for invT in (1.0, 2.5):
        for q_mode in (0, 1):
            check_trunc(orc, t, q, d, 3, 1, None, invT, 20, 0.95, q_mode, ties)
    print("near-ties:", ties.report())


def test_trunc_matches_plain_verify_when_off(orc):
    """top_k = 32 >= V and top_p = 1 keep every token: the verdicts of the
    untruncated oracle (orc_verify_sample) on the same inputs, up to its own
    near-tie margins."""
    need_cuda()
    rng = np.random.default_rng(23)
    B, G, V = 64, 5, 24
    t = (rng.standard_normal((B, G + 1, V)) * 2).astype(np.float32)
    q = (t[:, :G] + rng.standard_normal((B, G, V))).astype(np.float32)
    d = rng.integers(0, V, (B, G)).astype(np.int32)
    for q_mode in (0, 1):
        n, out = dfl.verify_sample_trunc(to_dev(t), to_dev(q) if q_mode == 0 else None, to_dev(d),
                                         1, 2, None, 1.0, 32, 1.0, q_mode)
        torch.cuda.synchronize()
        n, out = to_host(n), to_host(out)
        on, oout, _, _, macc, mres = orc.verify_sample(t, q if q_mode == 0 else None, d, 1, 2,
                                                       None, 1.0, q_mode)
        for b in range(B):
            if n[b] != on[b]:
                assert macc[b] < ACCEPT_BAND, (b, n[b], on[b])
            elif not np.array_equal(out[b], oout[b]):
                assert mres[b] < DRAW_BAND, (b, out[b], oout[b])


def test_trunc_two_calls_share_a_workspace(orc):
    """Consecutive calls on one workspace (its control words left zero by
    every call, its segment lists overwritten)."""
    w = synth.WORKLOADS["b8"]
    ws = dfl.Workspace(torch.device("cuda"))
    for first in (0, 8):
        b = synth.gen_batch(w, first=first)
        d = drafted(w, b, np.random.default_rng(first))
        check_trunc(orc, b.target, b.draft, d, 4, first, b.seq_id, ws=ws)
