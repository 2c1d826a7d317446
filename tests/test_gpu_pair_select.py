"""GPU parity of dflash2_pair_select against the CPU oracle (tamsi page,
"L’idée, sans le papier"; myaiexp page, "主な機能"; PSI page, "Résumé":
bilinear adjacent-pair scores and the best coherent path).

Both sides get identical inputs: the candidate lists and log-probabilities
come from the oracle's top-16 (rounded to fp32), never from the GPU.  The
path must equal the oracle's, except where the oracle's own rescore of the
GPU path is within 1e-5 * (1 + |best|) of the best (a counted near-tie);
path_score within 1e-5 relative."""
import numpy as np
import pytest
import torch

import block_draft_verification_b200 as dfl
import synth
from parity import count_compared, PATH_BAND, RTOL_F32, NearTies, assert_close, gpu, need_cuda, to_dev, to_host

pytestmark = gpu


def oracle_inputs(orc, w, B, first=0):
    b = synth.gen_batch(w, B=B, first=first)
    idx, _, logp, _ = orc.topk_softmax(b.draft.reshape(-1, w.V), w.inv_temperature)
    G = w.G
    return idx.reshape(B, G, 16), logp.astype(np.float32).reshape(B, G, 16), b.anchor


def run_and_check(orc, idx, logp, anchor, emb, W, ties=None):
    need_cuda()
    tok, rank, score = dfl.pair_select(to_dev(idx), to_dev(logp),
                                       None if anchor is None else to_dev(anchor),
                                       to_dev(emb), to_dev(W))
    torch.cuda.synchronize()
    tok, rank, score = to_host(tok), to_host(rank), to_host(score)
    otok, orank, oscore = orc.pair_select(idx, logp, anchor, emb, W)
    assert_close(score, oscore, RTOL_F32, "path_score")
    ties = ties if ties is not None else NearTies()
    count_compared("path", len(rank))
    diff = np.flatnonzero((rank != orank).any(axis=1))
    if diff.size:
        resc = orc.path_rescore(idx[diff], logp[diff], None if anchor is None else anchor[diff],
                                emb, W, rank[diff])
        margin = np.abs(resc - oscore[diff]) / (1.0 + np.abs(oscore[diff]))
        assert np.all(margin < PATH_BAND), (diff, margin)
        ties.add("path", diff.size)
    same = np.setdiff1d(np.arange(len(rank)), diff)
    np.testing.assert_array_equal(tok[same], otok[same])
    np.testing.assert_array_equal(tok, np.take_along_axis(idx, rank[..., None], 2)[..., 0])
    return ties


def test_tiny(orc):
    w = synth.WORKLOADS["tiny"]
    sel = synth.gen_selector(w)
    idx, logp, anchor = oracle_inputs(orc, w, 1)
    run_and_check(orc, idx, logp, anchor, sel.emb, sel.W)
    run_and_check(orc, idx, logp, None, sel.emb, sel.W)


@pytest.mark.parametrize("name,B", [("b1", 1), ("b8", 8), ("b32", 32), ("ctx16", 8)])
def test_full_vocab(orc, name, B):
    w = synth.WORKLOADS[name]
    sel = synth.gen_selector(w)
    idx, logp, anchor = oracle_inputs(orc, w, B)
    ties = run_and_check(orc, idx, logp, anchor, sel.emb, sel.W)
    print("near-ties:", ties.report())


@pytest.mark.parametrize("G", [1, 2, 5, 31])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_shapes_and_pair_heavy_weights(orc, G, d, dt):
    """Random candidate lists with W scaled up so the pair term decides often."""
    rng = np.random.default_rng(G * 1000 + d)
    B, V = 5, 3000
    idx = np.stack([np.stack([rng.choice(V, 16, replace=False) for _ in range(G)])
                    for _ in range(B)]).astype(np.int32)
    logp = np.sort(rng.standard_normal((B, G, 16)).astype(np.float32) - 3, axis=2)[:, :, ::-1].copy()
    emb = (rng.standard_normal((V, d)) / np.sqrt(d)).astype(np.float32)
    if dt == "bf16":
        emb = synth.to_bf16_bits(emb)
    W = (rng.standard_normal((d, d)) * 4 / np.sqrt(d)).astype(np.float32)
    anchor = rng.integers(0, V, B).astype(np.int32)
    run_and_check(orc, idx, logp, anchor, emb, W)
    run_and_check(orc, idx, logp, None, emb, W)


def test_exact_ties_resolve_like_the_oracle(orc):
    """Equal logp and W = 0: every path ties; both sides return rank 0."""
    rng = np.random.default_rng(9)
    B, G, V, d = 3, 7, 500, 64
    idx = np.stack([np.stack([rng.choice(V, 16, replace=False) for _ in range(G)])
                    for _ in range(B)]).astype(np.int32)
    logp = np.full((B, G, 16), -2.0, np.float32)
    emb = (rng.standard_normal((V, d)) / 8).astype(np.float32)
    W = np.zeros((d, d), np.float32)
    run_and_check(orc, idx, logp, rng.integers(0, V, B).astype(np.int32), emb, W)


def test_batch_invariance(orc):
    need_cuda()
    w = synth.WORKLOADS["b8"]
    sel = synth.gen_selector(w)
    idx, logp, anchor = oracle_inputs(orc, w, 8)
    E, Wd = to_dev(sel.emb), to_dev(sel.W)
    full = [to_host(t) for t in dfl.pair_select(to_dev(idx), to_dev(logp), to_dev(anchor), E, Wd)]
    one = [to_host(t) for t in dfl.pair_select(to_dev(idx[3:4]), to_dev(logp[3:4]),
                                               to_dev(anchor[3:4]), E, Wd)]
    for a, o in zip(full, one):
        np.testing.assert_array_equal(a[3:4], o)
