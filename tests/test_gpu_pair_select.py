"""GPU parity of dflash2_pair_select against the CPU oracle (tamsi page,
"L’idée, sans le papier"; myaiexp page, "主な機能"; PSI page, "Résumé":
bilinear adjacent-pair scores and the best coherent path).

Both sides get identical inputs: the candidate lists and log-probabilities
come from the oracle's top-16 (rounded to fp32), never from the GPU.  The
path must equal the oracle's, except where the oracle's own rescore of the
GPU path is within 1e-5 * (1 + |best|) of the best (a counted near-tie);
path_score within 1e-5 relative.  bf16 tables run both implementations
(dflash2_pair_select_ex): the CUDA-core one and the tensor-core one (F = E W on
tcgen05 with W split into three bf16 planes)."""
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


def run_and_check(orc, idx, logp, anchor, emb, W, ties=None, impl=dfl.SELECT_AUTO):
    need_cuda()
    tok, rank, score = dfl.pair_select(to_dev(idx), to_dev(logp),
                                       None if anchor is None else to_dev(anchor),
                                       to_dev(emb), to_dev(W), impl=impl)
    torch.cuda.synchronize()
    assert dfl.device_errors() == 0
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


IMPLS = [dfl.SELECT_SIMT, dfl.SELECT_TENSOR]


@pytest.mark.parametrize("name,B", [("b1", 1), ("b8", 8), ("b32", 32), ("ctx16", 8)])
@pytest.mark.parametrize("impl", IMPLS)
def test_full_vocab(orc, name, B, impl):
    w = synth.WORKLOADS[name]
    sel = synth.gen_selector(w)
    idx, logp, anchor = oracle_inputs(orc, w, B)
    ties = run_and_check(orc, idx, logp, anchor, sel.emb, sel.W, impl=impl)
    print("near-ties:", ties.report())


@pytest.mark.parametrize("G", [1, 2, 5, 8, 9, 15, 16, 31])
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
    for impl in (IMPLS if dt == "bf16" else [dfl.SELECT_AUTO]):
        run_and_check(orc, idx, logp, anchor, emb, W, impl=impl)
        run_and_check(orc, idx, logp, None, emb, W, impl=impl)


def test_tensor_path_needs_a_bf16_table():
    need_cuda()
    idx = torch.zeros((1, 2, 16), dtype=torch.int32, device="cuda")
    logp = torch.zeros((1, 2, 16), dtype=torch.float32, device="cuda")
    emb = torch.zeros((100, 64), dtype=torch.float32, device="cuda")
    W = torch.zeros((64, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(dfl.DFlash2Error) as e:
        dfl.pair_select(idx, logp, None, emb, W, impl=dfl.SELECT_TENSOR)
    assert e.value.status == 2  # DFLASH2_EDTYPE


def test_exact_ties_resolve_like_the_oracle(orc):
    """Equal logp and W = 0: every path ties; both sides return rank 0."""
    rng = np.random.default_rng(9)
    B, G, V, d = 3, 7, 500, 64
    idx = np.stack([np.stack([rng.choice(V, 16, replace=False) for _ in range(G)])
                    for _ in range(B)]).astype(np.int32)
    logp = np.full((B, G, 16), -2.0, np.float32)
    emb = (rng.standard_normal((V, d)) / 8).astype(np.float32)
    W = np.zeros((d, d), np.float32)
    anchor = rng.integers(0, V, B).astype(np.int32)
    run_and_check(orc, idx, logp, anchor, emb, W)
    embb = synth.to_bf16_bits(emb)
    for impl in IMPLS:
        run_and_check(orc, idx, logp, anchor, embb, W, impl=impl)


def test_tensor_path_one_hot_embeddings_fix_the_orientation(orc):
    """One-hot bf16 embeddings make pair(a, b) = W[a][b] exactly: the tensor
    path must use W, not W^T, and split W's fp32 values into planes without
    loss (W entries with more mantissa bits than bf16 holds)."""
    need_cuda()
    rng = np.random.default_rng(31)
    d, V, B, G = 64, 64, 4, 3
    emb = synth.to_bf16_bits(np.eye(V, d, dtype=np.float32))
    W = (rng.standard_normal((d, d)) * (1 + 2 ** -20)).astype(np.float32)
    idx = np.stack([np.stack([rng.choice(V, 16, replace=False) for _ in range(G)])
                    for _ in range(B)]).astype(np.int32)
    logp = np.zeros((B, G, 16), np.float32)
    anchor = rng.integers(0, V, B).astype(np.int32)
    for impl in IMPLS:
        tok, rank, score = (to_host(t) for t in dfl.pair_select(
            to_dev(idx), to_dev(logp), to_dev(anchor), to_dev(emb), to_dev(W), impl=impl))
        for b in range(B):
            expect = W[anchor[b], tok[b, 0]] + sum(W[tok[b, i - 1], tok[b, i]] for i in range(1, G))
            assert abs(score[b] - expect) <= 1e-6 * (1 + abs(expect)), (impl, b)
        otok, orank, oscore = orc.pair_select(idx, logp, anchor, emb, W)
        np.testing.assert_array_equal(rank, orank)


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


@pytest.mark.parametrize("impl", IMPLS)
def test_named_implementation_is_batch_invariant(orc, impl):
    """With the implementation named, a sequence's path and score are the same
    bits in a batch of 40 (above the automatic threshold) and alone."""
    need_cuda()
    w = synth.WORKLOADS["b32"]
    sel = synth.gen_selector(w)
    idx, logp, anchor = oracle_inputs(orc, w, 40)
    E, Wd = to_dev(sel.emb), to_dev(sel.W)
    full = [to_host(t) for t in dfl.pair_select(to_dev(idx), to_dev(logp), to_dev(anchor), E, Wd,
                                                impl=impl)]
    for s in (0, 17, 39):
        one = [to_host(t) for t in dfl.pair_select(to_dev(idx[s:s + 1]), to_dev(logp[s:s + 1]),
                                                   to_dev(anchor[s:s + 1]), E, Wd, impl=impl)]
        for a, o in zip(full, one):
            np.testing.assert_array_equal(a[s:s + 1], o)
