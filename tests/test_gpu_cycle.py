"""Chained-cycle parity: the GPU runs top-16 -> pair select -> verify on its own
outputs, the oracle runs the same chain on its own outputs, and the final
tokens are compared.  A sequence whose selected path differs by a counted
near-tie may legitimately verify differently downstream; every other
sequence must agree bit for bit (or by a counted accept/draw near-tie)."""
import numpy as np
import pytest
import torch

import block_draft_verification_b200 as dfl
import synth
from parity import count_compared, ACCEPT_BAND, DRAW_BAND, PATH_BAND, NearTies, gpu, need_cuda, to_dev, to_host

pytestmark = gpu


@pytest.mark.parametrize("name,sampling", [("tiny", False), ("tiny", True), ("b1", False),
                                           ("b8", True), ("b32", False), ("ctx16", False),
                                           ("ctx16", True)])
def test_chained_cycle(orc, name, sampling):
    need_cuda()
    w = synth.WORKLOADS[name]
    b = synth.gen_batch(w)
    sel = synth.gen_selector(w)
    B, G, V = b.target.shape[0], w.G, w.V
    T, Q = to_dev(b.target), to_dev(b.draft)
    idx, prob, logp, logz = dfl.topk_softmax(Q.view(-1, V), w.inv_temperature)
    tok, rank, score = dfl.pair_select(idx.view(B, G, 16), logp.view(B, G, 16), to_dev(b.anchor),
                                       to_dev(sel.emb), to_dev(sel.W))
    if sampling:
        n, out = dfl.verify_sample(T, Q, tok, w.seed, 0, to_dev(b.seq_id.view(np.int32)),
                                   w.inv_temperature)
    else:
        n, out = dfl.verify_greedy(T, tok)
    torch.cuda.synchronize()
    tok, rank, n, out = to_host(tok), to_host(rank), to_host(n), to_host(out)

    oidx, _, ologp, _ = orc.topk_softmax(b.draft.reshape(-1, V), w.inv_temperature)
    oidx, ologp = oidx.reshape(B, G, 16), ologp.astype(np.float32).reshape(B, G, 16)
    otok, orank, oscore = orc.pair_select(oidx, ologp, b.anchor, sel.emb, sel.W)
    if sampling:
        on, oout, _, _, macc, mres = orc.verify_sample(b.target, b.draft, otok, w.seed, 0,
                                                       b.seq_id, w.inv_temperature)
    else:
        on, oout = orc.verify_greedy(b.target, otok)
        macc = mres = np.zeros(B)
    ties = NearTies()
    count_compared("path", B)
    count_compared("accept" if sampling else "greedy", B)
    if sampling:
        count_compared("draw", B)
    for s in range(B):
        if not np.array_equal(rank[s], orank[s]):
            re = orc.path_rescore(oidx[s:s + 1], ologp[s:s + 1], b.anchor[s:s + 1], sel.emb, sel.W,
                                  rank[s:s + 1])[0]
            assert abs(re - oscore[s]) / (1 + abs(oscore[s])) < PATH_BAND, s
            ties.add("path")
            continue
        if n[s] != on[s]:
            assert sampling and macc[s] < ACCEPT_BAND, (s, n[s], on[s])
            ties.add("accept")
        elif not np.array_equal(out[s], oout[s]):
            assert sampling and mres[s] < DRAW_BAND, (s, out[s], oout[s])
            ties.add("draw")
    print(name, "sampling" if sampling else "greedy", "mean acceptance %.2f" % (on + 1).mean(),
          "near-ties:", ties.report())


def test_top16_oracle_paths(orc):
    """The acceptance study's three paths (bench.py --acceptance): the top-1
    and top-16 oracle paths and their greedy verification equal the oracle's
    chain exactly; per sequence the oracle path is accepted at least as far as
    any path drawn from the same 16 candidates (at the first position whose
    target token is not among them every such path mismatches)."""
    need_cuda()
    import bench
    w = synth.WORKLOADS["b1"]
    b = synth.gen_batch(w, B=8)
    sel = synth.gen_selector(w)
    B, G, V = b.target.shape[0], w.G, w.V
    T = to_dev(b.target)
    paths, hit16, hit1 = bench.acceptance_paths(dfl, torch, T, to_dev(b.draft), to_dev(b.anchor),
                                                to_dev(sel.emb), to_dev(sel.W), w.inv_temperature)
    n = {k: to_host(dfl.verify_greedy(T, p)[0]) for k, p in paths.items()}
    torch.cuda.synchronize()

    oidx = orc.topk_softmax(b.draft.reshape(-1, V), w.inv_temperature)[0].reshape(B, G, 16)
    tidx = orc.topk_softmax(b.target[:, :G].reshape(-1, V), w.inv_temperature)[0].reshape(B, G, 16)
    t = tidx[:, :, 0]
    ohit = (oidx == t[:, :, None]).any(-1)
    otop1 = oidx[:, :, 0].astype(np.int32)
    opath = np.where(ohit, t, otop1).astype(np.int32)
    np.testing.assert_array_equal(to_host(paths["top1"]), otop1)
    np.testing.assert_array_equal(to_host(paths["top16_oracle"]), opath)
    np.testing.assert_array_equal(to_host(hit16), ohit)
    np.testing.assert_array_equal(n["top1"], orc.verify_greedy(b.target, otop1)[0])
    np.testing.assert_array_equal(n["top16_oracle"], orc.verify_greedy(b.target, opath)[0])
    assert np.all(n["top16_oracle"] >= n["top1"]) and np.all(n["top16_oracle"] >= n["selector"])
    first_miss = np.where((~ohit).any(1), (~ohit).argmax(1), G)
    np.testing.assert_array_equal(n["top16_oracle"], first_miss)
