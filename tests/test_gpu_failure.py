"""Failure detection on the device, without faulting the GPU.

1. A bounded wait that runs out.  The sampling verify's draw warps wait
   (bounded, one second) for a sequence to be decided.  The test makes that
   wait run out by corrupting one word on the host, before the call: the
   scan-unit counter of the last sequence starts at 2^30 instead of 0, so no
   publish of its scan units ever brings it to the expected count (a small
   offset could: a partial sum may land on it), the sequence is never decided
   and never queued.  Its draw warps then give up
   after the bound, set error flag 16 and return; the call returns, the host
   reads the flag, re-zeroes the workspace's 64 KB control area as the
   header asks, and the next call is correct (checked against the oracle).
2. Token ids outside [0, V): never used as an address.  The verifies treat
   such a drafted token as not accepted, the selector gives an out-of-range
   id a zero embedding, and each call sets error flag 32.
"""
import numpy as np
import torch

import block_draft_verification_b200 as dfl
import synth
from parity import gpu, need_cuda, to_dev, to_host

pytestmark = gpu

ERR_STREAM, ERR_INPUT = 16, 32
CONTROL_BYTES = 65536
# Sampling verify control words (workspace.cuh, sample layout): word 0 the
# finish-queue length, word 32 the count of warps done (one 128-byte line
# each), then one scan-unit counter per sequence from word 64.
SCAN_COUNTER_WORD0 = 64


def _sample_inputs(B=4):
    w = synth.WORKLOADS["tiny"]
    b = synth.gen_batch(w, B=B)
    rng = np.random.default_rng(11)
    d = rng.integers(0, w.V, (B, w.G)).astype(np.int32)
    return w, b, d


def _run_sample(w, b, d, ws, step=3):
    n, out, ratio, u = dfl.verify_sample(to_dev(b.target), to_dev(b.draft), to_dev(d), w.seed,
                                         step, to_dev(b.seq_id.view(np.int32)),
                                         w.inv_temperature, debug=True, ws=ws)
    torch.cuda.synchronize()
    return to_host(n), to_host(out)


def test_draw_wait_runs_out_then_workspace_recovers(orc):
    need_cuda()
    dfl.device_errors(clear=True)
    w, b, d = _sample_inputs()
    B = d.shape[0]
    dev = torch.device("cuda", 0)
    ws = dfl.Workspace(dev, dfl.workspace_bytes(B, w.G, w.V))
    # a clean call first: the oracle agrees, no flag
    n0, out0 = _run_sample(w, b, d, ws)
    on, oout, *_ = orc.verify_sample(b.target, b.draft, d, w.seed, 3, b.seq_id, w.inv_temperature)
    np.testing.assert_array_equal(n0, on)
    np.testing.assert_array_equal(out0, oout)
    assert dfl.device_errors() == 0
    # the last sequence's scan-unit counter starts at 2^30: it is never decided
    ctl = ws.buf[:CONTROL_BYTES].view(torch.int32)
    ctl[SCAN_COUNTER_WORD0 + B - 1] = 1 << 30
    torch.cuda.synchronize()
    n1, out1 = _run_sample(w, b, d, ws)  # returns after the one-second bound
    flags = dfl.device_errors(clear=True)
    assert flags & ERR_STREAM, flags
    # the sequences that were decided still carry their accepted prefix
    for s in range(B - 1):
        assert n1[s] == on[s]
        np.testing.assert_array_equal(out1[s, :on[s]], oout[s, :on[s]])
    # the host re-zeroes the control area; the same workspace is correct again
    ws.buf[:CONTROL_BYTES].zero_()
    n2, out2 = _run_sample(w, b, d, ws)
    np.testing.assert_array_equal(n2, on)
    np.testing.assert_array_equal(out2, oout)
    assert dfl.device_errors() == 0


def test_out_of_range_tokens_are_never_addresses(orc):
    need_cuda()
    dfl.device_errors(clear=True)
    w, b, d = _sample_inputs(B=4)
    V, G = w.V, w.G
    bad = d.copy()
    bad[0, 0] = V          # just past the row
    bad[1, 2] = -3         # negative
    bad[2, 4] = 2 ** 31 - 1
    # greedy: a bad token is a mismatch; the prefix before it is unchanged
    t = b.target
    greedy_ok = t.argmax(axis=2)[:, :G].astype(np.int32)
    gbad = greedy_ok.copy()
    gbad[0, 0], gbad[1, 2], gbad[2, 4] = V, -3, 2 ** 31 - 1
    n, out = dfl.verify_greedy(to_dev(t), to_dev(gbad))
    torch.cuda.synchronize()
    assert dfl.device_errors() & ERR_INPUT
    n, out = to_host(n), to_host(out)
    assert list(n) == [0, 2, 4, G]
    np.testing.assert_array_equal(out[3], orc.verify_greedy(t, greedy_ok)[1][3])
    for s, j in ((0, 0), (1, 2), (2, 4)):
        assert out[s, j] == t[s, j].argmax()           # the correction token
    # sampling: a bad token is rejected (r = 0); the sequences without one agree with the oracle
    for q_mode in (0, 1):
        n, out, ratio, u = dfl.verify_sample(to_dev(t), to_dev(b.draft) if q_mode == 0 else None,
                                             to_dev(bad), w.seed, 1, None, w.inv_temperature,
                                             q_mode, debug=True)
        torch.cuda.synchronize()
        assert dfl.device_errors() & ERR_INPUT
        n, out, ratio = to_host(n), to_host(out), to_host(ratio)
        assert n[0] == 0 and n[1] <= 2 and n[2] <= 4
        assert ratio[0, 0] == 0.0 and ratio[1, 2] == 0.0 and ratio[2, 4] == 0.0
        assert np.all((out[np.arange(4), n] >= 0) & (out[np.arange(4), n] < V))
        on, oout, *_ = orc.verify_sample(t[3:], None if q_mode else b.draft[3:], bad[3:], w.seed,
                                         1, np.array([3], np.uint32), w.inv_temperature, q_mode)
        assert n[3] == on[0]
    # selector: an out-of-range anchor is a zero embedding (no pair term before position 0)
    sel = synth.gen_selector(w)
    idx, _, logp, _ = orc.topk_softmax(b.draft.reshape(-1, V), w.inv_temperature)
    idx3 = idx.reshape(4, G, 16)
    lp3 = logp.astype(np.float32).reshape(4, G, 16)
    anchor = np.array([V + 7, -1, 5, 2 ** 31 - 1], np.int32)
    tok, rank, score = dfl.pair_select(to_dev(idx3), to_dev(lp3), to_dev(anchor),
                                       to_dev(sel.emb), to_dev(sel.W))
    torch.cuda.synchronize()
    assert dfl.device_errors() & ERR_INPUT
    otok, orank, _ = orc.pair_select(idx3, lp3, None, sel.emb, sel.W)   # no anchor term
    for s in (0, 1, 3):
        np.testing.assert_array_equal(to_host(rank)[s], orank[s])
    assert dfl.device_errors() == 0
