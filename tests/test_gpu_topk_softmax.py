"""GPU parity of dflash2_topk_softmax against the CPU oracle (tamsi page,
"L’idée, sans le papier"; myaiexp page, "主な機能": the 16 best candidates
per drafted position and their probabilities).

idx is bit-exact (exact compares on the input values, lowest index on
ties, -0 == +0); prob, logp and logz within 1e-5 relative."""
import numpy as np
import pytest
import torch

import block_draft_verification_b200 as dfl
import synth
from parity import RTOL_F32, assert_close, gpu, need_cuda, to_dev, to_host

pytestmark = gpu


def check_rows(orc, x_np, invT=1.0, rows_sel=None, x_dev=None):
    """Run the GPU call on all rows; compare the oracle on rows_sel (all by default)."""
    need_cuda()
    xd = to_dev(x_np) if x_dev is None else x_dev
    idx, prob, logp, logz = dfl.topk_softmax(xd, invT)
    torch.cuda.synchronize()
    idx, prob, logp, logz = (to_host(t) for t in (idx, prob, logp, logz))
    sel = np.arange(x_np.shape[0]) if rows_sel is None else np.asarray(rows_sel)
    oi, op, ol, oz = orc.topk_softmax(np.ascontiguousarray(x_np[sel]), invT)
    np.testing.assert_array_equal(idx[sel], oi)
    assert_close(prob[sel], op, RTOL_F32, "prob")
    assert_close(logp[sel], ol, RTOL_F32, "logp")
    assert_close(logz[sel], oz, RTOL_F32, "logz")
    return idx, prob, logp, logz


def test_tiny_fp32(orc):
    w = synth.WORKLOADS["tiny"]
    b = synth.gen_batch(w)
    check_rows(orc, b.draft.reshape(-1, w.V), w.inv_temperature)


@pytest.mark.parametrize("name", ["b1", "ctx16"])
def test_full_vocab_bf16(orc, name):
    w = synth.WORKLOADS[name]
    b = synth.gen_batch(w, B=1)
    check_rows(orc, b.draft.reshape(-1, w.V), w.inv_temperature)


def test_b32_full_size_sampled_rows(orc):
    """The bench's launch: all 224 rows of the concurrency-32 workload in one
    call; the oracle checks a seeded sample of 12 rows (incl. first and last)."""
    w = synth.WORKLOADS["b32"]
    b = synth.gen_batch(w)
    x = b.draft.reshape(-1, w.V)
    rng = np.random.default_rng(0)
    sel = np.unique(np.concatenate([[0, x.shape[0] - 1], rng.choice(x.shape[0], 10, replace=False)]))
    check_rows(orc, x, 1.0, sel)


@pytest.mark.parametrize("V", [16, 17, 31, 100, 4099, 16384, 16385, 2 * 16384 + 5, 151936])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_ragged_vocab(orc, V, dt):
    rng = np.random.default_rng(V)
    x = (rng.standard_normal((5, V)) * 3).astype(np.float32)
    if dt == "bf16":
        x = synth.to_bf16_bits(x)
    check_rows(orc, x, 0.8)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_misaligned_rows_take_the_scalar_path(orc, dt):
    """row_stride = V = 4099 odd: rows are not 16-byte aligned."""
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((4, 4099)) * 2).astype(np.float32)
    if dt == "bf16":
        x = synth.to_bf16_bits(x)
    check_rows(orc, x, 1.0)


def test_strided_rows(orc):
    need_cuda()
    rng = np.random.default_rng(4)
    wide = synth.to_bf16_bits((rng.standard_normal((6, 20000)) * 2).astype(np.float32))
    dev = to_dev(wide)[:, 8:8 + 17000]      # 16-byte aligned start, stride 20000
    check_rows(orc, np.ascontiguousarray(wide[:, 8:8 + 17000]), 1.0, x_dev=dev)


def test_ties_signed_zeros_uniform_and_spikes(orc):
    V = 3 * 16384 + 77
    rng = np.random.default_rng(5)
    rows = []
    rows.append(np.full(V, 0.5, np.float32))                                    # uniform
    r = np.full(V, -1.0, np.float32)
    r[rng.choice(V, 40, replace=False)] = rng.choice([-0.0, 0.0], 40)           # +-0 maxima
    rows.append(r)
    r = rng.integers(-3, 4, V).astype(np.float32)                               # massive ties
    rows.append(r)
    r = np.zeros(V, np.float32)
    r[np.sort(rng.choice(V, 17, replace=False))] = 7.0                          # 17 maxima across chunks
    rows.append(r)
    r = (rng.standard_normal(V) * 3).astype(np.float32)
    r[V - 1] = 50.0                                                             # spike in the tail
    rows.append(r)
    x = np.stack(rows)
    check_rows(orc, x, 1.0)
    check_rows(orc, synth.to_bf16_bits(x), 1.3)


def test_fewer_than_16_elements_in_the_last_chunk(orc):
    V = 16384 + 5
    rng = np.random.default_rng(6)
    x = (rng.standard_normal((3, V)) * 2).astype(np.float32)
    x[:, -5:] = 40.0 + np.arange(5)          # the 5 largest live in the short chunk
    check_rows(orc, x, 1.0)


def test_batch_invariance(orc):
    """A row's outputs are bit-identical whatever batch it is computed in."""
    need_cuda()
    w = synth.WORKLOADS["b32"]
    b = synth.gen_batch(w, B=8)
    x = to_dev(b.draft.reshape(-1, w.V))
    full = [to_host(t) for t in dfl.topk_softmax(x)]
    perm = torch.randperm(x.shape[0], generator=torch.Generator().manual_seed(1))
    shuf = [to_host(t) for t in dfl.topk_softmax(x[perm.cuda()].contiguous())]
    one = [to_host(t) for t in dfl.topk_softmax(x[5:6].contiguous())]
    for a, s, o in zip(full, shuf, one):
        np.testing.assert_array_equal(a[perm.numpy()], s)
        np.testing.assert_array_equal(a[5:6], o)


def test_output_guard_bands(orc):
    """Outputs land exactly in their slots: canaries around them survive."""
    need_cuda()
    rng = np.random.default_rng(7)
    x = to_dev(synth.to_bf16_bits((rng.standard_normal((3, 5000)) * 2).astype(np.float32)))
    pad = 64
    canary_i = torch.full((3 * 16 + 2 * pad,), -12345, dtype=torch.int32, device="cuda")
    canary_f = torch.full((3 * 16 + 2 * pad,), 777.0, dtype=torch.float32, device="cuda")
    canary_f2 = canary_f.clone()
    canary_z = torch.full((3 + 2 * pad,), 777.0, dtype=torch.float32, device="cuda")
    out = (canary_i[pad:pad + 48].view(3, 16), canary_f[pad:pad + 48].view(3, 16),
           canary_f2[pad:pad + 48].view(3, 16), canary_z[pad:pad + 3])
    dfl.topk_softmax(x, 1.0, out=out)
    torch.cuda.synchronize()
    for c, fill in ((canary_i, -12345), (canary_f, 777.0), (canary_f2, 777.0)):
        h = to_host(c)
        assert np.all(h[:pad] == fill) and np.all(h[pad + 48:] == fill)
    hz = to_host(canary_z)
    assert np.all(hz[:pad] == 777.0) and np.all(hz[pad + 3:] == 777.0)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("invT", [1.0, 1.7])
def test_large_magnitude_logits(orc, dt, invT):
    """Logits near +-1000 and a one-hot row: the exponent of the row maximum
    must come out as exactly 0, not as the rounding error of max * c (up to
    6e-5 at this size, which would scale every probability by 2^6e-5)."""
    rng = np.random.default_rng(77)
    V = 2 * 16384 + 7
    rows = [rng.standard_normal(V) * 2.0 + off for off in (-900.0, 300.0, 1000.0)]
    hot = np.zeros(V)
    hot[12345] = 1000.0
    rows.append(hot)
    x = np.stack(rows).astype(np.float32)
    if dt == "bf16":
        x = synth.to_bf16_bits(x)
    check_rows(orc, x, invT)


@pytest.mark.parametrize("name", ["tiny", "b8"])
def test_row_stats(orc, name):
    """dflash2_topk_softmax_ex: row_max is the row maximum exactly, row_lse =
    logz - row_max * invT, the other outputs equal the plain call's bit for bit."""
    need_cuda()
    w = synth.WORKLOADS[name]
    b = synth.gen_batch(w)
    x = b.draft.reshape(-1, w.V)
    for invT in (w.inv_temperature, 0.7):
        X = to_dev(x)
        plain = [to_host(t) for t in dfl.topk_softmax(X, invT)]
        got = [to_host(t) for t in dfl.topk_softmax(X, invT, stats=True)]
        torch.cuda.synchronize()
        for a, g in zip(plain, got[:4]):
            np.testing.assert_array_equal(a, g)
        xf = synth.bf16_bits_to_f32(x) if x.dtype == np.uint16 else x
        np.testing.assert_array_equal(got[4], xf.max(axis=1))
        _, _, _, ologz = orc.topk_softmax(x, invT)
        assert_close(got[5], ologz - xf.max(axis=1).astype(np.float64) * invT, RTOL_F32, "row_lse")


def test_many_rows_memset_control(orc):
    """More rows than the 64 KB control area holds (10,000 rows: a counter and a
    shared top-16 bound each), so the call clears its control words with a
    memset; rows of one chunk and of two (V = 4,100 fp32: 2,048 + 2,048 + 4).
    Two calls on one workspace: the second must not inherit the first's
    bounds."""
    need_cuda()
    rng = np.random.default_rng(10000)
    ws = dfl.Workspace(torch.device("cuda"))
    for V in (64, 4100):
        rows = 10000 if V == 64 else 2000
        for rep in range(2):
            x = (rng.standard_normal((rows, V)) * (1.0 + rep)).astype(np.float32)
            idx, prob, logp, logz = (to_host(a) for a in
                                     dfl.topk_softmax(to_dev(x), 1.0, ws=ws))
            oi, op, ol, oz = orc.topk_softmax(x, 1.0)
            np.testing.assert_array_equal(idx, oi)
            assert_close(prob, op, RTOL_F32, "prob")
            assert_close(logz, oz, RTOL_F32, "logz")
    assert dfl.device_errors() == 0
