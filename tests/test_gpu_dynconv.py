"""GPU parity of dflash2_dynconv2 against the CPU oracle (tamsi page, "L’idée,
sans le papier": two-tap conv before/after each attention and MLP; myaiexp
page, "主な機能": 2-tap dynamic convolution).

fp32 outputs within 1e-5 relative, bf16 outputs within 2e-2 relative."""
import numpy as np
import pytest
import torch

import block_draft_verification_b200 as dfl
import synth
from parity import RTOL_BF16, RTOL_F32, assert_close, bf16_to_f64, gpu, need_cuda, to_dev, to_host

pytestmark = gpu


def run(x, xp, w):
    need_cuda()
    out = dfl.dynconv2(to_dev(x), to_dev(xp), to_dev(w))
    torch.cuda.synchronize()
    assert dfl.device_errors() == 0     # no bounded wait of the tensor-core kernel ran out
    return to_host(out)


def as_f64(a):
    return bf16_to_f64(a) if a.dtype == np.uint16 else a.astype(np.float64)


def test_tiny_fp32(orc):
    w = synth.WORKLOADS["tiny"]
    c = synth.gen_conv(w)
    out = run(c.x, c.x_prev, c.w_tap)
    assert_close(out, orc.dynconv2(c.x, c.x_prev, c.w_tap), RTOL_F32, "tiny")


def test_b1_bf16(orc):
    w = synth.WORKLOADS["b1"]
    c = synth.gen_conv(w)
    out = run(c.x, c.x_prev, c.w_tap)
    assert_close(as_f64(out), orc.dynconv2(c.x, c.x_prev, c.w_tap), RTOL_BF16, "b1")


def test_b32_full_size_sampled_sequences(orc):
    """The bench's launch (32 x 8 tokens, H = 5,120); the oracle checks
    sequences 0, 13 and 31 (their x_prev and tokens are independent)."""
    w = synth.WORKLOADS["b32"]
    c = synth.gen_conv(w)
    out = as_f64(run(c.x, c.x_prev, c.w_tap))
    for b in (0, 13, 31):
        ref = orc.dynconv2(c.x[b:b + 1], c.x_prev[b:b + 1], c.w_tap)
        assert_close(out[b:b + 1], ref, RTOL_BF16, "seq %d" % b)


@pytest.mark.parametrize("B,T,H", [(1, 1, 64), (3, 5, 64), (2, 7, 192), (5, 3, 320), (1, 40, 128),
                                   (40, 8, 128), (3, 200, 64)])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_ragged_shapes(orc, B, T, H, dt):
    rng = np.random.default_rng(B * 100 + T * 10 + H)
    x = rng.standard_normal((B, T, H)).astype(np.float32)
    xp = rng.standard_normal((B, H)).astype(np.float32)
    wt = (rng.standard_normal((2 * H, H)) / np.sqrt(H)).astype(np.float32)
    if dt == "bf16":
        x, xp, wt = synth.to_bf16_bits(x), synth.to_bf16_bits(xp), synth.to_bf16_bits(wt)
    out = run(x, xp, wt)
    assert_close(as_f64(out), orc.dynconv2(x, xp, wt), RTOL_F32 if dt == "f32" else RTOL_BF16, dt)


def test_special_weights_exact(orc):
    """W = [I; 0]: out = x + x*x; W = [0; I]: out = x_t + x_t * x_{t-1}."""
    rng = np.random.default_rng(8)
    B, T, H = 2, 4, 64
    x = rng.integers(-3, 4, (B, T, H)).astype(np.float32)
    xp = rng.integers(-3, 4, (B, H)).astype(np.float32)
    eye, zero = np.eye(H, dtype=np.float32), np.zeros((H, H), np.float32)
    for wt in (np.concatenate([eye, zero]), np.concatenate([zero, eye])):
        out = run(x, xp, wt)
        np.testing.assert_array_equal(out.astype(np.float64), orc.dynconv2(x, xp, wt))


@pytest.mark.parametrize("name,B", [("b1", 1), ("b8", 8), ("b32", 32)])
def test_packed_weights_give_the_same_bits(orc, name, B):
    """dflash2_dynconv2_packed (the tap weights packed once, dflash2_dynconv2_pack)
    reads the same bytes into the same shared-memory stages as dflash2_dynconv2:
    every output bit is equal; and it matches the oracle on sampled sequences."""
    need_cuda()
    w = synth.WORKLOADS[name]
    c = synth.gen_conv(w, B=B)
    x, xp, wt = to_dev(c.x), to_dev(c.x_prev), to_dev(c.w_tap)
    pk = dfl.PackedTap(wt)
    a = dfl.dynconv2(x, xp, wt)
    b = dfl.dynconv2(x, xp, pk)
    torch.cuda.synchronize()
    assert dfl.device_errors() == 0
    np.testing.assert_array_equal(to_host(a), to_host(b))
    s = [0, B - 1]
    assert_close(as_f64(to_host(b)[s]), orc.dynconv2(c.x[s], c.x_prev[s], c.w_tap), RTOL_BF16,
                 "packed")


@pytest.mark.parametrize("B,T,H", [(1, 1, 64), (3, 5, 192), (2, 40, 320)])
def test_packed_weights_ragged_shapes(orc, B, T, H):
    need_cuda()
    rng = np.random.default_rng(B * 1000 + T * 10 + H)
    x = synth.to_bf16_bits(rng.standard_normal((B, T, H)).astype(np.float32))
    xp = synth.to_bf16_bits(rng.standard_normal((B, H)).astype(np.float32))
    wt = synth.to_bf16_bits((rng.standard_normal((2 * H, H)) / np.sqrt(H)).astype(np.float32))
    out = dfl.dynconv2(to_dev(x), to_dev(xp), dfl.PackedTap(to_dev(wt)))
    torch.cuda.synchronize()
    assert dfl.device_errors() == 0
    np.testing.assert_array_equal(to_host(out), run(x, xp, wt))
    assert_close(as_f64(to_host(out)), orc.dynconv2(x, xp, wt), RTOL_BF16, "packed ragged")
