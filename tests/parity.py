"""Helpers of the GPU parity tests: device transfer of the seeded inputs, the
floating-point tolerance rule and the near-tie accounting.

Tolerances (fixed by the build's target): fp32 outputs within 1e-5 relative,
bf16 outputs within 2e-2 relative, measured as
    |gpu - oracle| <= rtol * (|oracle| + rms(oracle))
(the rms floor keeps values near zero from turning the rule into 0/0).
Integer outputs (indices, paths, accepted lengths, tokens) are bit-exact,
except decisions that a float rounding can flip, which are counted as
near-ties when the oracle's own margin is below the stated band:
    accept/reject:   |u - r| < 1e-6
    residual draw:   distance from t to the chosen interval's end < 1e-6 * R
    Viterbi path:    oracle rescore of the GPU path within 1e-5 * (1 + |best|)
"""
import numpy as np
import pytest
import torch

RTOL_F32 = 1e-5
RTOL_BF16 = 2e-2
ACCEPT_BAND = 1e-6
DRAW_BAND = 1e-6
PATH_BAND = 1e-5

gpu = pytest.mark.gpu


def need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def to_dev(a, bf16=None):
    """numpy -> CUDA tensor; uint16 arrays are bf16 bit patterns."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


def to_host(t):
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def bf16_to_f64(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def assert_close(gpu_vals, oracle_vals, rtol, what=""):
    g = np.asarray(gpu_vals, np.float64)
    o = np.asarray(oracle_vals, np.float64)
    assert g.shape == o.shape, (what, g.shape, o.shape)
    rms = float(np.sqrt(np.mean(o * o))) if o.size else 0.0
    err = np.abs(g - o)
    bound = rtol * (np.abs(o) + rms)
    bad = err > bound
    if bad.any():
        i = np.flatnonzero(bad.ravel())[0]
        raise AssertionError("%s: %d/%d outside rtol %g; first at %d: gpu %r oracle %r"
                             % (what, bad.sum(), bad.size, rtol, i, g.ravel()[i], o.ravel()[i]))


# Every near-tie excused in this test session, per kind (printed at the end of
# the run by conftest.py, so the counts are part of the run's record).
SESSION_NEAR_TIES = {}
SESSION_COMPARED = {}


def count_compared(kind, n):
    """Record n integer decisions of `kind` compared with the oracle."""
    SESSION_COMPARED[kind] = SESSION_COMPARED.get(kind, 0) + int(n)


class NearTies:
    """Counts mismatches that the stated bands excuse; anything else fails."""

    def __init__(self):
        self.counts = {}

    def add(self, kind, n=1):
        self.counts[kind] = self.counts.get(kind, 0) + n
        SESSION_NEAR_TIES[kind] = SESSION_NEAR_TIES.get(kind, 0) + n

    def report(self):
        return ", ".join("%s=%d" % kv for kv in sorted(self.counts.items())) or "none"
