"""dflash2_topk_softmax_noalloc, the allocation-free top-16 entry point, called
through the C ABI and checked against dflash2_topk_softmax (the entry point
that takes a caller workspace) on the same inputs, and against the CPU oracle
directly (indices bit-exact, probabilities within 1e-5 relative).

It exists for callers that cannot give this library device memory: an
inference engine that reserved nearly all of the GPU for its own pools and
lets no plugin call cudaMalloc, or a latency-critical path where cudaMalloc
could synchronise the device.  Its scratch is one fixed array inside the
library that every call reuses, so the test makes two calls in a row on
different inputs (the second call must not see the first call's leftovers).
"""
import ctypes as C

import numpy as np
import pytest
import torch

import block_draft_verification_b200 as dfl
import synth
from parity import RTOL_F32, assert_close, gpu, need_cuda, to_dev, to_host

pytestmark = gpu

EWORKSPACE = 4


def _entry():
    f = dfl.lib().dflash2_topk_softmax_noalloc
    f.argtypes = [C.c_void_p, C.c_int, C.c_int64, C.c_int64, C.c_int64, C.c_float, C.c_void_p,
                  C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]
    f.restype = C.c_int
    return f


def _noalloc(x, inv_t):
    rows, V = x.shape
    dev = x.device
    idx = torch.empty((rows, 16), dtype=torch.int32, device=dev)
    prob = torch.empty((rows, 16), dtype=torch.float32, device=dev)
    logp = torch.empty((rows, 16), dtype=torch.float32, device=dev)
    logz = torch.empty((rows,), dtype=torch.float32, device=dev)
    rc = _entry()(C.c_void_p(x.data_ptr()), 1 if x.dtype == torch.bfloat16 else 0, rows, V,
                  x.stride(0), inv_t, C.c_void_p(idx.data_ptr()), C.c_void_p(prob.data_ptr()),
                  C.c_void_p(logp.data_ptr()), C.c_void_p(logz.data_ptr()),
                  C.c_void_p(torch.cuda.current_stream(dev).cuda_stream))
    assert rc == 0, dfl.status_string(rc)
    return idx, prob, logp, logz


def _same(got, ref):
    gi, gp, gl, gz = (to_host(t) for t in got)
    ri, rp, rl, rz = (to_host(t) for t in ref)
    np.testing.assert_array_equal(gi, ri)
    assert_close(gp, rp, RTOL_F32, "prob")
    assert_close(gl, rl, RTOL_F32, "logp")
    assert_close(gz, rz, RTOL_F32, "logz")


def _matches_oracle(got, host_rows, inv_t, orc):
    gi, gp, gl, gz = (to_host(t) for t in got)
    oi, op, ol, oz = orc.topk_softmax(host_rows, inv_t)
    np.testing.assert_array_equal(gi, oi)
    assert_close(gp, op, RTOL_F32, "prob vs oracle")
    assert_close(gl, ol, RTOL_F32, "logp vs oracle")
    assert_close(gz, oz, RTOL_F32, "logz vs oracle")


@pytest.mark.parametrize("name,B", [("tiny", 1), ("b32", 4)])
def test_noalloc_matches_workspace_entry_on_two_calls(name, B, orc):
    need_cuda()
    w = synth.WORKLOADS[name]
    hosts = [synth.gen_batch(w, B=B, first=f).draft.reshape(-1, w.V) for f in (0, B)]
    for host_rows in hosts:
        x = to_dev(host_rows)
        ref = dfl.topk_softmax(x, w.inv_temperature)
        got = _noalloc(x, w.inv_temperature)
        torch.cuda.synchronize()
        assert dfl.device_errors() == 0
        _same(got, ref)
        _matches_oracle(got, host_rows, w.inv_temperature, orc)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    need_cuda()
    x = torch.zeros((2, 151936), dtype=torch.bfloat16, device="cuda")
    out = torch.empty(64, dtype=torch.float32, device="cuda")
    p = C.c_void_p(out.data_ptr())
    # 3,000 rows of 151,936 need more than the built-in array: refused before any launch
    rc = _entry()(C.c_void_p(x.data_ptr()), 1, 3000, 151936, 151936, 1.0, p, p, p, p,
                  C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == EWORKSPACE
    torch.cuda.synchronize()


def test_noalloc_refuses_bad_arguments_then_works(orc):
    """Bad scalars, pointers and alignment are refused with the same codes as
    the workspace entry; a correct call right after is still correct."""
    need_cuda()
    w = synth.WORKLOADS["tiny"]
    host_rows = synth.gen_batch(w, B=1, first=3).draft.reshape(-1, w.V)
    x = to_dev(host_rows)
    out = torch.empty(64, dtype=torch.float32, device="cuda")
    p = C.c_void_p(out.data_ptr())
    h = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    rows, V = x.shape
    bad = [
        (C.c_void_p(x.data_ptr()), 0, rows, V, V, float("nan"), p, p, p, p, h),  # EINVAL
        (C.c_void_p(x.data_ptr()), 0, rows, V, V, 1.0, None, p, p, p, h),          # EINVAL
        (C.c_void_p(x.data_ptr() + 2), 0, rows, V, V, 1.0, p, p, p, p, h),         # EALIGN
        (C.c_void_p(x.data_ptr()), 7, rows, V, V, 1.0, p, p, p, p, h),             # EDTYPE
    ]
    assert [_entry()(*a) for a in bad] == [1, 1, 6, 2]
    got = _noalloc(x, w.inv_temperature)
    torch.cuda.synchronize()
    assert dfl.device_errors() == 0
    _matches_oracle(got, host_rows, w.inv_temperature, orc)
