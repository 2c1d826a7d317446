"""The C ABI library loads on a machine without a GPU, exports every entry
point include/dflash2.h declares, and rejects bad arguments on the host with
the documented status codes before any CUDA call (none of these tests needs a
device: validation returns before anything is enqueued)."""
import ctypes as C
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")

OK, EINVAL, EDTYPE, ESHAPE, EWORKSPACE, ECUDA, EALIGN = range(7)


@pytest.fixture(scope="module")
def L():
    from block_draft_verification_b200 import build
    build.build()
    import block_draft_verification_b200 as d
    return d.lib()


def declared_symbols():
    names = set()
    for f in os.listdir(HEADER_DIR):
        if f.endswith(".h"):
            text = open(os.path.join(HEADER_DIR, f)).read()
            names |= set(re.findall(r"DFLASH2_API\s+[\w\s\*]+?\b(dflash2_\w+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported(L):
    names = declared_symbols()
    assert {"dflash2_topk_softmax", "dflash2_pair_select", "dflash2_verify_greedy",
            "dflash2_verify_sample", "dflash2_dynconv2"} <= names
    from block_draft_verification_b200 import LIB_PATH
    out = subprocess.run(["nm", "-D", "--defined-only", LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (dflash2_\w+)", out))
    assert names <= exported, names - exported
    # nothing but the declared ABI is exported under the dflash2_ prefix
    assert exported == names
    for n in names:
        assert getattr(L, n) is not None


def test_status_strings_and_version(L):
    import block_draft_verification_b200 as d
    for code in range(7):
        assert d.status_string(code).startswith("DFLASH2_")
    assert d.status_string(99) == "DFLASH2_UNKNOWN_STATUS"
    assert d.version() == (1, 0)


def test_workspace_bytes(L):
    import block_draft_verification_b200 as d
    assert d.workspace_bytes(1, 7, 151936) > 0
    assert d.workspace_bytes(32, 7, 151936) > d.workspace_bytes(8, 7, 151936)
    assert d.workspace_bytes(8, 15, 151936) > d.workspace_bytes(8, 7, 151936)
    assert d.workspace_bytes(1, 0, 100) == 0
    assert d.workspace_bytes(1, 32, 100) == 0
    assert d.workspace_bytes(-1, 7, 100) == 0
    assert d.workspace_bytes(0, 7, 100) >= 0
    assert d.workspace_bytes(4, 7, 100) % 256 == 0


# fake, aligned, never dereferenced device addresses: validation fails first
P = C.c_void_p(0x10000)
P2 = C.c_void_p(0x20000)
ODD = C.c_void_p(0x10001)
S0 = C.c_void_p(0)


def topk(L, logits=P, dtype=1, rows=7, V=151936, stride=151936, invT=1.0, idx=P, prob=P,
         logp=P, logz=P, ws=P2, wsb=1 << 30):
    return L.dflash2_topk_softmax(logits, dtype, rows, V, stride, invT, idx, prob, logp, logz, ws,
                                  wsb, S0)


def test_topk_validation(L):
    assert topk(L, dtype=5) == EDTYPE
    assert topk(L, V=15) == ESHAPE
    assert topk(L, stride=100) == ESHAPE
    assert topk(L, rows=-1) == ESHAPE
    assert topk(L, invT=0.0) == EINVAL
    assert topk(L, invT=float("inf")) == EINVAL
    assert topk(L, invT=float("nan")) == EINVAL
    assert topk(L, rows=0) == OK          # nothing to do, nothing launched
    assert topk(L, logits=None) == EINVAL
    assert topk(L, logz=None) == EINVAL
    assert topk(L, logits=ODD) == EALIGN
    assert topk(L, ws=None) == EWORKSPACE
    assert topk(L, ws=C.c_void_p(0x20010)) == EWORKSPACE   # not 256-aligned
    assert topk(L, wsb=1000) == EWORKSPACE


def test_select_validation(L):
    def sel(idx=P, logp=P, anchor=None, emb=P, edt=1, V=151936, d=128, W=P, B=2, G=7, tok=P,
            rank=P, score=P, ws=P2, wsb=1 << 30):
        return L.dflash2_pair_select(idx, logp, anchor, emb, edt, V, d, W, B, G, tok, rank, score,
                                     ws, wsb, S0)
    assert sel(edt=3) == EDTYPE
    assert sel(d=96) == ESHAPE
    assert sel(G=0) == ESHAPE
    assert sel(G=32) == ESHAPE
    assert sel(B=-2) == ESHAPE
    assert sel(B=0) == OK
    assert sel(W=None) == EINVAL
    assert sel(idx=ODD) == EALIGN
    assert sel(wsb=16) == EWORKSPACE


def test_verify_validation(L):
    def greedy(t=P, dt=1, B=2, G=7, V=151936, d=P, n=P, o=P, ws=P2, wsb=1 << 30):
        return L.dflash2_verify_greedy(t, dt, B, G, V, d, n, o, ws, wsb, S0)
    assert greedy(dt=2) == EDTYPE
    assert greedy(G=0) == ESHAPE
    assert greedy(G=32) == ESHAPE
    assert greedy(V=0) == ESHAPE
    assert greedy(B=0) == OK
    assert greedy(n=None) == EINVAL
    assert greedy(o=ODD) == EALIGN
    assert greedy(ws=None) == EWORKSPACE

    def sample(t=P, q=P, dt=1, B=2, G=7, V=151936, d=P, invT=1.0, qm=0, n=P, o=P, ws=P2,
               wsb=1 << 30):
        return L.dflash2_verify_sample(t, q, dt, B, G, V, d, invT, 0, 0, None, qm, n, o, None,
                                       None, ws, wsb, S0)
    assert sample(dt=9) == EDTYPE
    assert sample(G=40) == ESHAPE
    assert sample(invT=-1.0) == EINVAL
    assert sample(qm=2) == EINVAL
    assert sample(q=None) == EINVAL            # softmax mode needs the draft logits
    assert sample(B=0) == OK
    assert sample(t=ODD) == EALIGN
    assert sample(wsb=0) == EWORKSPACE

    def sample_ex(qmax=P, qlse=P, qm=0, B=2, ws=P2, wsb=1 << 30):
        return L.dflash2_verify_sample_ex(P, P, 1, B, 7, 151936, P, qmax, qlse, 1.0, 0, 0, None,
                                          qm, P, P, None, None, ws, wsb, S0)
    assert sample_ex(qlse=None) == EINVAL      # normalisers: both or neither
    assert sample_ex(qmax=None) == EINVAL
    assert sample_ex(qmax=ODD) == EALIGN
    assert sample_ex(wsb=0) == EWORKSPACE
    assert sample_ex(B=0) == OK


def test_topk_ex_validation(L):
    def topk_ex(rmax=P, rlse=P, V=151936):
        return L.dflash2_topk_softmax_ex(P, 1, 4, V, V, 1.0, P, P, P, P, rmax, rlse, P2, 1 << 30,
                                         S0)
    assert topk_ex(V=15) == ESHAPE
    assert topk_ex(rmax=ODD) == EALIGN
    assert topk_ex(rlse=ODD) == EALIGN


def test_dynconv_validation(L):
    def conv(x=P, xp=P, w=P, dt=1, B=2, T=8, H=5120, out=P2, ws=P2, wsb=1 << 30):
        return L.dflash2_dynconv2(x, xp, w, dt, B, T, H, out, ws, wsb, S0)
    assert conv(dt=4) == EDTYPE
    assert conv(H=100) == ESHAPE
    assert conv(H=0) == ESHAPE
    assert conv(B=-1) == ESHAPE
    assert conv(T=0) == OK
    assert conv(w=None) == EINVAL
    assert conv(x=C.c_void_p(0x10008)) == EALIGN
    assert conv(ws=None) == EWORKSPACE
    assert conv(ws=C.c_void_p(0x20010)) == EWORKSPACE   # not 256-aligned
    assert conv(wsb=1000) == EWORKSPACE
    # fp32 runs without a workspace
    assert L.dflash2_dynconv2_workspace_bytes(0, 2, 8, 5120) == 0
    need = L.dflash2_dynconv2_workspace_bytes(1, 32, 8, 5120)
    assert need > 0 and need == L.dflash2_dynconv2_workspace_bytes(1, 8, 32, 5120)
    assert L.dflash2_dynconv2_workspace_bytes(1, 2, 8, 100) == 0


def test_greedy_early_exit_validation(L):
    def ee(t=P, dt=1, B=2, G=7, V=151936, d=P, n=P, o=P, ws=P2, wsb=1 << 30):
        return L.dflash2_verify_greedy_early_exit(t, dt, B, G, V, d, n, o, ws, wsb, S0)
    assert ee(dt=2) == EDTYPE
    assert ee(G=0) == ESHAPE
    assert ee(G=32) == ESHAPE
    assert ee(B=0) == OK
    assert ee(n=None) == EINVAL
    assert ee(o=ODD) == EALIGN
    assert ee(ws=None) == EWORKSPACE
    assert ee(wsb=64) == EWORKSPACE


def test_select_ex_validation(L):
    def sel(edt=1, impl=0, wsb=1 << 30, B=2):
        return L.dflash2_pair_select_ex(P, P, None, P, edt, 151936, 128, P, B, 7, P, P, P, impl,
                                        P2, wsb, S0)
    assert sel(impl=3) == EINVAL
    assert sel(impl=-1) == EINVAL
    assert sel(edt=0, impl=2) == EDTYPE     # the tensor path takes bf16 tables only
    assert sel(B=0) == OK
    assert sel(wsb=16) == EWORKSPACE


def test_verify_trunc_validation(L):
    def trunc(t=P, q=P, dt=1, B=2, G=7, V=151936, d=P, invT=1.0, k=20, p=0.95, qm=0, n=P, o=P,
              ws=P2, wsb=1 << 30):
        return L.dflash2_verify_sample_trunc(t, q, dt, B, G, V, d, invT, k, p, 0, 0, None, qm, n,
                                             o, None, None, ws, wsb, S0)
    assert trunc(dt=3) == EDTYPE
    assert trunc(G=0) == ESHAPE
    assert trunc(k=0) == ESHAPE
    assert trunc(k=33) == ESHAPE               # the kernel keeps 32 keys per row
    assert trunc(p=0.0) == EINVAL
    assert trunc(p=1.5) == EINVAL
    assert trunc(p=float("nan")) == EINVAL
    assert trunc(invT=0.0) == EINVAL
    assert trunc(qm=3) == EINVAL
    assert trunc(q=None) == EINVAL             # softmax q needs the draft logits
    assert trunc(q=None, qm=1, B=0) == OK
    assert trunc(B=0) == OK
    assert trunc(o=ODD) == EALIGN
    assert trunc(wsb=0) == EWORKSPACE
    assert trunc(k=32, p=1.0, V=8, wsb=1 << 30) != ESHAPE   # top_k > V keeps V


def test_dynconv_packed_validation(L):
    assert L.dflash2_dynconv2_packed_bytes(1, 5120) == 4 * 5120 * 5120
    assert L.dflash2_dynconv2_packed_bytes(0, 5120) == 0     # fp32 has no packed form
    assert L.dflash2_dynconv2_packed_bytes(1, 100) == 0
    assert L.dflash2_dynconv2_pack(P, 0, 128, P2, S0) == EDTYPE
    assert L.dflash2_dynconv2_pack(P, 1, 100, P2, S0) == ESHAPE
    assert L.dflash2_dynconv2_pack(None, 1, 128, P2, S0) == EINVAL
    assert L.dflash2_dynconv2_pack(P, 1, 128, C.c_void_p(0x20010), S0) == EALIGN

    def packed(x=P, xp=P, w=P2, dt=1, B=2, T=8, H=5120, out=P2, ws=P2, wsb=1 << 30):
        return L.dflash2_dynconv2_packed(x, xp, w, dt, B, T, H, out, ws, wsb, S0)
    assert packed(dt=0) == EDTYPE
    assert packed(H=100) == ESHAPE
    assert packed(T=0) == OK
    assert packed(w=None) == EINVAL
    assert packed(w=C.c_void_p(0x20010)) == EALIGN
    assert packed(ws=None) == EWORKSPACE
    assert packed(wsb=1000) == EWORKSPACE
