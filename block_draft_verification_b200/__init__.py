"""Python binding of libdflash2.so, the C ABI of the DFlash 2 draft -> select
-> verify step on B200 (declared in include/dflash2.h).

Argument marshalling only: every function takes CUDA torch tensors, allocates
the outputs with torch, and passes raw device pointers and the current CUDA
stream to the library, where all of the work runs.  There is no other code
path: if the library is not built, or a call fails, an exception is raised.
"""
import ctypes as C
import os

import torch

__all__ = ["F32", "BF16", "Q_SOFTMAX", "Q_ONEHOT", "K", "DFlash2Error", "lib", "workspace_bytes",
           "Workspace", "topk_softmax", "pair_select", "verify_greedy", "verify_sample",
           "verify_sample_trunc", "dynconv2", "PackedTap", "status_string", "version",
           "device_errors"]

F32, BF16 = 0, 1
Q_SOFTMAX, Q_ONEHOT = 0, 1
K = 16
MAX_BLOCK = 32

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdflash2.so")
_lib = None


class DFlash2Error(RuntimeError):
    def __init__(self, where, status):
        super().__init__("%s: %s" % (where, status_string(status) if _lib else status))
        self.status = status


def lib():
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libdflash2.so is not built (python -m block_draft_verification_b200.build)")
        L = C.CDLL(LIB_PATH)
        vp, i32, i64, u32, u64, f32, sz = (C.c_void_p, C.c_int, C.c_int64, C.c_uint32, C.c_uint64,
                                           C.c_float, C.c_size_t)
        L.dflash2_status_string.argtypes = [i32]
        L.dflash2_status_string.restype = C.c_char_p
        L.dflash2_version.restype = i32
        L.dflash2_workspace_bytes.argtypes = [i32, i32, i64]
        L.dflash2_workspace_bytes.restype = sz
        L.dflash2_topk_softmax.argtypes = [vp, i32, i64, i64, i64, f32, vp, vp, vp, vp, vp, sz, vp]
        L.dflash2_topk_softmax_ex.argtypes = [vp, i32, i64, i64, i64, f32, vp, vp, vp, vp, vp, vp,
                                              vp, sz, vp]
        L.dflash2_pair_select.argtypes = [vp, vp, vp, vp, i32, i64, i32, vp, i32, i32, vp, vp, vp,
                                          vp, sz, vp]
        L.dflash2_pair_select_ex.argtypes = [vp, vp, vp, vp, i32, i64, i32, vp, i32, i32, vp, vp,
                                             vp, i32, vp, sz, vp]
        L.dflash2_verify_greedy.argtypes = [vp, i32, i32, i32, i64, vp, vp, vp, vp, sz, vp]
        L.dflash2_verify_greedy_early_exit.argtypes = [vp, i32, i32, i32, i64, vp, vp, vp, vp, sz,
                                                       vp]
        L.dflash2_verify_sample.argtypes = [vp, vp, i32, i32, i32, i64, vp, f32, u64, u32, vp, i32,
                                            vp, vp, vp, vp, vp, sz, vp]
        L.dflash2_verify_sample_ex.argtypes = [vp, vp, i32, i32, i32, i64, vp, vp, vp, f32, u64,
                                               u32, vp, i32, vp, vp, vp, vp, vp, sz, vp]
        L.dflash2_verify_sample_trunc.argtypes = [vp, vp, i32, i32, i32, i64, vp, f32, i32, f32,
                                                  u64, u32, vp, i32, vp, vp, vp, vp, vp, sz, vp]
        L.dflash2_dynconv2.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp, sz, vp]
        L.dflash2_dynconv2_packed.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp, sz, vp]
        L.dflash2_dynconv2_pack.argtypes = [vp, i32, i32, vp, vp]
        L.dflash2_dynconv2_packed_bytes.argtypes = [i32, i32]
        L.dflash2_dynconv2_packed_bytes.restype = sz
        L.dflash2_dynconv2_workspace_bytes.argtypes = [i32, i32, i32, i32]
        L.dflash2_dynconv2_workspace_bytes.restype = sz
        L.dflash2_device_errors.argtypes = [i32]
        L.dflash2_device_errors.restype = C.c_uint32
        for f in ("dflash2_topk_softmax", "dflash2_topk_softmax_ex", "dflash2_pair_select",
                  "dflash2_pair_select_ex", "dflash2_verify_greedy_early_exit",
                  "dflash2_verify_greedy", "dflash2_verify_sample", "dflash2_verify_sample_ex",
                  "dflash2_verify_sample_trunc", "dflash2_dynconv2", "dflash2_dynconv2_pack",
                  "dflash2_dynconv2_packed"):
            getattr(L, f).restype = i32
        _lib = L
    return _lib


def status_string(status):
    return lib().dflash2_status_string(int(status)).decode()


def version():
    v = lib().dflash2_version()
    return (v >> 16, v & 0xFFFF)


def device_errors(clear=True):
    """Flags set by a tensor-core kernel whose bounded wait ran out (0 = none)."""
    return int(lib().dflash2_device_errors(1 if clear else 0))


def workspace_bytes(B, G, V):
    return int(lib().dflash2_workspace_bytes(int(B), int(G), int(V)))


def _check(where, rc):
    if rc != 0:
        raise DFlash2Error(where, rc)


def _dtype(t):
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError("expected float32 or bfloat16, got %s" % t.dtype)


def _p(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(dev):
    return C.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("dflash2 calls take CUDA tensors")


class Workspace:
    """A device scratch buffer for the calls that take one.  Calls on one
    stream run in order, so one Workspace serves every call on that stream.
    It is zero-filled when (re)allocated: the calls expect their counters
    (the first 64 KB) zero and leave them zero when they complete."""

    def __init__(self, device=None, nbytes=0):
        self.device = torch.device(device if device is not None else "cuda")
        self.buf = torch.empty(0, dtype=torch.uint8, device=self.device)
        self.reserve(nbytes)

    def reserve(self, nbytes):
        if nbytes > self.buf.numel():
            self.buf = torch.zeros(int(nbytes), dtype=torch.uint8, device=self.device)
        return self

    def args(self, B, G, V):
        self.reserve(workspace_bytes(B, G, V))
        return C.c_void_p(self.buf.data_ptr()), C.c_size_t(self.buf.numel())

    def args_bytes(self, nbytes):
        self.reserve(nbytes)
        return C.c_void_p(self.buf.data_ptr()), C.c_size_t(self.buf.numel())


_ws_cache = {}


def _ws(ws, dev, B, G, V):
    if ws is None:
        ws = _ws_cache.setdefault((dev.index, torch.cuda.current_stream(dev).cuda_stream),
                                  Workspace(dev))
    return ws.args(B, G, V)


def topk_softmax(logits, inv_temperature=1.0, out=None, ws=None, stats=False):
    """logits [..., V] (rows may be strided) -> idx [..., 16] int32, prob, logp
    [..., 16] float32, logz [...] float32; with stats=True also row_max and
    row_lse [...] float32 (dflash2_topk_softmax_ex), the normalisers
    verify_sample(draft_stats=...) reuses."""
    _cuda(logits)
    V = logits.shape[-1]
    x = logits.reshape(-1, V) if logits.dim() != 2 else logits
    if x.stride(-1) != 1:
        x = x.contiguous()
    rows = x.shape[0]
    lead = logits.shape[:-1]
    dev = logits.device
    if out is None:
        out = (torch.empty(lead + (K,), dtype=torch.int32, device=dev),
               torch.empty(lead + (K,), dtype=torch.float32, device=dev),
               torch.empty(lead + (K,), dtype=torch.float32, device=dev),
               torch.empty(lead, dtype=torch.float32, device=dev))
    if stats and len(out) == 4:
        out = tuple(out) + (torch.empty(lead, dtype=torch.float32, device=dev),
                            torch.empty(lead, dtype=torch.float32, device=dev))
    idx, prob, logp, logz = out[:4]
    rmax = out[4] if len(out) > 4 else None
    rlse = out[5] if len(out) > 5 else None
    wp, wb = _ws(ws, dev, rows, 1, V)
    stride = x.stride(0) if rows > 1 else V
    if rmax is None and rlse is None:
        _check("dflash2_topk_softmax", lib().dflash2_topk_softmax(
            _p(x), _dtype(x), rows, V, stride, float(inv_temperature), _p(idx), _p(prob),
            _p(logp), _p(logz), wp, wb, _stream(dev)))
    else:
        _check("dflash2_topk_softmax_ex", lib().dflash2_topk_softmax_ex(
            _p(x), _dtype(x), rows, V, stride, float(inv_temperature), _p(idx), _p(prob),
            _p(logp), _p(logz), _p(rmax), _p(rlse), wp, wb, _stream(dev)))
    return tuple(out)


SELECT_AUTO, SELECT_SIMT, SELECT_TENSOR = 0, 1, 2


def pair_select(idx, logp, anchor, emb, W, out=None, ws=None, impl=SELECT_AUTO):
    """idx, logp [B, G, 16], anchor [B] int32 or None, emb [V, d], W [d, d] float32
    -> path_tok [B, G] int32, path_rank [B, G] int32, path_score [B] float32.
    impl: SELECT_AUTO (tensor cores for bf16 tables, dflash2_pair_select),
    SELECT_SIMT or SELECT_TENSOR (dflash2_pair_select_ex)."""
    _cuda(idx, logp, anchor, emb, W)
    B, G, _ = idx.shape
    V, d = emb.shape
    dev = idx.device
    if out is None:
        out = (torch.empty((B, G), dtype=torch.int32, device=dev),
               torch.empty((B, G), dtype=torch.int32, device=dev),
               torch.empty((B,), dtype=torch.float32, device=dev))
    tok, rank, score = out
    wp, wb = _ws(ws, dev, B, G, V)
    if impl == SELECT_AUTO:
        _check("dflash2_pair_select", lib().dflash2_pair_select(
            _p(idx.contiguous()), _p(logp.contiguous()), _p(anchor), _p(emb.contiguous()),
            _dtype(emb), V, d, _p(W.contiguous()), B, G, _p(tok), _p(rank), _p(score), wp, wb,
            _stream(dev)))
    else:
        _check("dflash2_pair_select_ex", lib().dflash2_pair_select_ex(
            _p(idx.contiguous()), _p(logp.contiguous()), _p(anchor), _p(emb.contiguous()),
            _dtype(emb), V, d, _p(W.contiguous()), B, G, _p(tok), _p(rank), _p(score), int(impl),
            wp, wb, _stream(dev)))
    return tok, rank, score


def verify_greedy(target, draft_tok, out=None, ws=None, early_exit=False):
    """target [B, G+1, V], draft_tok [B, G] int32 -> n_accept [B], out_tok [B, G+1] int32.
    early_exit: dflash2_verify_greedy_early_exit (the same results; rows after
    a sequence's first mismatch are not read)."""
    _cuda(target, draft_tok)
    B, G1, V = target.shape
    dev = target.device
    if out is None:
        out = (torch.empty((B,), dtype=torch.int32, device=dev),
               torch.empty((B, G1), dtype=torch.int32, device=dev))
    n, toks = out
    wp, wb = _ws(ws, dev, B, G1 - 1, V)
    name = "dflash2_verify_greedy_early_exit" if early_exit else "dflash2_verify_greedy"
    _check(name, getattr(lib(), name)(
        _p(target.contiguous()), _dtype(target), B, G1 - 1, V, _p(draft_tok.contiguous()), _p(n),
        _p(toks), wp, wb, _stream(dev)))
    return n, toks


def verify_sample(target, draft, draft_tok, seed, step, seq_id=None, inv_temperature=1.0,
                  q_mode=Q_SOFTMAX, debug=False, out=None, ws=None, draft_stats=None):
    """target [B, G+1, V], draft [B, G, V] (None in one-hot mode), draft_tok [B, G]
    -> n_accept [B], out_tok [B, G+1] (+ ratio [B, G], u [B, G] if debug).
    draft_stats = (row_max, row_lse) [B, G] from topk_softmax(stats=True) on the
    draft rows: the fused cycle (dflash2_verify_sample_ex), no second pass over
    the draft rows."""
    _cuda(target, draft, draft_tok, seq_id)
    B, G1, V = target.shape
    G = G1 - 1
    dev = target.device
    if out is None:
        out = (torch.empty((B,), dtype=torch.int32, device=dev),
               torch.empty((B, G1), dtype=torch.int32, device=dev))
        if debug:
            out = out + (torch.empty((B, G), dtype=torch.float32, device=dev),
                         torch.empty((B, G), dtype=torch.float32, device=dev))
    n, toks = out[0], out[1]
    ratio = out[2] if len(out) > 2 else None
    u = out[3] if len(out) > 3 else None
    wp, wb = _ws(ws, dev, B, G, V)
    q = None if draft is None else draft.contiguous()
    sid = None if seq_id is None else seq_id.to(torch.int32).contiguous()
    qmax = qlse = None
    if draft_stats is not None:
        qmax, qlse = (t.contiguous() for t in draft_stats)
        _cuda(qmax, qlse)
    seed, step = int(seed) & (2 ** 64 - 1), int(step) & 0xFFFFFFFF
    if qmax is None:
        _check("dflash2_verify_sample", lib().dflash2_verify_sample(
            _p(target.contiguous()), _p(q), _dtype(target), B, G, V, _p(draft_tok.contiguous()),
            float(inv_temperature), seed, step, _p(sid), int(q_mode), _p(n), _p(toks), _p(ratio),
            _p(u), wp, wb, _stream(dev)))
    else:
        _check("dflash2_verify_sample_ex", lib().dflash2_verify_sample_ex(
            _p(target.contiguous()), _p(q), _dtype(target), B, G, V, _p(draft_tok.contiguous()),
            _p(qmax), _p(qlse), float(inv_temperature), seed, step, _p(sid), int(q_mode), _p(n),
            _p(toks), _p(ratio), _p(u), wp, wb, _stream(dev)))
    return out


def verify_sample_trunc(target, draft, draft_tok, seed, step, seq_id=None, inv_temperature=1.0,
                        top_k=20, top_p=0.95, q_mode=Q_SOFTMAX, debug=False, out=None, ws=None):
    """The sampling verify on top-k / top-p truncated distributions
    (dflash2_verify_sample_trunc): target [B, G+1, V], draft [B, G, V] (None in
    one-hot mode), draft_tok [B, G] -> n_accept [B], out_tok [B, G+1]
    (+ ratio [B, G], u [B, G] if debug)."""
    _cuda(target, draft, draft_tok, seq_id)
    B, G1, V = target.shape
    G = G1 - 1
    dev = target.device
    if out is None:
        out = (torch.empty((B,), dtype=torch.int32, device=dev),
               torch.empty((B, G1), dtype=torch.int32, device=dev))
        if debug:
            out = out + (torch.empty((B, G), dtype=torch.float32, device=dev),
                         torch.empty((B, G), dtype=torch.float32, device=dev))
    n, toks = out[0], out[1]
    ratio = out[2] if len(out) > 2 else None
    u = out[3] if len(out) > 3 else None
    wp, wb = _ws(ws, dev, B, G, V)
    q = None if draft is None else draft.contiguous()
    sid = None if seq_id is None else seq_id.to(torch.int32).contiguous()
    seed, step = int(seed) & (2 ** 64 - 1), int(step) & 0xFFFFFFFF
    _check("dflash2_verify_sample_trunc", lib().dflash2_verify_sample_trunc(
        _p(target.contiguous()), _p(q), _dtype(target), B, G, V, _p(draft_tok.contiguous()),
        float(inv_temperature), int(top_k), float(top_p), seed, step, _p(sid), int(q_mode), _p(n),
        _p(toks), _p(ratio), _p(u), wp, wb, _stream(dev)))
    return out


class PackedTap:
    """Tap weights [2H, H] bf16 packed once for the tensor-core path
    (dflash2_dynconv2_pack); pass it to dynconv2 in place of w_tap."""

    def __init__(self, w_tap):
        _cuda(w_tap)
        if w_tap.dtype != torch.bfloat16:
            raise TypeError("packed tap weights are bf16")
        self.H = w_tap.shape[1]
        n = int(lib().dflash2_dynconv2_packed_bytes(BF16, self.H))
        self.buf = torch.empty(n, dtype=torch.uint8, device=w_tap.device)
        _check("dflash2_dynconv2_pack", lib().dflash2_dynconv2_pack(
            _p(w_tap.contiguous()), BF16, self.H, _p(self.buf), _stream(w_tap.device)))


def dynconv2(x, x_prev, w_tap, out=None, ws=None):
    """x [B, T, H], x_prev [B, H], w_tap [2H, H] (one dtype) or a PackedTap ->
    out [B, T, H]."""
    if isinstance(w_tap, PackedTap):
        return _dynconv2_packed(x, x_prev, w_tap, out, ws)
    _cuda(x, x_prev, w_tap)
    B, T, H = x.shape
    if out is None:
        out = torch.empty_like(x)
    need = lib().dflash2_dynconv2_workspace_bytes(_dtype(x), B, T, H)
    if ws is None:
        ws = _ws_cache.setdefault((x.device.index, torch.cuda.current_stream(x.device).cuda_stream),
                                  Workspace(x.device))
    wp, wb = ws.args_bytes(need)
    _check("dflash2_dynconv2", lib().dflash2_dynconv2(
        _p(x.contiguous()), _p(x_prev.contiguous()), _p(w_tap.contiguous()), _dtype(x), B, T, H,
        _p(out), wp, wb, _stream(x.device)))
    return out


def _dynconv2_packed(x, x_prev, pk, out, ws):
    _cuda(x, x_prev)
    B, T, H = x.shape
    if out is None:
        out = torch.empty_like(x)
    need = lib().dflash2_dynconv2_workspace_bytes(BF16, B, T, H)
    if ws is None:
        ws = _ws_cache.setdefault((x.device.index, torch.cuda.current_stream(x.device).cuda_stream),
                                  Workspace(x.device))
    wp, wb = ws.args_bytes(need)
    _check("dflash2_dynconv2_packed", lib().dflash2_dynconv2_packed(
        _p(x.contiguous()), _p(x_prev.contiguous()), _p(pk.buf), _dtype(x), B, T, H, _p(out), wp,
        wb, _stream(x.device)))
    return out
