"""CPU oracle for the DFlash 2 draft -> select -> verify step (fp64, plain C++).

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the benchmark's CPU-baseline leg may import this package.  It shares no
code with the CUDA library; the two meet only through the seeded input
generators in ``synth``.

Every wrapper takes numpy arrays in their storage type: fp32 arrays as
``float32``, bf16 arrays as ``uint16`` bit patterns (dtype flag 1).  Floating
outputs come back as float64, unrounded.
"""
import ctypes as C

import numpy as np

from . import build as _build

F32, BF16 = 0, 1
Q_SOFTMAX, Q_ONEHOT = 0, 1
K = 16

_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(_build.build())
        _sig()
    return _lib


def _p(a):
    return None if a is None else C.c_void_p(a.ctypes.data)


def _sig():
    L = _lib
    vp, i32, i64, u32, u64, dbl = C.c_void_p, C.c_int, C.c_int64, C.c_uint32, C.c_uint64, C.c_double
    L.orc_philox4x32_10.argtypes = [vp, vp, vp]
    L.orc_philox4x32_10.restype = None
    L.orc_uniform.argtypes = [u64, u32, u32, u32, u32]
    L.orc_uniform.restype = dbl
    L.orc_uniforms.argtypes = [u64, u32, vp, i64, u32, u32, vp]
    L.orc_uniforms.restype = None
    L.orc_topk_softmax.argtypes = [vp, i32, i64, i64, i64, dbl, vp, vp, vp, vp]
    L.orc_pair.argtypes = [vp, i32, i32, vp, C.c_int32, C.c_int32]
    L.orc_pair.restype = dbl
    L.orc_pair_select.argtypes = [vp, vp, vp, vp, i32, i64, i32, vp, i32, i32, vp, vp, vp]
    L.orc_path_rescore.argtypes = [vp, vp, vp, vp, i32, i64, i32, vp, i32, i32, vp, vp]
    L.orc_verify_greedy.argtypes = [vp, i32, i32, i32, i64, vp, vp, vp]
    L.orc_verify_sample_u.argtypes = [vp, vp, i32, i32, i32, i64, vp, dbl, i32, vp, vp,
                                      vp, vp, vp, vp, vp]
    L.orc_verify_sample.argtypes = [vp, vp, i32, i32, i32, i64, vp, dbl, u64, u32, vp, i32,
                                    vp, vp, vp, vp, vp, vp]
    L.orc_verify_sample_trunc_u.argtypes = [vp, vp, i32, i32, i32, i64, vp, dbl, i32, dbl, i32,
                                            vp, vp, vp, vp, vp, vp, vp, vp]
    L.orc_verify_sample_trunc.argtypes = [vp, vp, i32, i32, i32, i64, vp, dbl, i32, dbl, u64,
                                          u32, vp, i32, vp, vp, vp, vp, vp, vp, vp]
    L.orc_dynconv2.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp]


def _dtype_of(a):
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError("oracle inputs are float32 or uint16 (bf16 bits), got %s" % a.dtype)


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def _check(rc, what):
    if rc != 0:
        raise ValueError("oracle %s rejected its arguments" % what)


# ---------------------------------------------------------------- Philox
def philox4x32_10(ctr, key):
    c = _c(ctr, np.uint32)
    k = _c(key, np.uint32)
    out = np.zeros(4, np.uint32)
    lib().orc_philox4x32_10(_p(c), _p(k), _p(out))
    return out


def uniform(seed, step, seq_id, pos, purpose):
    return lib().orc_uniform(seed, step, seq_id, pos, purpose)


def uniforms(seed, step, seq_ids, pos, purpose):
    s = _c(seq_ids, np.uint32)
    out = np.zeros(s.shape, np.float64)
    lib().orc_uniforms(seed, step, _p(s), s.size, pos, purpose, _p(out))
    return out


# ---------------------------------------------------------------- softmax + top-16
def topk_softmax(logits, inv_temperature=1.0):
    """logits [rows, V] (float32 or bf16 bits) -> idx, prob, logp [rows,16], logz [rows]."""
    x = logits
    if x.ndim != 2 or x.strides[1] != x.itemsize or x.strides[0] % x.itemsize:
        x = np.ascontiguousarray(x)
    rows, V = x.shape
    stride = x.strides[0] // x.itemsize if rows > 1 else V
    idx = np.zeros((rows, K), np.int32)
    prob = np.zeros((rows, K), np.float64)
    logp = np.zeros((rows, K), np.float64)
    logz = np.zeros(rows, np.float64)
    _check(lib().orc_topk_softmax(_p(x), _dtype_of(x), rows, V, stride, float(inv_temperature),
                                  _p(idx), _p(prob), _p(logp), _p(logz)), "topk_softmax")
    return idx, prob, logp, logz


# ---------------------------------------------------------------- pair selector
def pair(emb, W, a, b):
    e = np.ascontiguousarray(emb)
    w = _c(W, np.float32)
    return lib().orc_pair(_p(e), _dtype_of(e), e.shape[1], _p(w), int(a), int(b))


def pair_select(idx, logp, anchor, emb, W):
    """idx [B,G,16] int32, logp [B,G,16] float32, anchor [B] int32 or None,
    emb [V,d], W [d,d] float32 -> path_tok [B,G], path_rank [B,G], path_score [B]."""
    i = _c(idx, np.int32)
    lp = _c(logp, np.float32)
    B, G, _ = i.shape
    e = np.ascontiguousarray(emb)
    w = _c(W, np.float32)
    a = None if anchor is None else _c(anchor, np.int32)
    tok = np.zeros((B, G), np.int32)
    rank = np.zeros((B, G), np.int32)
    score = np.zeros(B, np.float64)
    _check(lib().orc_pair_select(_p(i), _p(lp), _p(a), _p(e), _dtype_of(e), e.shape[0], e.shape[1],
                                 _p(w), B, G, _p(tok), _p(rank), _p(score)), "pair_select")
    return tok, rank, score


def path_rescore(idx, logp, anchor, emb, W, path_rank):
    i = _c(idx, np.int32)
    lp = _c(logp, np.float32)
    B, G, _ = i.shape
    e = np.ascontiguousarray(emb)
    w = _c(W, np.float32)
    a = None if anchor is None else _c(anchor, np.int32)
    r = _c(path_rank, np.int32)
    score = np.zeros(B, np.float64)
    _check(lib().orc_path_rescore(_p(i), _p(lp), _p(a), _p(e), _dtype_of(e), e.shape[0],
                                  e.shape[1], _p(w), B, G, _p(r), _p(score)), "path_rescore")
    return score


# ---------------------------------------------------------------- verify
def verify_greedy(target, draft_tok):
    """target [B, G+1, V], draft_tok [B, G] -> n_accept [B], out_tok [B, G+1]."""
    t = np.ascontiguousarray(target)
    B, G1, V = t.shape
    d = _c(draft_tok, np.int32)
    n = np.zeros(B, np.int32)
    out = np.zeros((B, G1), np.int32)
    _check(lib().orc_verify_greedy(_p(t), _dtype_of(t), B, G1 - 1, V, _p(d), _p(n), _p(out)),
           "verify_greedy")
    return n, out


def verify_sample_u(target, draft, draft_tok, u_acc, u_res, inv_temperature=1.0,
                    q_mode=Q_SOFTMAX):
    """Explicit uniforms: u_acc [B,G], u_res [B,G+1].  Returns n, out, ratio,
    margin_acc, margin_res."""
    t = np.ascontiguousarray(target)
    B, G1, V = t.shape
    G = G1 - 1
    q = None if draft is None else np.ascontiguousarray(draft)
    d = _c(draft_tok, np.int32)
    ua = _c(u_acc, np.float64)
    ur = _c(u_res, np.float64)
    n = np.zeros(B, np.int32)
    out = np.zeros((B, G1), np.int32)
    ratio = np.zeros((B, G), np.float64)
    ma = np.zeros(B, np.float64)
    mr = np.zeros(B, np.float64)
    _check(lib().orc_verify_sample_u(_p(t), _p(q), _dtype_of(t), B, G, V, _p(d),
                                     float(inv_temperature), q_mode, _p(ua), _p(ur), _p(n),
                                     _p(out), _p(ratio), _p(ma), _p(mr)), "verify_sample_u")
    return n, out, ratio, ma, mr


def verify_sample(target, draft, draft_tok, seed, step, seq_id=None, inv_temperature=1.0,
                  q_mode=Q_SOFTMAX):
    """Philox uniforms.  Returns n, out, ratio, u, margin_acc, margin_res."""
    t = np.ascontiguousarray(target)
    B, G1, V = t.shape
    G = G1 - 1
    q = None if draft is None else np.ascontiguousarray(draft)
    d = _c(draft_tok, np.int32)
    sid = None if seq_id is None else _c(seq_id, np.uint32)
    n = np.zeros(B, np.int32)
    out = np.zeros((B, G1), np.int32)
    ratio = np.zeros((B, G), np.float64)
    u = np.zeros((B, G), np.float64)
    ma = np.zeros(B, np.float64)
    mr = np.zeros(B, np.float64)
    _check(lib().orc_verify_sample(_p(t), _p(q), _dtype_of(t), B, G, V, _p(d),
                                   float(inv_temperature), int(seed), int(step), _p(sid), q_mode,
                                   _p(n), _p(out), _p(ratio), _p(u), _p(ma), _p(mr)),
           "verify_sample")
    return n, out, ratio, u, ma, mr


def verify_sample_trunc_u(target, draft, draft_tok, u_acc, u_res, inv_temperature=1.0,
                          top_k=20, top_p=0.95, q_mode=Q_SOFTMAX):
    """Verification of top-k / top-p truncated distributions with explicit
    uniforms u_acc [B,G], u_res [B,G+1].  Returns n, out, ratio, margin_acc,
    margin_res, margin_trunc."""
    t = np.ascontiguousarray(target)
    B, G1, V = t.shape
    G = G1 - 1
    q = None if draft is None else np.ascontiguousarray(draft)
    d = _c(draft_tok, np.int32)
    ua = _c(u_acc, np.float64)
    ur = _c(u_res, np.float64)
    n = np.zeros(B, np.int32)
    out = np.zeros((B, G1), np.int32)
    ratio = np.zeros((B, G), np.float64)
    ma, mr, mt = (np.zeros(B, np.float64) for _ in range(3))
    _check(lib().orc_verify_sample_trunc_u(_p(t), _p(q), _dtype_of(t), B, G, V, _p(d),
                                           float(inv_temperature), int(top_k), float(top_p),
                                           q_mode, _p(ua), _p(ur), _p(n), _p(out), _p(ratio),
                                           _p(ma), _p(mr), _p(mt)), "verify_sample_trunc_u")
    return n, out, ratio, ma, mr, mt


def verify_sample_trunc(target, draft, draft_tok, seed, step, seq_id=None, inv_temperature=1.0,
                        top_k=20, top_p=0.95, q_mode=Q_SOFTMAX):
    """Philox uniforms.  Returns n, out, ratio, u, margin_acc, margin_res,
    margin_trunc."""
    t = np.ascontiguousarray(target)
    B, G1, V = t.shape
    G = G1 - 1
    q = None if draft is None else np.ascontiguousarray(draft)
    d = _c(draft_tok, np.int32)
    sid = None if seq_id is None else _c(seq_id, np.uint32)
    n = np.zeros(B, np.int32)
    out = np.zeros((B, G1), np.int32)
    ratio = np.zeros((B, G), np.float64)
    u = np.zeros((B, G), np.float64)
    ma, mr, mt = (np.zeros(B, np.float64) for _ in range(3))
    _check(lib().orc_verify_sample_trunc(_p(t), _p(q), _dtype_of(t), B, G, V, _p(d),
                                         float(inv_temperature), int(top_k), float(top_p),
                                         int(seed), int(step), _p(sid), q_mode, _p(n), _p(out),
                                         _p(ratio), _p(u), _p(ma), _p(mr), _p(mt)),
           "verify_sample_trunc")
    return n, out, ratio, u, ma, mr, mt


# ---------------------------------------------------------------- dynconv
def dynconv2(x, x_prev, w_tap):
    """x [B,T,H], x_prev [B,H], w_tap [2H,H] (all float32 or all bf16 bits) -> out [B,T,H] f64."""
    xx = np.ascontiguousarray(x)
    xp = np.ascontiguousarray(x_prev)
    w = np.ascontiguousarray(w_tap)
    dt = _dtype_of(xx)
    if _dtype_of(xp) != dt or _dtype_of(w) != dt:
        raise TypeError("dynconv2 operands must share one dtype")
    B, T, H = xx.shape
    out = np.zeros((B, T, H), np.float64)
    _check(lib().orc_dynconv2(_p(xx), _p(xp), _p(w), dt, B, T, H, _p(out)), "dynconv2")
    return out
