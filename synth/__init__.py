"""Seeded synthetic inputs for the draft -> select -> verify step.

This module draws random numbers and lays them out; it holds none of the
method's arithmetic.  It is the one module that both the CPU oracle's tests
and the CUDA library's tests and benchmark read their inputs from.

Every array is produced on the host with numpy's PCG64, one stream per
(workload, sequence) from ``SeedSequence([workload_id, sequence])``, so a
sequence's data does not depend on the batch it sits in.  Values are drawn in
fp32; bf16 arrays are rounded to nearest-even and returned as uint16 bit
patterns (numpy has no bf16 type).

Workloads (shapes and distributions of the pages' decode setting: block 8 =
7 drafted tokens + 1 bonus row, vocabulary 151,936, concurrency 1 / 8 / 32):

  tiny        B=1,  block 8,  V=4,096   fp32  target N(0,2^2), draft = target + N(0,1.5^2);
              emb 4,096x64 fp32 N(0,1/64), W 64x64 N(0,1/64); dynconv H=256, T=8 fp32
  b1          B=1,  block 8,  V=151,936 bf16  target N(0,3^2) + 12 at one seeded index per row,
              draft = target + N(0, sigma_4.8^2); emb 151,936x128 bf16 N(0,1/128),
              W 128x128 fp32 N(0,1/128); dynconv H=5,120 bf16, T=8
  b8          B=8,  b1 shapes, sampling at temperature 1.0, seq_id = b
  b32         B=32, b1 shapes, per-sequence sigma_b ~ U[sigma_5.5, sigma_3.5]; dynconv 32x8 tokens
  ctx16       B=8,  block 16, V=151,936 bf16, sigma = 0.05, spike +20 (context reproduction)

sigma_a is the draft noise at which the greedy cycle's mean acceptance length
(tokens completed per verify step) is a; the values were found on 2,000 seeded
greedy cycles of the CPU oracle (tests/golden/calibrate_sigma.py, which writes
sigma_calibration.json beside this file).
"""
from dataclasses import dataclass
from typing import Optional

import numpy as np

F32, BF16 = 0, 1



def _load_calibration():
    """Draft noise for a mean greedy acceptance length on the b1 distribution,
    as written by tests/golden/calibrate_sigma.py into sigma_calibration.json."""
    import json
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "sigma_calibration.json")
    table = {4.8: None, 3.5: None, 5.5: None}
    if os.path.exists(path):
        with open(path) as f:
            for k, v in json.load(f)["sigma_for_accept"].items():
                table[float(k)] = float(v["sigma"])
    return table


SIGMA_FOR_ACCEPT = _load_calibration()


@dataclass(frozen=True)
class Workload:
    name: str
    wid: int            # first word of every SeedSequence of this workload
    B: int
    BS: int             # block size = drafted positions + 1
    V: int
    dtype: int          # F32 or BF16 for logits, embeddings and dynconv operands
    d: int              # selector embedding width
    target_std: float
    spike: float        # added to one seeded index of every target row (0 = none)
    sigma: Optional[float] = None          # draft = target + N(0, sigma^2), fixed
    accept: Optional[float] = None         # ... or sigma = sigma_accept (calibrated)
    accept_range: Optional[tuple] = None   # ... or sigma_b ~ U[sigma(hi), sigma(lo)] per sequence
    H: int = 256        # dynconv hidden size
    T: int = 8          # dynconv tokens per sequence
    sampling: bool = False
    inv_temperature: float = 1.0
    seed: int = 0       # Philox seed of the verify step

    @property
    def G(self):
        return self.BS - 1


WORKLOADS = {
    "tiny": Workload("tiny", 1, B=1, BS=8, V=4096, dtype=F32, d=64, target_std=2.0, spike=0.0,
                     sigma=1.5, H=256, T=8),
    "b1": Workload("b1", 2, B=1, BS=8, V=151936, dtype=BF16, d=128, target_std=3.0, spike=12.0,
                   accept=4.8, H=5120, T=8),
    "b8": Workload("b8", 3, B=8, BS=8, V=151936, dtype=BF16, d=128, target_std=3.0, spike=12.0,
                   accept=4.8, H=5120, T=8, sampling=True),
    "b32": Workload("b32", 4, B=32, BS=8, V=151936, dtype=BF16, d=128, target_std=3.0, spike=12.0,
                    accept_range=(5.5, 3.5), H=5120, T=8),
    "ctx16": Workload("ctx16", 5, B=8, BS=16, V=151936, dtype=BF16, d=128, target_std=3.0,
                      spike=20.0, sigma=0.05, H=5120, T=16),
}


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even) and return the uint16 bit patterns."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(a, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _store(a: np.ndarray, dtype: int) -> np.ndarray:
    return to_bf16_bits(a) if dtype == BF16 else np.ascontiguousarray(a, dtype=np.float32)


def rng_for(wid: int, *words: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([wid, *words])))


def resolve_sigma(w: Workload, rng: np.random.Generator) -> float:
    """Draft noise for one sequence of workload w."""
    if w.sigma is not None:
        return float(w.sigma)
    if w.accept is not None:
        s = SIGMA_FOR_ACCEPT.get(w.accept)
        if s is None:
            raise RuntimeError("draft noise for acceptance %.1f is not calibrated" % w.accept)
        return float(s)
    hi, lo = w.accept_range
    s_hi, s_lo = SIGMA_FOR_ACCEPT.get(hi), SIGMA_FOR_ACCEPT.get(lo)
    if s_hi is None or s_lo is None:
        raise RuntimeError("draft noise range is not calibrated")
    return float(rng.uniform(s_hi, s_lo))


@dataclass
class Sequence:
    target: np.ndarray   # [G+1, V] storage dtype
    draft: np.ndarray    # [G, V]
    anchor: int
    sigma: float


def gen_sequence(w: Workload, b: int, sigma: Optional[float] = None, wid: Optional[int] = None,
                 V: Optional[int] = None) -> Sequence:
    """Logits of sequence b.  ``sigma`` overrides the workload's draft noise
    (used by the calibration); ``V`` overrides the vocabulary (small tests)."""
    rng = rng_for(w.wid if wid is None else wid, b)
    V = w.V if V is None else V
    G = w.G
    s = resolve_sigma(w, rng) if sigma is None else float(sigma)
    tgt = rng.standard_normal((G + 1, V), dtype=np.float32) * np.float32(w.target_std)
    if w.spike:
        spikes = rng.integers(0, V, size=G + 1)
        tgt[np.arange(G + 1), spikes] += np.float32(w.spike)
    noise = rng.standard_normal((G, V), dtype=np.float32)
    drf = tgt[:G] + np.float32(s) * noise
    anchor = int(rng.integers(0, V))
    return Sequence(_store(tgt, w.dtype), _store(drf, w.dtype), anchor, s)


@dataclass
class Batch:
    w: Workload
    target: np.ndarray   # [B, G+1, V]
    draft: np.ndarray    # [B, G, V]
    anchor: np.ndarray   # [B] int32
    sigma: np.ndarray    # [B] float64
    seq_id: np.ndarray   # [B] uint32


def gen_batch(w: Workload, B: Optional[int] = None, first: int = 0, V: Optional[int] = None) -> Batch:
    B = w.B if B is None else B
    seqs = [gen_sequence(w, first + b, V=V) for b in range(B)]
    return Batch(w,
                 np.stack([s.target for s in seqs]),
                 np.stack([s.draft for s in seqs]),
                 np.array([s.anchor for s in seqs], np.int32),
                 np.array([s.sigma for s in seqs], np.float64),
                 np.arange(first, first + B, dtype=np.uint32))


@dataclass
class Selector:
    emb: np.ndarray      # [V, d] storage dtype
    W: np.ndarray        # [d, d] float32


def gen_selector(w: Workload, V: Optional[int] = None, d: Optional[int] = None) -> Selector:
    V = w.V if V is None else V
    d = w.d if d is None else d
    rng = rng_for(w.wid, 1_000_003)
    emb = rng.standard_normal((V, d), dtype=np.float32) * np.float32(1.0 / np.sqrt(d))
    W = rng.standard_normal((d, d), dtype=np.float32) * np.float32(1.0 / np.sqrt(d))
    return Selector(_store(emb, w.dtype), W.astype(np.float32))


@dataclass
class ConvInputs:
    x: np.ndarray        # [B, T, H]
    x_prev: np.ndarray   # [B, H]
    w_tap: np.ndarray    # [2H, H]


def gen_conv_weights(w: Workload, H: Optional[int] = None) -> np.ndarray:
    H = w.H if H is None else H
    rng = rng_for(w.wid, 2_000_003)
    wt = rng.standard_normal((2 * H, H), dtype=np.float32) * np.float32(1.0 / np.sqrt(H))
    return _store(wt, w.dtype)


def gen_conv(w: Workload, B: Optional[int] = None, T: Optional[int] = None,
             H: Optional[int] = None, first: int = 0) -> ConvInputs:
    B = w.B if B is None else B
    T = w.T if T is None else T
    H = w.H if H is None else H
    xs, xp = [], []
    for b in range(first, first + B):
        rng = rng_for(w.wid, 3_000_003, b)
        xp.append(rng.standard_normal(H, dtype=np.float32))
        xs.append(rng.standard_normal((T, H), dtype=np.float32))
    x = np.stack(xs) if xs else np.zeros((0, T, H), np.float32)
    x_prev = np.stack(xp) if xp else np.zeros((0, H), np.float32)
    return ConvInputs(_store(x, w.dtype), _store(x_prev, w.dtype), gen_conv_weights(w, H))
