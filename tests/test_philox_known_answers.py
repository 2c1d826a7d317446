"""The oracle's Philox4x32-10 stream pinned against two implementations
written by third parties, called as libraries (no constants copied):

  - PyTorch's host engine (ATen/core/PhiloxRNGEngine.h, at::Philox4_32), on
    the CPU;
  - cuRAND's device API (curand_init + curand4 on a curandStatePhilox4_32_10_t,
    and curand_Philox4x32_10 on a counter directly), on the GPU.

Philox4x32-10 is defined in Salmon et al., "Parallel Random Numbers: As Easy
as 1, 2, 3" (SC'11), section 5.  Both libraries follow that definition, so
every output word of the oracle must equal theirs bit for bit: a swapped
multiplier, a hi/lo swap in one lane or a missing key bump changes almost
every word.  The counters cover random words, the verify step's own counters
(step, seq_id, position, purpose) and the extremes of each word.
"""
import ctypes as C
import os
import sys

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "philox_ref"))
import build as philox_ref_build  # noqa: E402  (tests/philox_ref/build.py)

from parity import gpu, need_cuda  # noqa: E402


def _cases(seed=20261202, n=2048, word1_max=2 ** 32):
    rng = np.random.default_rng(seed)
    ctr = rng.integers(0, 2 ** 32, size=(n, 4), dtype=np.uint64).astype(np.uint32)
    ctr[:, 1] = rng.integers(0, word1_max, size=n, dtype=np.uint64).astype(np.uint32)
    key = rng.integers(0, 2 ** 32, size=(n, 2), dtype=np.uint64).astype(np.uint32)
    # the verify step's counters: (step, seq_id, position, purpose), key = seed halves
    extra_c, extra_k = [], []
    for seed_ in (0, 1, 0xDEADBEEFCAFEF00D):
        for step in (0, 1, 12345):
            for sid in (0, 5, 31):
                for pos in (0, 3, 7, 15):
                    for purpose in (0, 1, 2):
                        extra_c.append((step, sid, pos, purpose))
                        extra_k.append((seed_ & 0xFFFFFFFF, seed_ >> 32))
    # extremes of every word
    top1 = min(word1_max - 1, 2 ** 32 - 1)
    for c in ((0, 0, 0, 0), (2 ** 32 - 1, top1, 2 ** 32 - 1, 2 ** 32 - 1), (1, 0, 0, 0),
              (0, 1, 0, 0), (0, 0, 1, 0), (0, 0, 0, 1)):
        for k in ((0, 0), (2 ** 32 - 1, 2 ** 32 - 1), (1, 0), (0, 1)):
            extra_c.append(c)
            extra_k.append(k)
    ctr = np.concatenate([ctr, np.array(extra_c, np.uint64).astype(np.uint32)])
    key = np.concatenate([key, np.array(extra_k, np.uint64).astype(np.uint32)])
    return np.ascontiguousarray(ctr), np.ascontiguousarray(key)


def _oracle_words(orc, ctr, key):
    return np.stack([orc.philox4x32_10(c, k) for c, k in zip(ctr, key)])


def _ptr(a):
    return a.ctypes.data_as(C.c_void_p)


def test_oracle_matches_pytorch_philox_engine(orc):
    lib = C.CDLL(philox_ref_build.build_torch_ref())
    lib.torch_philox_words.argtypes = [C.c_void_p, C.c_void_p, C.c_int64, C.c_void_p]
    lib.torch_philox_words.restype = None
    ctr, key = _cases()
    ref = np.zeros((len(ctr), 4), np.uint32)
    lib.torch_philox_words(_ptr(ctr), _ptr(key), len(ctr), _ptr(ref))
    got = _oracle_words(orc, ctr, key)
    bad = np.flatnonzero(np.any(got != ref, axis=1))
    assert bad.size == 0, "first mismatch: counter %s key %s oracle %s torch %s" % (
        ctr[bad[0]], key[bad[0]], got[bad[0]], ref[bad[0]])
    # and the uniforms the verify step draws are the first word's top 24 bits
    for (step, sid, pos, purpose), (k0, k1), w in list(zip(ctr, key, ref))[-500:]:
        seed = int(k0) | (int(k1) << 32)
        assert orc.uniform(seed, int(step), int(sid), int(pos), int(purpose)) == \
            (int(w[0]) >> 8) / 2.0 ** 24


@gpu
def test_oracle_matches_curand_philox4_32_10(orc):
    need_cuda()
    lib = C.CDLL(philox_ref_build.build_curand_ref())
    lib.curand_philox_words.argtypes = [C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p]
    lib.curand_philox_words.restype = C.c_int
    # curand_init's offset is 4 x (counter words 0-1), so word 1 stays below 2^30
    ctr, key = _cases(seed=7, word1_max=2 ** 30)
    via_state = np.zeros((len(ctr), 4), np.uint32)
    direct = np.zeros((len(ctr), 4), np.uint32)
    rc = lib.curand_philox_words(_ptr(ctr), _ptr(key), len(ctr), _ptr(via_state), _ptr(direct))
    assert rc == 0, "CUDA error %d" % rc
    got = _oracle_words(orc, ctr, key)
    np.testing.assert_array_equal(direct, got)
    np.testing.assert_array_equal(via_state, got)
