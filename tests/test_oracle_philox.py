"""Pins of the oracle's Philox4x32-10 stream and the uniforms drawn from it.

Philox4x32-10 is defined in Salmon et al., "Parallel Random Numbers: As Easy
as 1, 2, 3" (SC'11), section 5.  No third-party known-answer vectors are used;
the oracle is pinned by what the construction guarantees: outputs that are
uniform, independent across the counter words, a key that matters in both
halves, and full avalanche after ten rounds.  The GPU implementation is a
separate restatement checked against this one on the GPU.
"""
import numpy as np
import pytest
from scipy import stats


def _words(orc, ctr, key):
    return orc.philox4x32_10(np.array(ctr, np.uint32), np.array(key, np.uint32))


def test_uniform_is_24_bit_grid(orc):
    u = orc.uniforms(7, 3, np.arange(4096, dtype=np.uint32), 0, 0)
    k = u * 2.0 ** 24
    assert np.all(k == np.floor(k))
    assert np.all((u >= 0.0) & (u < 1.0))
    # u is word0 >> 8 scaled: recompute from the raw words
    w = _words(orc, [3, 5, 0, 0], [7, 0])
    assert orc.uniform(7, 3, 5, 0, 0) == (int(w[0]) >> 8) / 2.0 ** 24


def test_uniformity_chi_square(orc):
    n = 1 << 20
    u = orc.uniforms(0, 0, np.arange(n, dtype=np.uint32), 0, 0)
    counts = np.bincount((u * 256).astype(np.int64), minlength=256)
    stat, p = stats.chisquare(counts)
    assert p > 1e-3, (stat, p)
    # the low-order bits the >> 8 keeps are uniform too
    low = np.bincount(((u * 2.0 ** 24).astype(np.int64) & 255), minlength=256)
    assert stats.chisquare(low)[1] > 1e-3


@pytest.mark.parametrize("other", [(1, 0), (0, 1)])
def test_independence_between_purposes_and_positions(orc, other):
    """(purpose 0, position 0) vs (purpose 1, position 0) and (purpose 0, position 1)."""
    n = 1 << 18
    sid = np.arange(n, dtype=np.uint32)
    a = orc.uniforms(11, 2, sid, 0, 0)
    pos, purpose = (0, 1) if other == (1, 0) else (1, 0)
    b = orc.uniforms(11, 2, sid, pos, purpose)
    table = np.zeros((16, 16), np.int64)
    np.add.at(table, ((a * 16).astype(int), (b * 16).astype(int)), 1)
    stat, p = stats.chisquare(table.ravel())
    assert p > 1e-3, (stat, p)
    assert abs(np.corrcoef(a, b)[0, 1]) < 5.0 / np.sqrt(n)


def test_every_counter_word_and_key_half_matters(orc):
    base = orc.uniform(0x0000000100000002, 10, 20, 3, 0)
    assert orc.uniform(0x0000000100000002, 11, 20, 3, 0) != base        # step
    assert orc.uniform(0x0000000100000002, 10, 21, 3, 0) != base        # seq_id
    assert orc.uniform(0x0000000100000002, 10, 20, 4, 0) != base        # position
    assert orc.uniform(0x0000000100000002, 10, 20, 3, 1) != base        # purpose
    assert orc.uniform(0x0000000200000002, 10, 20, 3, 0) != base        # key high half
    assert orc.uniform(0x0000000100000003, 10, 20, 3, 0) != base        # key low half


def test_avalanche(orc):
    """Ten rounds diffuse every input bit: flipping any one counter or key bit
    flips each output bit with probability 1/2.  A dropped round, a swapped
    hi/lo or a missing key bump shows up as a biased flip count."""
    rng = np.random.default_rng(5)
    trials = 96
    flips = np.zeros(192, np.float64)
    for _ in range(trials):
        ctr = rng.integers(0, 2 ** 32, 4, dtype=np.uint64).astype(np.uint32)
        key = rng.integers(0, 2 ** 32, 2, dtype=np.uint64).astype(np.uint32)
        ref = _words(orc, ctr, key)
        for bit in range(192):
            c, k = ctr.copy(), key.copy()
            if bit < 128:
                c[bit // 32] ^= np.uint32(1 << (bit % 32))
            else:
                k[(bit - 128) // 32] ^= np.uint32(1 << (bit % 32))
            out = _words(orc, c, k)
            flips[bit] += sum(bin(int(x) ^ int(y)).count("1") for x, y in zip(out, ref))
    mean = flips / trials
    # each mean is over 96 * 128 fair coin flips: sd of the mean = sqrt(32/96) = 0.58
    assert np.all(np.abs(mean - 64.0) < 4.0), mean.min()
    assert abs(mean.mean() - 64.0) < 0.3
