"""The arithmetic the centroid update rests on (CPU only, no library code).

Member sums are taken in fp64 over bf16 components, with |x| < 2^-24 counted as
zero. Every remaining component is a multiple of 2^-31, so while N max|x| < 2^22
every partial sum is an exact multiple of 2^-31 below 2^53 units: fp64 adds
without rounding. Two consequences the kernels rely on are checked here on
seeded data of the workloads' kind:

* the sum does not depend on the order of the additions (the GPU adds
  per-warp partial sums with atomics in no fixed order);
* keeping a cluster's sum across k-means rounds and moving only the tokens
  whose label changed (+x to the new cluster, -x from the old one, in any
  order) gives the same bits as summing the new members again.
"""
import numpy as np

import workload
from workload import bf16_bits_to_f32

FLUSH = 2.0 ** -24


def _flushed(x_bits):
    x = bf16_bits_to_f32(x_bits).astype(np.float64)
    x[np.abs(x) < FLUSH] = 0.0
    return x


def _sums_in_order(x, labels, C, order):
    s = np.zeros((C, x.shape[1]), dtype=np.float64)
    for t in order:  # one addition at a time, in the given order
        s[labels[t]] += x[t]
    return s


def _data(seed=3, n=3000, d=16, C=24):
    rng = np.random.default_rng(seed)
    x = rng.normal(0.0, 2.0, size=(n, d)).astype(np.float32)
    x[rng.random((n, d)) < 0.05] *= 1e-8   # some components below the flush threshold
    bits = workload.f32_to_bf16_bits(x)
    labels = rng.integers(0, C, size=n)
    return _flushed(bits), labels, C, rng


def test_member_sums_do_not_depend_on_order():
    x, labels, C, rng = _data()
    ref = _sums_in_order(x, labels, C, range(len(x)))
    for _ in range(3):
        got = _sums_in_order(x, labels, C, rng.permutation(len(x)))
        assert np.array_equal(got.view(np.uint64), ref.view(np.uint64))


def test_incremental_moves_equal_a_fresh_sum():
    x, labels, C, rng = _data(seed=5)
    sums = _sums_in_order(x, labels, C, range(len(x)))
    cur = labels.copy()
    for frac in (0.35, 0.08, 0.01):  # the share of moved tokens falls over the rounds
        new = cur.copy()
        moved = rng.random(len(x)) < frac
        new[moved] = rng.integers(0, C, size=int(moved.sum()))
        entries = [(t, +1, new[t]) for t in np.nonzero(new != cur)[0]]
        entries += [(t, -1, cur[t]) for t in np.nonzero(new != cur)[0]]
        for i in rng.permutation(len(entries)):
            t, sign, j = entries[i]
            sums[j] += sign * x[t]
        cur = new
        fresh = _sums_in_order(x, cur, C, range(len(x)))
        assert np.array_equal(sums.view(np.uint64), fresh.view(np.uint64))
        # and the centroid, the exact mean rounded once to fp32, follows
        n = np.bincount(cur, minlength=C)
        keep = n > 0
        assert np.array_equal((sums[keep] / n[keep, None]).astype(np.float32),
                              (fresh[keep] / n[keep, None]).astype(np.float32))


def test_without_the_flush_the_order_would_matter():
    """The flush is what makes the sums exact: with a component far below
    2^-24 kept, the order of the additions changes the bits ((1 + e) - 1 loses
    e, (1 - 1) + e keeps it); with it flushed to zero, both orders agree."""
    e = 2.0 ** -60  # below the fp64 ulp of 1 (2^-52), and below 2^-24: flushed
    assert (1.0 + e) - 1.0 != (1.0 - 1.0) + e
    f = 0.0 if abs(e) < FLUSH else e
    assert (1.0 + f) - 1.0 == (1.0 - 1.0) + f
