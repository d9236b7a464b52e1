"""The benchmark's work count, pinned to PSA's Table 2 (PSA: Parameterized
Stripe Attention, section 4.2): the work of one attention call is 4 N^2 d H
FLOP when dense and (1 - sparsity) x dense for a sparse mask, and MFU is that
work over the time over the peak. `bench._alg_flops` counts the work from a
plan (4 d sum over query groups of rows x kept key rows); here it is fed
synthetic plans on the CPU whose dense or 25 %-kept structure reproduces the
table's rows, and `bench._rate` reproduces the table's MFU example. Every
TFLOPS and roofline number of the benchmark goes through these two functions.
"""
import json
import os

import numpy as np
import pytest
import torch

import bench

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = json.load(open(os.path.join(HERE, "golden", "psa_table2_flops.json")))


class _FakePlan:
    """Just the plan arrays _alg_flops reads, as CPU tensors."""

    def __init__(self, q_sizes, k_sizes, kept):
        BH, Gq = q_sizes.shape
        Gk = k_sizes.shape[1]
        W = (Gk + 63) // 64
        km = np.zeros((BH, Gq, W), dtype=np.uint64)
        for b in range(Gk):
            km[:, :, b // 64] |= kept[:, :, b].astype(np.uint64) << np.uint64(b % 64)
        off = lambda s: np.concatenate([np.zeros((BH, 1), np.int64), np.cumsum(s, 1)], 1).astype(np.int32)
        self._v = dict(q_off=torch.from_numpy(off(q_sizes)), k_off=torch.from_numpy(off(k_sizes)),
                       kmask=torch.from_numpy(km.view(np.int64)))

    def views(self):
        return self._v


def _split(N, G, rng):
    """G group sizes summing to N (some of them empty)."""
    cuts = np.sort(rng.integers(0, N + 1, size=G - 1))
    return np.diff(np.concatenate([[0], cuts, [N]])).astype(np.int64)


def _plan(case, rng):
    N, H, keep = case["N"], case["H"], case["keep"]
    Gq, Gk = 256, 256   # more than 64 key groups: the mask spans several words
    q_sizes = np.stack([_split(N, Gq, rng) for _ in range(H)])
    if keep == 1.0:
        k_sizes = np.stack([_split(N, Gk, rng) for _ in range(H)])
        kept = np.ones((H, Gq, Gk), dtype=bool)
    else:
        # four key groups of N/4 rows at scattered ids, the others empty; every
        # query group keeps one of the four (and some empty groups, which add
        # no work): each query row attends exactly N/4 keys
        assert keep == 0.25 and N % 4 == 0
        k_sizes = np.zeros((H, Gk), np.int64)
        big = np.array([3, 70, 131, 250])
        k_sizes[:, big] = N // 4
        kept = rng.random((H, Gq, Gk)) < 0.2
        kept[:, :, big] = False
        kept[np.arange(H)[:, None], np.arange(Gq)[None, :], big[rng.integers(0, 4, size=(H, Gq))]] = True
    return _FakePlan(q_sizes, k_sizes, kept)


@pytest.mark.parametrize("case", GOLDEN["cases"], ids=[c["name"] for c in GOLDEN["cases"]])
def test_alg_flops_reproduces_table2(case):
    rng = np.random.default_rng(7)
    flops = bench._alg_flops(_plan(case, rng), case["d"])
    assert flops == 4.0 * case["keep"] * case["N"] ** 2 * case["d"] * case["H"]
    assert round(flops / 1e12, 2) == case["tflop"], (case["name"], flops / 1e12)


def test_alg_flops_counts_only_kept_pairs():
    """One head, hand-sized groups: work = 4 d sum_a n_a sum_{b kept} m_b."""
    q = np.array([[5, 0, 7]])
    k = np.array([[2, 3, 11]])
    kept = np.array([[[1, 0, 1], [1, 1, 1], [0, 1, 0]]], dtype=bool)
    assert bench._alg_flops(_FakePlan(q, k, kept), 64) == 4 * 64 * (5 * 13 + 0 + 7 * 3)


def test_rate_reproduces_table2_mfu():
    m = GOLDEN["mfu_case"]
    tflops, frac = bench._rate(m["tflop"] * 1e12, m["ms"], m["peak_tflops"])
    assert abs(tflops - m["tflop"] / (m["ms"] * 1e-3)) < 1e-9
    assert round(100 * frac, 2) == m["mfu_percent"]
