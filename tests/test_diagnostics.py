"""Attention-fidelity diagnostics (selection overlap, mass inside the kept set,
output MSE against dense attention): the metric definitions on small CPU
cases, then, on the GPU, the co-clustering against independent Euclidean
clustering on a synthetic workload (the comparison of iCATS sec. 5.2 /
App. D)."""
import types

import numpy as np
import pytest
import torch

import workload
import free_sparse_attention_head_b200 as svoo
from free_sparse_attention_head_b200 import diagnostics as diag
from _parity import qkv_tensors


def test_overlap_of_exact_top_k_is_one_and_disjoint_is_zero():
    p = torch.tensor([[0.5, 0.3, 0.15, 0.05], [0.1, 0.2, 0.3, 0.4]])
    top = torch.tensor([[True, True, False, False], [False, False, True, True]])
    ov, mass, n = diag.selection_metrics(p, top)
    assert ov.tolist() == [1.0, 1.0]
    assert np.allclose(mass.numpy(), [0.8, 0.7])
    assert n.tolist() == [2, 2]
    bottom = ~top
    ov, mass, _ = diag.selection_metrics(p, bottom)
    assert ov.tolist() == [0.0, 0.0]
    assert np.allclose(mass.numpy(), [0.2, 0.3])


def test_overlap_counts_partial_hits():
    p = torch.tensor([[0.4, 0.3, 0.2, 0.1]])
    sel = torch.tensor([[True, False, True, False]])   # top-2 is {0, 1}: one hit of two
    ov, mass, _ = diag.selection_metrics(p, sel)
    assert ov.item() == 0.5 and abs(mass.item() - 0.6) < 1e-6
    ov, _, _ = diag.selection_metrics(p, torch.ones(1, 4, dtype=torch.bool))
    assert ov.item() == 1.0


def test_key_groups_and_selected_keys_from_plan_arrays():
    # one head, N = 6: key groups {0: tokens 4, 1}, {1: token 0}, {2: tokens 2, 3, 5}
    k_perm = torch.tensor([[4, 1, 0, 2, 3, 5]], dtype=torch.int32)
    k_off = torch.tensor([[0, 2, 3, 6]], dtype=torch.int32)
    plan = types.SimpleNamespace(BH=1, shape=types.SimpleNamespace(N=6),
                                 views=lambda: dict(k_perm=k_perm, k_off=k_off))
    kg = diag.key_groups(plan)
    assert kg.tolist() == [[1, 0, 2, 2, 0, 2]]
    # query group 0 attends key groups {0, 2}; query group 1 attends {1}
    kmask = torch.tensor([[0b101], [0b010]], dtype=torch.int64)
    sel = diag.selected_keys(kmask, torch.tensor([0, 1]), kg[0])
    assert sel.tolist() == [[False, True, True, True, True, True], [True, False, False, False, False, False]]


def test_key_groups_handles_empty_groups_and_high_words():
    N = 3
    k_perm = torch.tensor([[2, 0, 1]], dtype=torch.int32)
    k_off = torch.tensor([[0] + [0] * 70 + [1, 3]], dtype=torch.int32)   # groups 0..69 empty
    plan = types.SimpleNamespace(BH=1, shape=types.SimpleNamespace(N=N),
                                 views=lambda: dict(k_perm=k_perm, k_off=k_off))
    kg = diag.key_groups(plan)
    assert kg.tolist() == [[71, 71, 70]]
    kmask = torch.zeros(1, 2, dtype=torch.int64)
    kmask[0, 1] = 1 << (71 - 64)
    sel = diag.selected_keys(kmask, torch.tensor([0]), kg[0])
    assert sel.tolist() == [[True, True, False]]


@pytest.mark.gpu
def test_fidelity_keep_one_is_dense():
    w = workload.get("tiny")
    q, k, v = qkv_tensors(*workload.make_qkv(w), w.B, w.H)
    cfg = svoo.Config(n_qc=w.n_qc, n_kc=w.n_kc, iters=w.iters, block_q=w.block_q)
    keep = torch.ones(w.B * w.H, dtype=torch.float32)
    f = diag.fidelity(q, k, v, keep, cfg, n_text=w.n_text, rows=128)
    assert f.overlap == 1.0 and abs(f.mass - 1.0) < 1e-5 and f.density == 1.0
    assert f.mse < 1e-4


@pytest.mark.gpu
def test_interaction_vs_identity_fidelity_report():
    """Both clusterings on one synthetic workload at the keep ratios the
    workload states; prints the numbers (the comparison is a measurement on
    synthetic data, so only validity is asserted)."""
    import dataclasses
    w = dataclasses.replace(workload.get("wan2.1-1.3b"), H=2)
    q, k, v = qkv_tensors(*workload.make_qkv(w), w.B, w.H)
    cfg = svoo.Config(n_qc=w.n_qc, n_kc=w.n_kc, iters=w.iters, block_q=w.block_q)
    keep = torch.from_numpy(w.keep_ratios())
    res = diag.compare_metrics(q, k, v, keep, cfg, n_text=w.n_text, rows=256)
    for name, f in res.items():
        print(f"fidelity {name}: overlap {f.overlap:.4f} mass {f.mass:.4f} mse {f.mse:.3e} "
              f"density {f.density:.4f}")
        assert 0.0 < f.overlap <= 1.0 and 0.0 < f.mass <= 1.0 + 1e-5 and f.mse >= 0.0
        assert 0.0 < f.density <= 1.0
