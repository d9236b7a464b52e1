"""The device timeout path, run on the GPU with the test-only build
libsvoo_stall.so (compiled with SVOO_TEST_STALL).

In that build each pipelined kernel (the clustering assignment kernel and the
attention kernel) makes one wait on an mbarrier that nothing completes, under
a pipeline wait budget of about 10 ms. The wait runs out; the CTA raises its
abort flag and its other roles leave their loops; the cleanup waits (on the
full budget) let the copies and MMAs already issued land; the kernel sets its
bit in the caller's error word and returns; later CTAs see the bit and skip
their work. No fault, trap or endless wait is involved.

The test checks that each call comes back, that the right bit is set, and
that once the word is cleared the normal build, in the same CUDA context,
still matches the oracle on the same inputs.
"""
import contextlib
import time

import numpy as np
import pytest
import torch

import oracle
import workload
import free_sparse_attention_head_b200 as svoo
from free_sparse_attention_head_b200 import build as svoo_build

from _parity import (check_attention, from_dev_bf16, gather_by_plan, inject_plan, oracle_plan_heads,
                     qkv_tensors, scale_of)

pytestmark = pytest.mark.gpu

TIMEOUT_ATTN = 1 << 0     # error word bit: an attention pipeline wait ran out
TIMEOUT_CLUSTER = 1 << 1  # error word bit: a clustering pipeline wait ran out


@contextlib.contextmanager
def _stall_library():
    """The binding's calls go to libsvoo_stall.so inside the block."""
    saved = svoo._lib
    svoo._lib = None
    try:
        yield svoo.load(svoo_build.STALL_LIB)
    finally:
        svoo._lib = saved


def test_timeout_path_reports_and_recovers():
    svoo_build.build()
    svoo.load()
    w = workload.get("tiny")
    q, k, v = workload.make_qkv(w)
    heads = list(range(w.B * w.H))
    BH = len(heads)
    cfg = svoo.Config(n_qc=w.n_qc, n_kc=w.n_kc, iters=w.iters, block_q=w.block_q)
    # a valid plan and gathered inputs, from the oracle
    plans = oracle_plan_heads(w, q, k, heads, w.keep_ratios())
    plan = svoo.Plan(svoo.Shape(1, BH, w.N, w.d, w.n_text), cfg, "cuda")
    inject_plan(plan, plans, heads)
    qp, kp, vp = qkv_tensors(*gather_by_plan(q, k, v, plans, heads), 1, BH)
    qd, kd, _ = qkv_tensors(q, k, v, w.B, w.H)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    with _stall_library():
        t0 = time.perf_counter()
        svoo.cluster(qd, kd, cfg, n_text=w.n_text, dev_err=err)
        torch.cuda.synchronize()
        t_cluster = time.perf_counter() - t0
        bits_cluster = int(err.item())
        err.zero_()
        t0 = time.perf_counter()
        svoo.sparse_attn(qp, kp, vp, plan, dev_err=err)
        torch.cuda.synchronize()
        t_attn = time.perf_counter() - t0
        bits_attn = int(err.item())
    print(f"stalled calls: clustering {t_cluster * 1e3:.1f} ms, error word {bits_cluster:#x}; "
          f"attention {t_attn * 1e3:.1f} ms, error word {bits_attn:#x}")
    assert bits_cluster & TIMEOUT_CLUSTER, bits_cluster
    assert bits_attn & TIMEOUT_ATTN, bits_attn
    # a stalled CTA gives up after its ~10 ms budget and the rest skip their work
    assert t_cluster < 20.0 and t_attn < 20.0

    # the same context, the normal build, the same inputs
    err.zero_()
    out = svoo.sparse_attn(qp, kp, vp, plan, dev_err=err)
    cl = svoo.cluster(qd, kd, cfg, n_text=w.n_text, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    o = from_dev_bf16(out).reshape(BH, w.N, w.d)
    rows = np.arange(w.N, dtype=np.int32)
    for h in heads:
        p = plans[h]
        ref, _, _ = oracle.attn_rows(q[h], k[h], v[h], scale_of(w.d), p["q_label"], p["k_label"], p["kmask"],
                                     rows)
        check_attention(o[h], ref, f"head {h} after the stalled calls")
        agree = float((cl["q_assign"][h].cpu().numpy() == p["cl"]["q_assign"]).mean())
        assert agree >= 0.999, f"head {h}: query assignments agree on {agree:.4f}"
