"""GPU parity of the static stripe-mask path (PSA sec. 3.2, Algorithm 1 at
PSABlock granularity) against the oracle: the plan that svoo_psa_mask writes
(block mask, labels, block sizes, kept-pair and tile counts) bit for bit, then
the whole path (svoo_psa_mask -> svoo_permute -> svoo_sparse_attn) on sampled
rows within the attention tolerance, from tiny grids through the ragged
text-token case and the 256-block maximum to the Wan 2.1 14B call
(40 heads, 21 x 45 x 80 tokens, PSABlock 3 x 8 x 16, Table 7's mix)."""
import dataclasses
import math

import numpy as np
import pytest
import torch

import oracle
import workload
import free_sparse_attention_head_b200 as svoo
from free_sparse_attention_head_b200 import build as svoo_build

from _parity import check_attention, from_dev_bf16, qkv_tensors, ragged_workload, sample_rows, scale_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    svoo_build.build()
    svoo.load()


def _cases():
    tiny = workload.get("tiny")
    rag = ragged_workload()
    w13 = dataclasses.replace(workload.get("wan2.1-1.3b"), H=3)
    # 256 blocks of one token each, plus a text group: 257 groups, 5 mask words
    maxb = dataclasses.replace(tiny, name="max-blocks", grid=(4, 8, 8), n_text=5, H=2)
    one = dataclasses.replace(tiny, name="one-block", H=2)
    return {
        "tiny": (tiny, (2, 4, 4)),
        "ragged-text": (rag, (1, 4, 8)),
        "wan1.3b-3heads": (w13, (3, 8, 16)),
        "max-blocks": (maxb, (1, 1, 1)),
        "one-block": (one, (8, 32, 32)),
    }


CASES = _cases()


def _extra_params(w, block):
    """The workload's Table 7 draw, plus offsets and finite strides on both axes."""
    prm = workload.psa_strategies(w, block)
    more = [(1, 1, math.inf, 2, -1, math.inf), (2, -2, 3, 3, 1, 5), (1, 0, 2, 1, 0, 2)]
    return [more[h % len(more)] if h % 2 else prm[h] for h in range(w.B * w.H)]


def _run_plan(w, block, params):
    sh = svoo.Shape(w.B, w.H, w.N, w.d, w.n_text)
    cfg = svoo.psa_config(w.grid, block, w.block_q)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    plan, k_assign = svoo.psa_mask(sh, w.grid, block, svoo.psa_params(params, "cuda"), cfg, dev_err=err)
    torch.cuda.synchronize()
    return plan, k_assign, err


def _check_plan(w, block, params, plan, k_assign, heads):
    V = plan.views()
    nv = w.n_video
    for h in heads:
        o = oracle.psa_plan(*w.grid, block, w.n_text, params[h])
        G = o["G"]
        km = V["kmask"][h].cpu().numpy().view(np.uint64)
        assert np.array_equal(km, o["kmask"]), (w.name, h, "kmask")
        assert np.array_equal(V["q_label"][h].cpu().numpy(), o["label"]), (w.name, h, "q_label")
        assert np.array_equal(k_assign[h].cpu().numpy(), o["label"][:nv]), (w.name, h, "k_assign")
        assert np.array_equal(V["q_sizes"][h].cpu().numpy(), o["sizes"]), (w.name, h, "q_sizes")
        st = V["stats"][h].cpu().numpy()
        nb = o["nb"]
        bits = ((o["kmask"][:nb, np.arange(nb) // 64] >> (np.arange(nb) % 64).astype(np.uint64)) & np.uint64(1))
        assert st[0] == int(bits.sum()) and st[1] == nb, (w.name, h, "stats")
        tiles = int(sum(-(-int(n) // w.block_q) for n in o["sizes"]))
        assert st[5] == tiles and st[6] == tiles, (w.name, h, "tiles")
        assert G == plan.Gq


@pytest.mark.parametrize("name", list(CASES))
def test_psa_plan_bit_exact(name):
    w, block = CASES[name]
    params = _extra_params(w, block)
    plan, k_assign, err = _run_plan(w, block, params)
    svoo.check_device_errors(err)
    _check_plan(w, block, params, plan, k_assign, range(w.B * w.H))


def test_psa_out_of_range_parameters_flag_and_empty_the_head():
    w, block = CASES["ragged-text"]
    params = _extra_params(w, block)
    params[1] = (1, 0, 0, 1, 0, math.inf)    # Ts = 0: out of range
    plan, k_assign, err = _run_plan(w, block, params)
    assert int(err.item()) == 4
    V = plan.views()
    nb = plan.Gq - 1                          # text group last
    km = V["kmask"][1].cpu().numpy().view(np.uint64)
    bits = (km[:, np.arange(plan.Gq) // 64] >> (np.arange(plan.Gq) % 64).astype(np.uint64)) & np.uint64(1)
    assert bits[:nb, :nb].sum() == 0 and bits[nb].all() and bits[:, nb].all()
    assert V["stats"][1][0].item() == 0
    # the other heads are untouched by the bad one
    _check_plan(w, block, params, plan, k_assign, [0, 2])


def _attention_case(w, block, params, heads, rows_per_head, seed=0):
    q, k, v = workload.make_qkv(w)
    qd, kd, vd = qkv_tensors(q, k, v, w.B, w.H)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, aux = svoo.psa_attention(qd, kd, vd, w.grid, block, svoo.psa_params(params, "cuda"),
                                  n_text=w.n_text, block_q=w.block_q, dev_err=err)
    torch.cuda.synchronize()
    svoo.check_device_errors(err)
    o = from_dev_bf16(out).reshape(w.B * w.H, w.N, w.d)
    scale = scale_of(w.d)
    worst = (0.0, 0.0)
    for h in heads:
        p = oracle.psa_plan(*w.grid, block, w.n_text, params[h])
        rows = sample_rows(w.N, rows_per_head, seed + h)
        ref, _, _ = oracle.attn_rows(q[h], k[h], v[h], scale, p["label"], p["label"], p["kmask"], rows)
        ma, fr = check_attention(o[h][rows], ref, f"{w.name} head {h} {params[h]}")
        worst = (max(worst[0], ma), max(worst[1], fr))
    print(f"psa attention {w.name}: worst max-abs {worst[0]:.3e}, worst rel-Frobenius {worst[1]:.3e}")
    return aux


@pytest.mark.parametrize("name", list(CASES))
def test_psa_attention_end_to_end(name):
    w, block = CASES[name]
    params = _extra_params(w, block)
    rows = w.N if w.N <= 2048 else 512
    _attention_case(w, block, params, range(w.B * w.H), rows)


def test_psa_full_window_equals_dense_attention():
    w, block = CASES["tiny"]
    Tb, Hb, Wb = (-(-a // b) for a, b in zip(w.grid, block))
    params = [(Tb, 0, math.inf, Hb * Wb, 0, math.inf)] * (w.B * w.H)
    q, k, v = workload.make_qkv(w)
    qd, kd, vd = qkv_tensors(q, k, v, w.B, w.H)
    out, _ = svoo.psa_attention(qd, kd, vd, w.grid, block, svoo.psa_params(params, "cuda"),
                                block_q=w.block_q)
    torch.cuda.synchronize()
    o = from_dev_bf16(out).reshape(w.B * w.H, w.N, w.d)
    rows = np.arange(w.N, dtype=np.int32)
    for h in range(w.B * w.H):
        check_attention(o[h], oracle.dense_attn_rows(q[h], k[h], v[h], scale_of(w.d), rows), f"dense {h}")


def test_psa_wan14b_full_size():
    """The Wan 2.1 14B call at full size with the seeded Table 7 mix: every
    head's plan bit for bit, attention on sampled rows of a few heads."""
    w = workload.get("wan2.1-14b")
    block = workload.PSA_BLOCKS[w.name]
    params = workload.psa_strategies(w, block)
    plan, k_assign, err = _run_plan(w, block, params)
    svoo.check_device_errors(err)
    _check_plan(w, block, params, plan, k_assign, range(w.B * w.H))
    del plan, k_assign
    heads = [0, 1, 3]
    _attention_case(w, block, params, heads, 48, seed=5)
