"""Attention-fidelity diagnostics of the sparse path against dense attention.

iCATS (sec. 5.2, Table 2; App. D, Table 3) compares its interaction-aware
co-clustering with independent Euclidean clustering by two numbers measured
against exact dense attention: how well the selected query-key pairs match the
ones dense attention ranks highest ("selection overlap"), and the mean squared
error of the attention output. The pages do not spell either out; this module
takes the plainest reading:

* selection overlap of a query row: the row keeps a set S of keys (the key
  groups its merged query group attends, from the plan's mask); T is the |S|
  keys with the largest dense attention weights of that row; the overlap is
  |S and T| / |S|. Also reported: the dense attention mass inside S (recall of
  probability mass), which needs no top-k.
* output MSE: mean over the sampled rows and the head dimension of
  (O_sparse - O_dense)^2, O_sparse being the library's output.

The sparse output comes from the library (its CUDA kernels, unchanged); the
dense rows are plain PyTorch fp32 on a sample of query rows per head, a
measurement and not part of the path.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

from . import Config, Plan, check_device_errors, sparse_attention


def key_groups(plan: Plan) -> torch.Tensor:
    """Key group of every key token, int64 [BH, N], from the plan's k_perm / k_off."""
    v = plan.views()
    BH, N = plan.BH, plan.shape.N
    k_perm = v["k_perm"].long()
    k_off = v["k_off"].long()
    pos = torch.arange(N, device=k_perm.device).expand(BH, N).contiguous()
    gpos = torch.searchsorted(k_off[:, 1:].contiguous(), pos, right=True)
    kg = torch.empty_like(gpos)
    kg.scatter_(1, k_perm, gpos)
    return kg


def selected_keys(kmask_head: torch.Tensor, q_groups: torch.Tensor, k_groups: torch.Tensor) -> torch.Tensor:
    """Bool [R, N]: key j is kept for query row r (bit k_groups[j] of kmask row q_groups[r])."""
    words = kmask_head[q_groups][:, k_groups >> 6]
    return ((words >> (k_groups & 63)) & 1).bool()


def selection_metrics(p: torch.Tensor, sel: torch.Tensor):
    """Per row: (top-|S| overlap, dense mass inside S, |S|) for dense weights p [R, N]."""
    nsel = sel.sum(1)
    order = torch.argsort(p, dim=1, descending=True, stable=True)
    rank = torch.empty_like(order)
    rank.scatter_(1, order, torch.arange(p.shape[1], device=p.device).expand_as(order).contiguous())
    in_top = rank < nsel[:, None]
    overlap = (sel & in_top).sum(1).double() / nsel.clamp(min=1).double()
    mass = (p.double() * sel.double()).sum(1)
    return overlap, mass, nsel


@dataclasses.dataclass
class Fidelity:
    overlap: float       # mean selection overlap over sampled rows and heads
    mass: float          # mean dense attention mass inside the kept set
    mse: float           # mean squared error of O against dense attention
    density: float       # mean fraction of keys kept per sampled row
    per_head: list       # (overlap, mass, mse, density) per head


def fidelity(q, k, v, keep, cfg: Config, n_text: int = 0, rows: int = 256, seed: int = 0,
             scale: Optional[float] = None) -> Fidelity:
    """Runs the sparse path on (q, k, v) [B, H, N, d] bf16 with per-head keep
    values `keep` [B*H] and measures it against dense attention on `rows`
    randomly chosen query tokens of every head."""
    out, aux = sparse_attention(q, k, v, keep, cfg, n_text=n_text)
    torch.cuda.synchronize()
    check_device_errors(aux["dev_err"])
    plan = aux["plan"]
    views = plan.views()
    kg = key_groups(plan)
    B, H, N, d = q.shape
    if scale is None:
        scale = cfg.scale if cfg.scale is not None else 1.0 / math.sqrt(d)
    g = torch.Generator(device="cpu").manual_seed(seed)
    per_head = []
    for bh in range(B * H):
        b, h = divmod(bh, H)
        r = torch.randperm(N, generator=g)[:min(rows, N)].to(q.device)
        qh, kh, vh = q[b, h].float(), k[b, h].float(), v[b, h].float()
        p = torch.softmax((qh[r] @ kh.T) * scale, dim=1)
        o_dense = p @ vh
        sel = selected_keys(views["kmask"][bh], views["q_label"][bh, r].long(), kg[bh])
        overlap, mass, nsel = selection_metrics(p, sel)
        mse = ((out[b, h, r].float() - o_dense) ** 2).mean().item()
        per_head.append((overlap.mean().item(), mass.mean().item(), mse, nsel.double().mean().item() / N))
    n = len(per_head)
    return Fidelity(*(sum(x[i] for x in per_head) / n for i in range(4)), per_head=per_head)


def compare_metrics(q, k, v, keep, cfg: Config, n_text: int = 0, rows: int = 256, seed: int = 0) -> dict:
    """Fidelity of the co-clustering (interaction metric) and of independent
    Euclidean clustering (identity metric) on the same inputs and keep values."""
    res = {}
    for name, metric in (("interaction", 0), ("identity", 1)):
        res[name] = fidelity(q, k, v, keep, dataclasses.replace(cfg, metric=metric), n_text, rows, seed)
    return res
