"""Shared helpers of the GPU parity tests (not collected by pytest).

The GPU stages are always fed inputs that came from the generator or from the
oracle, never from another GPU stage, so each comparison is against the oracle
alone.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import workload
from workload import bf16_bits_to_f32

# Tolerances (floating-point attention output against the fp64 oracle on the same mask).
ATTN_MAX_ABS = 2e-2
ATTN_REL_FRO = 1e-2
# Assignments: share of tokens that agree, and the largest relative distance
# gap (D2 - D1) / D2 at which an fp32 evaluation may legitimately pick the
# other cluster than the fp64 oracle.
ASSIGN_AGREE = 0.999
ASSIGN_GAP = 1e-4


def to_dev_bf16(a: np.ndarray, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device)
    return t.view(torch.bfloat16)


def from_dev_bf16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def qkv_tensors(q, k, v, B, H):
    """uint16 [BH, N, d] -> bf16 device [B, H, N, d]."""
    BH, N, d = q.shape
    return tuple(to_dev_bf16(x).view(B, H, N, d) for x in (q, k, v))


def check_assign(gpu_assign, o_assign, best, second, what=""):
    """>= 99.9% agreement; each disagreement sits at a relative gap < 1e-4."""
    g = np.asarray(gpu_assign)
    o = np.asarray(o_assign)
    diff = g != o
    agree = 1.0 - diff.mean()
    gap_max = 0.0
    if diff.any():
        gap = (second[diff] - best[diff]) / np.maximum(second[diff], 1e-30)
        gap_max = float(gap.max())
    assert gap_max < ASSIGN_GAP, f"{what}: {int(diff.sum())} disagreement(s), relative gap up to {gap_max:.3e}"
    assert agree >= ASSIGN_AGREE, f"{what}: agreement {agree:.6f} (gaps below {gap_max:.3e})"
    return agree, int(diff.sum())


# Centroid update: the member sums are exact on both sides (the oracle sums in
# fp64 in token order, the GPU adds fp64 partial sums in any order; with the
# components below 2^-24 counted as zero every partial sum is a multiple of
# 2^-31 below 2^22, which fp64 holds exactly), and both round sum / n once to
# fp32: given the same labels the centroids are bit-identical.


def check_centroids(gpu_cent, x_bits, labels, want, old, what=""):
    """GPU centroids against the oracle's update (want) for the same labels:
    bit-identical, and clusters left empty keep their old centroid exactly."""
    C = want.shape[0]
    n = np.bincount(labels, minlength=C)
    empty = n == 0
    assert np.array_equal(gpu_cent[empty].view(np.uint32), old[empty].view(np.uint32)), what
    diff = gpu_cent.view(np.uint32) != want.astype(np.float32).view(np.uint32)
    assert not diff.any(), f"{what}: {int(diff.sum())} centroid components differ from the oracle's, " \
                           f"largest gap {float(np.abs(gpu_cent.astype(np.float64) - want)[diff].max()):.3e}"


def oracle_plan_heads(w: workload.Workload, q, k, heads, keeps, iters=None, mode=0):
    """Oracle plan (cluster -> mask -> merge -> permutation) of each listed head."""
    out = []
    for i, h in enumerate(heads):
        out.append(oracle.plan_head(q[i], k[i], w.n_qc, w.n_kc, iters if iters else w.iters,
                                    float(keeps[h]) if mode == 0 else 0.0, w.block_q,
                                    n_text=w.n_text, mode=mode,
                                    top_p=float(keeps[h]) if mode == 1 else 0.0))
    return out


def kv_len(p, n_kc, n_text):
    Gk = n_kc + (1 if n_text else 0)
    sizes = np.diff(p["k_off"])
    km = p["kmask"]
    Gq = km.shape[0]
    L = np.zeros(Gq, dtype=np.int64)
    for g in range(Gq):
        for b in range(Gk):
            if (int(km[g, b // 64]) >> (b % 64)) & 1:
                L[g] += sizes[b]
    return L


def inject_plan(plan, plans, src_of_head):
    """Writes oracle plans into the GPU plan buffers; head h gets plans[src_of_head[h]]."""
    V = plan.views()
    cap = plan.tile_cap
    for h, s in enumerate(src_of_head):
        p = plans[s]
        V["kmask"][h].copy_(dev(p["kmask"].view(np.int64)))
        V["q_label"][h].copy_(dev(p["q_label"]))
        sizes = np.diff(p["q_off"]).astype(np.int32)
        V["q_sizes"][h].copy_(dev(sizes))
        V["q_perm"][h].copy_(dev(p["q_perm"]))
        V["q_off"][h].copy_(dev(p["q_off"]))
        V["k_perm"][h].copy_(dev(p["k_perm"]))
        V["k_off"][h].copy_(dev(p["k_off"]))
        t = np.zeros((cap, 4), dtype=np.int32)
        L = kv_len(p, plan.cfg.n_kc, plan.shape.n_text)
        n = p["tiles"].shape[0]
        t[:n, :3] = p["tiles"]
        t[:n, 3] = L[p["tiles"][:, 0]]
        V["tiles"][h].copy_(dev(t))
        V["tile_count"][h] = n
        u = np.zeros((plan.unit_cap, 4), dtype=np.int32)
        nu = 0
        for g in range(len(p["q_off"]) - 1):  # attention work units: 256 rows of one group
            ng = int(p["q_off"][g + 1] - p["q_off"][g])
            for s0 in range(0, ng, 256):
                u[nu] = (g, p["q_off"][g] + s0, min(256, ng - s0), L[g])
                nu += 1
        V["units"][h].copy_(dev(u))
        V["unit_count"][h] = nu


def gather_by_plan(q, k, v, plans, src_of_head):
    """Cluster-ordered copies of Q, K, V by the oracle permutations (numpy indexing)."""
    qp, kp, vp = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    for h, s in enumerate(src_of_head):
        p = plans[s]
        qp[h] = q[h][p["q_perm"]]
        kp[h] = k[h][p["k_perm"]]
        vp[h] = v[h][p["k_perm"]]
    return qp, kp, vp


def check_attention(o_gpu_bf16_rows, o_ref, what=""):
    g = bf16_bits_to_f32(o_gpu_bf16_rows).astype(np.float64)
    err = np.abs(g - o_ref)
    max_abs = float(err.max()) if err.size else 0.0
    fro = float(np.linalg.norm(g - o_ref) / max(np.linalg.norm(o_ref), 1e-30))
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    assert max_abs <= ATTN_MAX_ABS, f"{what}: max abs {max_abs:.3e}"
    assert fro <= ATTN_REL_FRO, f"{what}: relative Frobenius {fro:.3e}"
    return max_abs, fro


def sample_rows(N, n, seed):
    rng = np.random.default_rng(seed)
    if n >= N:
        return np.arange(N, dtype=np.int32)
    return np.sort(rng.choice(N, size=n, replace=False)).astype(np.int32)


def ragged_workload():
    """Small case with a ragged tail, text tokens, empty clusters and d = 128."""
    return workload.Workload("ragged-text", 1, 3, 128, (2, 10, 27), 37, 12, (1, 3, 3), 24, 40, 4,
                             128, 128, "choice", (0.05, 0.3, 1.0), seed=3)


def scale_of(d):
    return float(np.float32(1.0 / math.sqrt(d)))
