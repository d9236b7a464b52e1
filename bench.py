"""Benchmark of the online co-clustered block-sparse attention path on B200.

One step = one attention call of the Wan2.1-14B shape through the whole path
(svoo_cluster -> svoo_build_mask -> svoo_permute -> svoo_sparse_attn) on
seeded synthetic inputs already resident in HBM (Q, K, V = 2.3 GB, larger than
the 126 MB L2, so no flush between steps).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

value = effective TFLOPS of the whole call: algorithmic attention FLOPs on the
kept blocks (4 d sum_g n_g L_g over real tokens after tail merging, the
accounting of PSA's Table 2) divided by the device time of the whole step.
Multi-GPU (torchrun): every rank runs its own call (its own batch element,
weak scaling, no data-path collective); time = max over ranks.
--impl reference times the CPU oracle (the only reference this path has) on a
bounded sample of the same workload and extrapolates by algorithmic work.

--mask psa measures the second plan source instead: PSA's static stripe mask
(svoo_psa_mask -> svoo_permute -> svoo_sparse_attn) on the same call, PSABlock
3 x 8 x 16, per-head parameters drawn from PSA's Table 7 mix.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workload  # noqa: E402

METRIC = "sparse-attn ms/call & effective TFLOPS (% bf16 TC peak) at Wan-14B shape"
METRIC_PSA = "PSA stripe-mask sparse-attn effective TFLOPS (% bf16 TC peak) at Wan-14B shape"
WORKLOAD = "wan2.1-14b"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), float(p["hbm_gbs"]), "measured"
    except Exception:
        return 1590.0, 1400.0, 6650.0, "fallback"


def _config_psa(w, n_gpus, block, params):
    from collections import Counter
    fmt = lambda p: "(" + ",".join("inf" if v == math.inf else str(v) for v in p) + ")"
    top = ", ".join(f"{c} x {n}" for c, n in Counter(fmt(p) for p in params).most_common(3))
    return {
        "workload": f"{w.name}: B=1 per GPU, H={w.H}, N={w.N} ({'x'.join(map(str, w.grid))}), d={w.d}, "
                    f"PSA stripe mask, PSABlock {'x'.join(map(str, block))}, per-head (Tw,To,Ts,Sw,So,Ss) "
                    f"seeded from PSA Table 7's head-count mix (most frequent here: {top})",
        "global_batch": n_gpus,
        "seq_len": w.N,
        "parallelism": f"independent calls per GPU x{n_gpus}",
        "l2": "inputs 2.3 GB per GPU > 126 MB L2; no flush between steps",
    }


def _config(w, n_gpus):
    return {
        "workload": f"{w.name}: B=1 per GPU, H={w.H}, N={w.N} ({'x'.join(map(str, w.grid))}), d={w.d}, "
                    f"{w.n_qc}/{w.n_kc} clusters, {w.iters} k-means iterations, block {w.block_q}x{w.block_q}, "
                    f"per-head keep ratio profile {w.keep_args[0]}-{w.keep_args[1]}",
        "global_batch": n_gpus,
        "seq_len": w.N,
        "parallelism": f"independent calls per GPU x{n_gpus}",
        "l2": "inputs 2.3 GB per GPU > 126 MB L2; no flush between steps",
    }


def _launch_count(iters, psa=False):
    # psa: labels + mask 2; permute 5 (sort, tiles, 3 gathers); attention 1
    if psa:
        return 2 + 5 + 1
    # init x2; round 0: q (nu, assign, finalize) + k (m, nu, assign, finalize);
    # later rounds 4 + 4; mask 3; permute 5; attention 1
    return 2 + 7 + 8 * (iters - 1) + 3 + 5 + 1


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 6:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[2:6]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def _alg_flops(plan, d):
    """4 d sum_g n_g L_g from the plan (post-merge sizes, kept key rows)."""
    import torch
    V = plan.views()
    ksz = (V["k_off"][:, 1:] - V["k_off"][:, :-1]).to(torch.int64)      # [BH, Gk]
    km = V["kmask"]                                                      # [BH, Gq, W]
    Gk = ksz.shape[1]
    bits = torch.arange(Gk, device=km.device)
    kept = ((km[:, :, bits // 64] >> (bits % 64)) & 1).to(torch.int64)  # [BH, Gq, Gk]
    L = (kept * ksz[:, None, :]).sum(-1)                                 # [BH, Gq]
    nq = (V["q_off"][:, 1:] - V["q_off"][:, :-1]).to(torch.int64)
    return 4.0 * d * float((nq * L).sum().item())


def _rank_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def _reduce_max_sum(ms, work, device):
    """Across the ranks (every rank calls it): the largest time and the summed
    work, so the whole-job rate is (work of all ranks) / (slowest rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(ms), float(work)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    f = torch.tensor([float(work)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(f, op=dist.ReduceOp.SUM)
    return float(t.item()), float(f.item())


def _rank_seed(seed, rank):
    """Each rank runs its own batch element: the workload seed shifted by the rank."""
    return seed + rank


TRAFFIC_FILE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "profiles",
                            "sparse_attn_wan14b_traffic.json")
TRAFFIC_FILE_PSA = os.path.join(os.path.dirname(os.path.abspath(__file__)), "profiles",
                                "sparse_attn_wan14b_psa_traffic.json")


def _attn_source_digest():
    import hashlib
    h = hashlib.sha256()
    root = os.path.join(os.path.dirname(os.path.abspath(__file__)), "free_sparse_attention_head_b200", "csrc")
    for name in ("attn.cu", "common.cuh"):
        with open(os.path.join(root, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _attn_traffic(flops, psa=False):
    """DRAM bytes of one attention launch from a committed ncu capture of a
    smaller case (of the same plan source), scaled by the algorithmic FLOPs;
    None when the capture is absent or the kernel's source changed since."""
    try:
        with open(TRAFFIC_FILE_PSA if psa else TRAFFIC_FILE) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("source_sha256") != _attn_source_digest():
        return None
    return rec["dram_bytes"] * flops / rec["alg_flops"]


# ----------------------------------------------------------------------------- CPU oracle


def cpu_oracle_sample(w, head=0, iters=1, attn_rows=64, seed=0):
    """Times the oracle on one head: `iters` clustering rounds, mask + merge +
    permutation, and `attn_rows` query rows of attention; returns the
    extrapolated seconds of one full call and the algorithmic FLOPs."""
    import oracle
    q, k, v = workload.make_qkv(w, heads=[head])
    q, k, v = q[0], k[0], v[0]
    nv = w.n_video
    keep = float(w.keep_ratios()[head])
    t0 = time.perf_counter()
    cl = oracle.cluster(q[:nv], k[:nv], w.n_qc, w.n_kc, iters)
    t1 = time.perf_counter()
    p = oracle.plan_head(q, k, w.n_qc, w.n_kc, iters, keep, w.block_q, n_text=w.n_text, clusters=cl)
    t2 = time.perf_counter()
    rows = np.sort(np.random.default_rng(seed).choice(w.N, attn_rows, replace=False)).astype(np.int32)
    _, _, nk = oracle.attn_rows(q, k, v, p["scale"], p["q_label"], p["k_label"], p["kmask"], rows)
    t3 = time.perf_counter()
    sizes = np.diff(p["q_off"]).astype(np.int64)
    ksz = np.diff(p["k_off"]).astype(np.int64)
    km = p["kmask"]
    Gk = ksz.shape[0]
    L = np.array([sum(ksz[b] for b in range(Gk) if (int(km[g, b // 64]) >> (b % 64)) & 1)
                  for g in range(km.shape[0])], dtype=np.int64)
    head_flops = 4.0 * w.d * float((sizes * L).sum())
    sample_flops = 4.0 * w.d * float(nk.sum())
    BH = w.B * w.H
    # full call: clustering scales with rounds, mask per head, attention by FLOPs
    mean_keep = float(np.mean(w.keep_ratios()))
    full_flops = head_flops * BH * (mean_keep / keep)
    est = (t1 - t0) * (w.iters / iters) * BH + (t2 - t1) * BH + (t3 - t2) * (full_flops / max(sample_flops, 1.0))
    return dict(est_seconds=est, full_flops=full_flops, t_cluster=t1 - t0, t_mask=t2 - t1,
                t_attn=t3 - t2, sample=f"1 head of {w.name} (head {head}, keep {keep:.3f}): {iters} k-means "
                f"round(s) of {w.iters}, mask + tail merge + permutation, {attn_rows} of {w.N} attention rows; "
                f"extrapolated x{w.iters // iters} rounds, x{BH} heads, attention by algorithmic FLOPs",
                sample_seconds=t3 - t0)


def cpu_oracle_sample_psa(w, block, params, head=0, attn_rows=64, seed=0):
    """Times the oracle's stripe-mask plan and `attn_rows` attention rows of one
    head; returns the extrapolated seconds of one full call."""
    import oracle
    q, k, v = workload.make_qkv(w, heads=[head])
    q, k, v = q[0], k[0], v[0]
    BH = w.B * w.H
    t0 = time.perf_counter()
    p = oracle.psa_plan_head(*w.grid, block, w.n_text, params[head], w.block_q)
    t1 = time.perf_counter()
    rows = np.sort(np.random.default_rng(seed).choice(w.N, attn_rows, replace=False)).astype(np.int32)
    _, _, nk = oracle.attn_rows(q, k, v, float(np.float32(1.0 / math.sqrt(w.d))), p["q_label"],
                                p["k_label"], p["kmask"], rows)
    t2 = time.perf_counter()
    full_flops = 0.0
    for h in range(BH):
        o = oracle.psa_plan(*w.grid, block, w.n_text, params[h])
        G = o["G"]
        bits = (o["kmask"][:, np.arange(G) // 64] >> (np.arange(G) % 64).astype(np.uint64)) & np.uint64(1)
        L = (bits.astype(np.int64) * o["sizes"][None, :]).sum(1)
        full_flops += 4.0 * w.d * float((o["sizes"].astype(np.int64) * L).sum())
    sample_flops = 4.0 * w.d * float(nk.sum())
    est = (t1 - t0) * BH + (t2 - t1) * (full_flops / max(sample_flops, 1.0))
    return dict(est_seconds=est, full_flops=full_flops, sample_seconds=t2 - t0,
                sample=f"1 head of {w.name} (head {head}, {params[head]}): stripe-mask plan + permutation, "
                       f"{attn_rows} of {w.N} attention rows; extrapolated x{BH} heads, attention by "
                       f"algorithmic FLOPs")


def run_reference(args):
    rank, world, _ = _rank_env()
    if rank != 0:
        return 0
    w = workload.get(WORKLOAD)
    psa = args.mask == "psa"
    if psa:
        block = workload.PSA_BLOCKS[w.name]
        prm = workload.psa_strategies(w, block)

        def sample(head, rows, seed=0):
            return cpu_oracle_sample_psa(w, block, prm, head=head, attn_rows=rows, seed=seed)
    else:
        def sample(head, rows, seed=0):
            return cpu_oracle_sample(w, head=head, iters=1, attn_rows=rows, seed=seed)
    for _ in range(args.warmup):
        sample(0, 8)
    vals, secs = [], []
    cores = 1
    info = None
    for s in range(args.steps):
        info = sample(s % (w.B * w.H), 32, seed=s)
        vals.append(info["full_flops"] / info["est_seconds"] / 1e12)
        secs.append(info["est_seconds"])
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC_PSA if psa else METRIC, "value": value, "unit": "TFLOPS",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": statistics.median(secs) * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config_psa(w, world, block, prm) if psa else _config(w, world),
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": cores, "kind": "oracle",
                         "sample": info["sample"] + " (one step = one such sample)"},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU


def run_gpu(args):
    import torch
    import torch.distributed as dist

    import free_sparse_attention_head_b200 as svoo
    from free_sparse_attention_head_b200 import build as svoo_build

    rank, world, local = _rank_env()
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if rank == 0:
        svoo_build.build()
    if world > 1:
        dist.barrier()
    svoo.load()

    w = workload.get(WORKLOAD)
    import dataclasses
    w = dataclasses.replace(w, seed=_rank_seed(w.seed, rank))  # this rank's own batch element
    if args.heads:
        w = dataclasses.replace(w, H=args.heads)
    q, k, v = workload.make_qkv(w)
    BH, N, d = w.B * w.H, w.N, w.d

    def as_dev(a):
        return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16).view(w.B, w.H, N, d)

    qd, kd, vd = as_dev(q), as_dev(k), as_dev(v)
    keep = torch.from_numpy(w.keep_ratios()).to(dev)
    psa = args.mask == "psa"
    sh = svoo.make_shape(qd)
    if psa:
        block = workload.PSA_BLOCKS[w.name]
        psa_prm = workload.psa_strategies(w, block)
        params = svoo.psa_params(psa_prm, dev)
        cfg = svoo.psa_config(w.grid, block, w.block_q)
        k_assign = torch.empty(BH, w.n_video, dtype=torch.int32, device=dev)
    else:
        cfg = svoo.Config(n_qc=w.n_qc, n_kc=w.n_kc, iters=w.iters, block_q=w.block_q)
        cws, mws = svoo.workspace_sizes(sh, cfg)
        ws_c = torch.empty(cws, dtype=torch.uint8, device=dev)
        ws_m = torch.empty(mws, dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    plan = svoo.Plan(sh, cfg, dev)
    qp, kp, vp, out = (torch.empty_like(qd) for _ in range(4))
    stream = torch.cuda.current_stream(dev)

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        if psa:
            if evs:
                evs[1].record(stream)
            svoo.psa_mask(sh, w.grid, block, params, cfg, plan=plan, k_assign=k_assign, dev_err=err)
            ka = k_assign
        else:
            cl = svoo.cluster(qd, kd, cfg, workspace=ws_c, dev_err=err)
            if evs:
                evs[1].record(stream)
            svoo.build_mask(sh, cl, keep, cfg, plan=plan, workspace=ws_m, dev_err=err)
            ka = cl["k_assign"]
        if evs:
            evs[2].record(stream)
        svoo.permute(qd, kd, vd, ka, plan, qp=qp, kp=kp, vp=vp, dev_err=err)
        if evs:
            evs[3].record(stream)
        svoo.sparse_attn(qp, kp, vp, plan, out=out, dev_err=err)
        if evs:
            evs[4].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    svoo.check_device_errors(err)
    flops = _alg_flops(plan, d)
    stats = plan.views()["stats"].cpu().numpy()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for s in range(args.steps):
        step(evs[s])
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    svoo.check_device_errors(err)
    total_ms, job_flops = _reduce_max_sum(t_start.elapsed_time(t_end), flops, dev)
    ms_step = total_ms / args.steps
    stage = np.array([[evs[s][i].elapsed_time(evs[s][i + 1]) for i in range(4)] for s in range(args.steps)])
    stage_ms = stage.mean(0)
    attn_ms = float(stage_ms[3])
    burst, sustained, hbm, peak_src = _peaks()
    attn_tflops = flops / (attn_ms * 1e-3) / 1e12
    value = job_flops / (ms_step * 1e-3) / 1e12

    # dense self-path (keep = 1.0, or PSA's full window): same library, every pair kept
    dense_plan = svoo.Plan(sh, cfg, dev)
    if psa:
        Tb, Hb, Wb = (-(-a // b) for a, b in zip(w.grid, block))
        full = svoo.psa_params([(Tb, 0, math.inf, Hb * Wb, 0, math.inf)] * BH, dev)
        svoo.psa_mask(sh, w.grid, block, full, cfg, plan=dense_plan, k_assign=k_assign, dev_err=err)
        svoo.permute(qd, kd, vd, k_assign, dense_plan, qp=qp, kp=kp, vp=vp, dev_err=err)
    else:
        cl = svoo.cluster(qd, kd, cfg, workspace=ws_c, dev_err=err)
        svoo.build_mask(sh, cl, torch.ones_like(keep), cfg, plan=dense_plan, workspace=ws_m, dev_err=err)
        svoo.permute(qd, kd, vd, cl["k_assign"], dense_plan, qp=qp, kp=kp, vp=vp, dev_err=err)
    svoo.sparse_attn(qp, kp, vp, dense_plan, out=out, dev_err=err)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 3
    e0.record(stream)
    for _ in range(reps):
        svoo.sparse_attn(qp, kp, vp, dense_plan, out=out, dev_err=err)
    e1.record(stream)
    torch.cuda.synchronize()
    dense_ms = e0.elapsed_time(e1) / reps
    dense_flops = 4.0 * N * N * d * BH
    svoo.check_device_errors(err)

    # end to end through the public call with host buffers
    qh, kh, vh = (x.cpu().pin_memory() for x in (qd, kd, vd))
    oh = torch.empty(qd.shape, dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(1, min(args.steps, 5))
    torch.cuda.synchronize()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(e2e_steps):
        qd.copy_(qh, non_blocking=True)
        kd.copy_(kh, non_blocking=True)
        vd.copy_(vh, non_blocking=True)
        if psa:
            o_dev, _ = svoo.psa_attention(qd, kd, vd, w.grid, block, params, block_q=w.block_q, dev_err=err)
        else:
            o_dev, _ = svoo.sparse_attention(qd, kd, vd, keep, cfg, dev_err=err)
        oh.copy_(o_dev, non_blocking=True)
    a1.record(stream)
    torch.cuda.synchronize()
    e2e_ms, _ = _reduce_max_sum(a0.elapsed_time(a1) / e2e_steps, flops, dev)
    e2e_val = job_flops / (e2e_ms * 1e-3) / 1e12

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        if psa:
            info = cpu_oracle_sample_psa(w, block, psa_prm, head=0, attn_rows=256)
        else:
            info = cpu_oracle_sample(workload.get(WORKLOAD), head=0, iters=2, attn_rows=256)
        cpu = {"value": info["full_flops"] / info["est_seconds"] / 1e12, "unit": "TFLOPS", "cores": 1,
               "kind": "oracle", "sample": info["sample"],
               "est_ms_per_call": info["est_seconds"] * 1e3, "sample_seconds": info["sample_seconds"]}

    if rank == 0:
        line = {
            "metric": METRIC_PSA if psa else METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded center-mixture Q/K, Gaussian V)",
            "config": _config_psa(w, world, block, psa_prm) if psa else _config(w, world),
            "roofline": {"bound": "tensor", "kernel": "sparse_attn_kernel<128>",
                         "achieved": attn_tflops, "peak": sustained, "unit": "TFLOP/s",
                         "frac": attn_tflops / sustained, "traffic": _attn_traffic(flops, psa),
                         "peak_kind": f"bf16 sustained ({peak_src}); kernel timed inside a long step loop",
                         "frac_of_burst_peak": attn_tflops / burst,
                         "alg_flops_per_launch": flops},
            "stages_ms": ({"psa_mask": float(stage_ms[1]), "permute": float(stage_ms[2]),
                           "attention": attn_ms} if psa else
                          {"cluster": float(stage_ms[0]), "mask_merge": float(stage_ms[1]),
                           "permute": float(stage_ms[2]), "attention": attn_ms}),
            "overhead_ratio": float((stage_ms[0] + stage_ms[1]) / attn_ms),
            "dense_self": {"ms": dense_ms, "tflops": dense_flops / (dense_ms * 1e-3) / 1e12,
                           "alg_tflop": dense_flops / 1e12},
            "kept_pairs_mean": float(stats[:, 0].mean()),
            "query_tiles_before_after_merge": [int(stats[:, 5].sum()), int(stats[:, 6].sum())],
            "e2e": {"value": e2e_val, "unit": "TFLOPS", "ms_per_call": e2e_ms,
                    "h2d_bytes_per_step": 3 * qd.numel() * 2, "d2h_bytes_per_step": qd.numel() * 2},
            "gpu_launches": _launch_count(w.iters, psa) * args.steps,
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_cluster_report(args):
    """Clustering stage alone at the Wan2.1-14B call, three ways (one JSON line,
    not the benchmark line): the cold 10-round co-clustering the bench step
    runs, the same with the identity metric (independent k-means of each side),
    and a 2-round warm start from the cold result (the next timestep's call)."""
    import dataclasses
    import torch

    import free_sparse_attention_head_b200 as svoo
    from free_sparse_attention_head_b200 import build as svoo_build

    svoo_build.build()
    svoo.load()
    dev = torch.device("cuda", 0)
    w = workload.get(WORKLOAD)
    if args.heads:
        w = dataclasses.replace(w, H=args.heads)
    q, k, _ = workload.make_qkv(w)
    as_dev = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16).view(w.B, w.H, w.N, w.d)
    qd, kd = as_dev(q), as_dev(k)
    del q, k
    sh = svoo.make_shape(qd)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    base = svoo.Config(n_qc=w.n_qc, n_kc=w.n_kc, iters=w.iters, block_q=w.block_q)
    ws = torch.empty(svoo.workspace_sizes(sh, base)[0], dtype=torch.uint8, device=dev)
    cold = svoo.cluster(qd, kd, base, workspace=ws, dev_err=err)
    warm_state = (cold["q_cent"], cold["k_cent"], cold["k_sizes"])
    cases = {
        "cold_interaction_10": (base, None),
        "cold_identity_10": (dataclasses.replace(base, metric=1), None),
        "warm_interaction_2": (dataclasses.replace(base, iters=2), warm_state),
    }
    res = {}
    for name, (cfg, warm) in cases.items():
        for _ in range(max(args.warmup, 3)):
            svoo.cluster(qd, kd, cfg, warm=warm, workspace=ws, dev_err=err)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            svoo.cluster(qd, kd, cfg, warm=warm, workspace=ws, dev_err=err)
        e1.record()
        torch.cuda.synchronize()
        svoo.check_device_errors(err)
        res[name] = e0.elapsed_time(e1) / args.steps
    print(json.dumps({"report": "clustering stage, ms per call", "workload": f"{w.name}, H={w.H}, N={w.N}",
                      "steps": args.steps, "warmup": args.warmup, "ms": res}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="svoo", choices=["svoo", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--mask", default="cluster", choices=["cluster", "psa"],
                    help="plan source: online co-clustering (default) or PSA's static stripe mask")
    ap.add_argument("--heads", type=int, default=0,
                    help="run the first H heads only (smaller profiling captures; not a bench line)")
    ap.add_argument("--cluster-report", action="store_true",
                    help="time the clustering stage alone (cold, identity metric, warm start); not a bench line")
    args = ap.parse_args()
    if args.cluster_report:
        return run_cluster_report(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
