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
bounded sample of the same workload, one head per host thread, and
extrapolates by algorithmic work; the GPU line's cpu_baseline is the same
sample.

roofline.frac is the attention kernel's algorithmic TFLOP/s over the measured
burst bf16 peak; the line also carries its fraction of the sustained peak, the
warm-started next-timestep clustering (warm_start), achieved GB/s of the
clustering and permutation stages (hbm), and the work density (density).

--workload {wan2.1-1.3b, hunyuanvideo-13b, sweep} prints the line of another
configuration instead (per-call or per-point stage times, TFLOPS, % of peak,
overhead ratio, query tiles before / after merging).

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
    # cold co-clustering call: init x2, |x|^2 x2; round 0: q (nu, assign, fixup,
    # update, finalize) + k (m and the same five); later rounds 6 + 6; mask 3
    # (pair mass, select, tail merge); permute 5; attention 1
    return 2 + 2 + 5 + 6 + 12 * (iters - 1) + 3 + 5 + 1


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


def _rate(flops, ms, peak_tflops):
    """Achieved TFLOP/s of `flops` in `ms` milliseconds and its fraction of a peak."""
    tflops = flops / (ms * 1e-3) / 1e12
    return tflops, tflops / peak_tflops


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


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _plan_flops(p, d):
    """4 d sum_g n_g L_g of one oracle plan (the same count as _alg_flops)."""
    sizes = np.diff(p["q_off"]).astype(np.int64)
    ksz = np.diff(p["k_off"]).astype(np.int64)
    km = p["kmask"]
    G = ksz.shape[0]
    bits = (km[:, np.arange(G) // 64] >> (np.arange(G) % 64).astype(np.uint64)) & np.uint64(1)
    return 4.0 * d * float((sizes * (bits.astype(np.int64) * ksz[None, :]).sum(1)).sum())


def _oracle_head(w, q, k, v, head, keep, iters, attn_rows, seed, psa=None):
    """The oracle on one head: `iters` clustering rounds (or the stripe-mask
    plan), mask + merge + permutation, `attn_rows` rows of attention. Returns
    its seconds and work; runs in a worker thread (the oracle's C calls drop
    the GIL)."""
    import oracle
    t0 = time.perf_counter()
    if psa is None:
        nv = w.n_video
        cl = oracle.cluster(q[:nv], k[:nv], w.n_qc, w.n_kc, iters)
        t1 = time.perf_counter()
        p = oracle.plan_head(q, k, w.n_qc, w.n_kc, iters, keep, w.block_q, n_text=w.n_text, clusters=cl)
        scale = p["scale"]
    else:
        block, prm = psa
        t1 = time.perf_counter()
        p = oracle.psa_plan_head(*w.grid, block, w.n_text, prm, w.block_q)
        scale = float(np.float32(1.0 / math.sqrt(w.d)))
    t2 = time.perf_counter()
    rows = np.sort(np.random.default_rng(seed + head).choice(w.N, attn_rows, replace=False)).astype(np.int32)
    _, _, nk = oracle.attn_rows(q, k, v, scale, p["q_label"], p["k_label"], p["kmask"], rows)
    t3 = time.perf_counter()
    return dict(t_cluster=t1 - t0, t_mask=t2 - t1, t_attn=t3 - t2, head_flops=_plan_flops(p, w.d),
                sample_flops=4.0 * w.d * float(nk.sum()))


def cpu_oracle_sample(w, threads=None, iters=1, attn_rows=32, seed=0, psa=None, qkv=None):
    """One bounded sample of the oracle on the workload, parallel over heads
    (one head per host thread, as an OpenMP loop over (b, h) would run it):
    heads 0 .. n-1 with n = min(threads, B*H), `iters` of the config's k-means
    rounds each, the whole mask / merge / permutation, `attn_rows` attention
    rows per head. A full call is extrapolated from it: clustering by rounds,
    attention by algorithmic work, the heads by B*H / n; on `threads` cores the
    (b, h) loop takes the summed head time / min(threads, B*H).
    Returns both that estimate and the single-core one, with the sample's
    description. Both benchmark arms use this same sample."""
    from concurrent.futures import ThreadPoolExecutor
    BH = w.B * w.H
    threads = max(1, min(threads or host_cores(), BH))
    heads = list(range(threads))
    if qkv is None:
        q, k, v = workload.make_qkv(w, heads=heads)
    else:
        q, k, v = (a[heads] for a in qkv)
    keeps = w.keep_ratios()
    prm = None
    if psa is not None:
        block, params = psa
    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as ex:
        futs = [ex.submit(_oracle_head, w, q[i], k[i], v[i], h, float(keeps[h]), iters, attn_rows, seed,
                          None if psa is None else (block, params[h])) for i, h in enumerate(heads)]
        res = [f.result() for f in futs]
    wall = time.perf_counter() - t0
    rounds = 1.0 if psa is not None else w.iters / iters
    per_head = [r["t_cluster"] * rounds + r["t_mask"] + r["t_attn"] * r["head_flops"] / max(r["sample_flops"], 1.0)
                for r in res]
    scale_heads = BH / len(heads)
    total_cpu = sum(per_head) * scale_heads
    full_flops = sum(r["head_flops"] for r in res) * scale_heads
    if psa is None:
        what = (f"heads 0-{len(heads) - 1} of {w.name} (one per thread): {iters} k-means round(s) of "
                f"{w.iters}, mask + tail merge + permutation, {attn_rows} of {w.N} attention rows each")
        extra = f"x{rounds:g} rounds, "
    else:
        what = (f"heads 0-{len(heads) - 1} of {w.name} (one per thread): stripe-mask plan + permutation, "
                f"{attn_rows} of {w.N} attention rows each")
        extra = ""
    return dict(cores=threads, wall_seconds=wall, est_seconds=total_cpu / threads,
                est_seconds_1core=total_cpu, full_flops=full_flops,
                sample=f"{what}; extrapolated {extra}x{scale_heads:g} heads, attention by algorithmic work")


def _cpu_line(info):
    v = info["full_flops"] / info["est_seconds"] / 1e12
    return {"value": v, "unit": "TFLOPS", "cores": info["cores"], "kind": "oracle", "extrapolated": True,
            "sample": info["sample"], "sample_wall_s": info["wall_seconds"],
            "est_ms_per_call": info["est_seconds"] * 1e3,
            "single_core": {"value": info["full_flops"] / info["est_seconds_1core"] / 1e12,
                            "est_ms_per_call": info["est_seconds_1core"] * 1e3}}


def run_reference(args):
    rank, world, _ = _rank_env()
    if rank != 0:
        return 0
    w = workload.get(WORKLOAD)
    psa = args.mask == "psa"
    prm = block = None
    if psa:
        block = workload.PSA_BLOCKS[w.name]
        prm = workload.psa_strategies(w, block)
    threads = args.cpu_threads or host_cores()
    # the sample's heads 0 .. n-1, generated once (make_qkv's arrays index them 0 .. n-1)
    qkv = workload.make_qkv(w, heads=range(max(1, min(threads, w.B * w.H))))

    def sample():
        return cpu_oracle_sample(w, threads=threads, psa=(block, prm) if psa else None, qkv=qkv)

    for _ in range(args.warmup):
        sample()
    vals, secs, info = [], [], None
    for _ in range(args.steps):
        info = sample()
        vals.append(info["full_flops"] / info["est_seconds"] / 1e12)
        secs.append(info["est_seconds"])
    value = statistics.median(vals)
    cpu = _cpu_line(info)
    cpu["value"] = value
    cpu["sample"] += " (one step = one such sample)"
    line = {
        "impl": "reference", "metric": METRIC_PSA if psa else METRIC, "value": value, "unit": "TFLOPS",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": statistics.median(secs) * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config_psa(w, world, block, prm) if psa else _config(w, world),
        "cpu_baseline": cpu,
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU


class Call:
    """Device buffers and the library calls of one attention call of a
    workload (the whole path), reused across steps so a step allocates nothing."""

    def __init__(self, svoo, w, q, k, v, dev, psa=False):
        import torch
        self.svoo, self.w, self.dev, self.psa = svoo, w, dev, psa
        BH, N, d = w.B * w.H, w.N, w.d

        def as_dev(a):
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16).view(w.B, w.H, N, d)

        self.qd, self.kd, self.vd = as_dev(q), as_dev(k), as_dev(v)
        self.sh = svoo.make_shape(self.qd, w.n_text)
        if psa:
            self.block = workload.PSA_BLOCKS[w.name]
            self.psa_prm = workload.psa_strategies(w, self.block)
            self.params = svoo.psa_params(self.psa_prm, dev)
            self.cfg = svoo.psa_config(w.grid, self.block, w.block_q)
            self.k_assign = torch.empty(BH, w.n_video, dtype=torch.int32, device=dev)
        else:
            self.cfg = svoo.Config(n_qc=w.n_qc, n_kc=w.n_kc, iters=w.iters, block_q=w.block_q)
            cws, mws = svoo.workspace_sizes(self.sh, self.cfg)
            self.ws_c = torch.empty(cws, dtype=torch.uint8, device=dev)
            self.ws_m = torch.empty(mws, dtype=torch.uint8, device=dev)
            self.cl = svoo.cluster_outputs(self.sh, self.cfg, dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.plan = svoo.Plan(self.sh, self.cfg, dev)
        self.qp, self.kp, self.vp, self.out = (torch.empty_like(self.qd) for _ in range(4))
        self.stream = torch.cuda.current_stream(dev)

    def step(self, keep, evs=None, plan=None):
        svoo, s, plan = self.svoo, self.stream, plan or self.plan
        if evs:
            evs[0].record(s)
        if self.psa:
            if evs:
                evs[1].record(s)
            svoo.psa_mask(self.sh, self.w.grid, self.block, self.params, self.cfg, plan=plan,
                          k_assign=self.k_assign, dev_err=self.err)
            ka = self.k_assign
        else:
            svoo.cluster(self.qd, self.kd, self.cfg, n_text=self.w.n_text, workspace=self.ws_c,
                         dev_err=self.err, out=self.cl)
            if evs:
                evs[1].record(s)
            svoo.build_mask(self.sh, self.cl, keep, self.cfg, plan=plan, workspace=self.ws_m, dev_err=self.err)
            ka = self.cl["k_assign"]
        if evs:
            evs[2].record(s)
        svoo.permute(self.qd, self.kd, self.vd, ka, plan, qp=self.qp, kp=self.kp, vp=self.vp, dev_err=self.err)
        if evs:
            evs[3].record(s)
        svoo.sparse_attn(self.qp, self.kp, self.vp, plan, out=self.out, dev_err=self.err)
        if evs:
            evs[4].record(s)


def _timed_steps(call, keep, steps, ev_count=5):
    """`steps` calls with per-stage CUDA events; returns (total ms, stage ms mean [4])."""
    import torch
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(ev_count)] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(call.stream)
    for s in range(steps):
        call.step(keep, evs[s])
    t1.record(call.stream)
    torch.cuda.synchronize()
    stage = np.array([[evs[s][i].elapsed_time(evs[s][i + 1]) for i in range(4)] for s in range(steps)])
    return t0.elapsed_time(t1), stage.mean(0)


def _event_ms(fn, reps, stream):
    import torch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def _bytes_fields(w, stage_ms, hbm):
    """Achieved GB/s of the HBM-bound stages: clustering reads X (queries and
    keys, d bf16 values per video token) once per half-step; the permutation
    stage reads Q, K, V and writes their cluster-ordered copies."""
    BH = w.B * w.H
    x_bytes = 2.0 * BH * w.n_video * w.d * 2 * w.iters
    perm_bytes = 6.0 * BH * w.N * w.d * 2
    out = {"cluster_x_bytes": x_bytes, "cluster_gbs": x_bytes / (stage_ms[0] * 1e-3) / 1e9,
           "permute_bytes": perm_bytes, "permute_gbs": perm_bytes / (stage_ms[2] * 1e-3) / 1e9,
           "peak_gbs": hbm}
    out["cluster_frac"] = out["cluster_gbs"] / hbm
    out["permute_frac"] = out["permute_gbs"] / hbm
    return out


def run_gpu(args):
    import dataclasses

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
    w = dataclasses.replace(w, seed=_rank_seed(w.seed, rank))  # this rank's own batch element
    if args.heads:
        w = dataclasses.replace(w, H=args.heads)
    q, k, v = workload.make_qkv(w)
    BH, N, d = w.B * w.H, w.N, w.d
    psa = args.mask == "psa"
    call = Call(svoo, w, q, k, v, dev, psa=psa)
    keep = torch.from_numpy(w.keep_ratios()).to(dev)
    stream = call.stream

    for _ in range(max(args.warmup, 3)):
        call.step(keep)
    torch.cuda.synchronize()
    svoo.check_device_errors(call.err)
    flops = _alg_flops(call.plan, d)
    stats = call.plan.views()["stats"].cpu().numpy()
    dense_flops = 4.0 * N * N * d * BH

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    total_ms, stage_ms = _timed_steps(call, keep, args.steps)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    svoo.check_device_errors(call.err)
    total_ms, job_flops = _reduce_max_sum(total_ms, flops, dev)
    ms_step = total_ms / args.steps
    attn_ms = float(stage_ms[3])
    burst, sustained, hbm, peak_src = _peaks()
    attn_tflops, frac_burst = _rate(flops, attn_ms, burst)
    value = job_flops / (ms_step * 1e-3) / 1e12

    # warm start: the next timestep's call (inputs drifted by a seeded
    # perturbation) clustered from this call's clusters, `warm_iters` rounds
    warm = None
    if not psa:
        q2 = workload.next_timestep(q, 0.1, seed=11)
        k2 = workload.next_timestep(k, 0.1, seed=12)
        q2d = torch.from_numpy(q2.view(np.int16)).to(dev).view(torch.bfloat16).view(w.B, w.H, N, d)
        k2d = torch.from_numpy(k2.view(np.int16)).to(dev).view(torch.bfloat16).view(w.B, w.H, N, d)
        del q2, k2
        wcfg = dataclasses.replace(call.cfg, iters=args.warm_iters)
        wout = svoo.cluster_outputs(call.sh, wcfg, dev)
        state = [t.clone() for t in (call.cl["q_cent"], call.cl["k_cent"], call.cl["k_sizes"])]

        def warm_call():
            svoo.cluster(q2d, k2d, wcfg, warm=state, workspace=call.ws_c, dev_err=call.err, out=wout)

        for _ in range(3):
            warm_call()
        warm_ms = _event_ms(warm_call, max(3, min(args.steps, 10)), stream)
        warm = {"rounds": args.warm_iters, "cluster_ms": warm_ms,
                "overhead_ratio": (warm_ms + float(stage_ms[1])) / attn_ms,
                "inputs": "next timestep: Q, K + 0.1 N(0, I) (seeded), clusters of this call as the start"}
        del q2d, k2d
        svoo.check_device_errors(call.err)

    # dense self-path (keep = 1.0, or PSA's full window): same library, every pair kept
    dense_plan = svoo.Plan(call.sh, call.cfg, dev)
    if psa:
        Tb, Hb, Wb = (-(-a // b) for a, b in zip(w.grid, call.block))
        full = svoo.psa_params([(Tb, 0, math.inf, Hb * Wb, 0, math.inf)] * BH, dev)
        svoo.psa_mask(call.sh, w.grid, call.block, full, call.cfg, plan=dense_plan, k_assign=call.k_assign,
                      dev_err=call.err)
        svoo.permute(call.qd, call.kd, call.vd, call.k_assign, dense_plan, qp=call.qp, kp=call.kp, vp=call.vp,
                     dev_err=call.err)
    else:
        call.step(torch.ones_like(keep), plan=dense_plan)
    dense_ms = _event_ms(lambda: svoo.sparse_attn(call.qp, call.kp, call.vp, dense_plan, out=call.out,
                                                  dev_err=call.err), 3, stream)
    svoo.check_device_errors(call.err)
    del dense_plan

    # end to end through the public call with host buffers
    qh, kh, vh = (x.cpu().pin_memory() for x in (call.qd, call.kd, call.vd))
    oh = torch.empty(call.qd.shape, dtype=torch.bfloat16).pin_memory()

    def e2e_call():
        call.qd.copy_(qh, non_blocking=True)
        call.kd.copy_(kh, non_blocking=True)
        call.vd.copy_(vh, non_blocking=True)
        if psa:
            o_dev, _ = svoo.psa_attention(call.qd, call.kd, call.vd, w.grid, call.block, call.params,
                                          block_q=w.block_q, dev_err=call.err)
        else:
            o_dev, _ = svoo.sparse_attention(call.qd, call.kd, call.vd, keep, call.cfg, dev_err=call.err)
        oh.copy_(o_dev, non_blocking=True)

    torch.cuda.synchronize()
    e2e_ms, _ = _reduce_max_sum(_event_ms(e2e_call, max(1, min(args.steps, 5)), stream), flops, dev)
    e2e_val = job_flops / (e2e_ms * 1e-3) / 1e12

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        info = cpu_oracle_sample(w, threads=args.cpu_threads or host_cores(),
                                 psa=(call.block, call.psa_prm) if psa else None, qkv=(q, k, v))
        cpu = _cpu_line(info)

    if rank == 0:
        per_head = _alg_flops_per_head(call.plan, d) / (4.0 * N * N * d)
        line = {
            "metric": METRIC_PSA if psa else METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded center-mixture Q/K, Gaussian V)",
            "config": _config_psa(w, world, call.block, call.psa_prm) if psa else _config(w, world),
            "roofline": {"bound": "tensor", "kernel": "sparse_attn_kernel<128>",
                         "achieved": attn_tflops, "peak": burst, "unit": "TFLOP/s", "frac": frac_burst,
                         "traffic": _attn_traffic(flops, psa),
                         "peak_kind": f"bf16 dense burst ({peak_src}, MEASURED_PEAKS bf16_tflops)",
                         "frac_of_sustained_peak": attn_tflops / sustained, "sustained_peak": sustained,
                         "alg_flops_per_launch": flops},
            "stages_ms": ({"psa_mask": float(stage_ms[1]), "permute": float(stage_ms[2]),
                           "attention": attn_ms} if psa else
                          {"cluster": float(stage_ms[0]), "mask_merge": float(stage_ms[1]),
                           "permute": float(stage_ms[2]), "attention": attn_ms}),
            "overhead_ratio": float((stage_ms[0] + stage_ms[1]) / attn_ms),
            "warm_start": warm,
            "hbm": _bytes_fields(w, stage_ms, hbm) if not psa else
            {"permute_gbs": 6.0 * BH * N * d * 2 / (stage_ms[2] * 1e-3) / 1e9, "peak_gbs": hbm},
            "dense_self": {"ms": dense_ms, "tflops": dense_flops / (dense_ms * 1e-3) / 1e12,
                           "alg_tflop": dense_flops / 1e12},
            "density": {"flops_vs_dense": flops / dense_flops, "per_head_min": float(per_head.min()),
                        "per_head_max": float(per_head.max()),
                        "kept_pairs_mean": float(stats[:, 0].mean()),
                        "keep_ratio_mean": float(np.mean(w.keep_ratios()))},
            "query_tiles_before_after_merge": [int(stats[:, 5].sum()), int(stats[:, 6].sum())],
            "e2e": {"value": e2e_val, "unit": "TFLOPS", "ms_per_call": e2e_ms,
                    "h2d_bytes_per_step": 3 * call.qd.numel() * 2, "d2h_bytes_per_step": call.qd.numel() * 2},
            "gpu_launches": _launch_count(w.iters, psa) * args.steps,
            "clocks": clocks,
            "attention_gcycles": (attn_ms * 1e-3 * clocks["sm_mhz"] * 1e6 / 1e9) if clocks.get("sm_mhz") else None,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def _alg_flops_per_head(plan, d):
    """4 d sum_g n_g L_g of every head (numpy [BH])."""
    import torch
    V = plan.views()
    ksz = (V["k_off"][:, 1:] - V["k_off"][:, :-1]).to(torch.int64)
    km = V["kmask"]
    Gk = ksz.shape[1]
    bits = torch.arange(Gk, device=km.device)
    kept = ((km[:, :, bits // 64] >> (bits % 64)) & 1).to(torch.int64)
    L = (kept * ksz[:, None, :]).sum(-1)
    nq = (V["q_off"][:, 1:] - V["q_off"][:, :-1]).to(torch.int64)
    return 4.0 * d * (nq * L).sum(-1).double().cpu().numpy()


def run_config(args):
    """Bench lines of the other configurations (not the headline): the
    Wan2.1-1.3B call; the HunyuanVideo-13B schedule of 50 calls with
    r(t) = 0.1 + 0.4 (1 - t/50) and 256 text tokens; the 25-point sweep
    (N x keep ratio, Zipf-skewed clusters). One JSON line each, with per-call
    or per-point stage times, TFLOPS, % of the burst peak, overhead ratio and
    query tiles before / after merging."""
    import dataclasses

    import torch

    import free_sparse_attention_head_b200 as svoo
    from free_sparse_attention_head_b200 import build as svoo_build

    svoo_build.build()
    svoo.load()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    burst, _, hbm, peak_src = _peaks()
    steps = max(1, args.steps)

    def measure(w, keeps_list, label_fn):
        q, k, v = workload.make_qkv(w)
        call = Call(svoo, w, q, k, v, dev)
        del q, k, v
        d, N, BH = w.d, w.N, w.B * w.H
        points = []
        for keep_np in keeps_list:
            keep = torch.from_numpy(np.asarray(keep_np, np.float32)).to(dev)
            for _ in range(max(args.warmup, 2)):
                call.step(keep)
            torch.cuda.synchronize()
            svoo.check_device_errors(call.err)
            flops = _alg_flops(call.plan, d)
            stats = call.plan.views()["stats"].cpu().numpy()
            total_ms, st = _timed_steps(call, keep, steps)
            svoo.check_device_errors(call.err)
            tf, fr = _rate(flops, float(st[3]), burst)
            points.append(dict(label_fn(keep_np), ms_per_call=total_ms / steps,
                               stages_ms={"cluster": float(st[0]), "mask_merge": float(st[1]),
                                          "permute": float(st[2]), "attention": float(st[3])},
                               attn_tflops=tf, frac_of_burst=fr, alg_tflop=flops / 1e12,
                               flops_vs_dense=flops / (4.0 * N * N * d * BH),
                               overhead_ratio=float((st[0] + st[1]) / st[3]),
                               effective_tflops=flops / (total_ms / steps * 1e-3) / 1e12,
                               query_tiles_before_after_merge=[int(stats[:, 5].sum()), int(stats[:, 6].sum())]))
        del call
        torch.cuda.empty_cache()
        return points

    name = args.workload
    if name == "wan2.1-1.3b":
        w = workload.get(name)
        pts = measure(w, [w.keep_ratios()], lambda kp: {"keep_ratios": sorted(set(map(float, kp)))})
    elif name == "hunyuanvideo-13b":
        w = workload.get(name)
        pts = measure(w, [w.keep_ratios(t=t) for t in range(50)], lambda kp: {"keep": float(kp[0])})
        for t, p in enumerate(pts):
            p["t"] = t
    elif name == "sweep":
        pts = []
        for n_tok in (8192, 16384, 32768, 65536, 131072):
            w = workload.sweep_workload(n_tok, 1.0)
            keeps = [np.full(w.B * w.H, r, np.float32) for r in (0.05, 0.1, 0.25, 0.5, 1.0)]
            got = measure(w, keeps, lambda kp, n=n_tok: {"N": n, "keep": float(kp[0])})
            pts.extend(got)
            w_last = w
        w = w_last
    else:
        raise SystemExit(f"unknown workload {name}")
    tot_flops = sum(p["alg_tflop"] for p in pts) * 1e12
    tot_ms = sum(p["ms_per_call"] for p in pts)
    attn_ms = sum(p["stages_ms"]["attention"] for p in pts)
    line = {
        "metric": f"sparse-attn effective TFLOPS (% bf16 TC peak), {name}", "workload": name,
        "value": tot_flops / (tot_ms * 1e-3) / 1e12, "unit": "TFLOPS", "n_gpus": 1, "steps": steps,
        "warmup": args.warmup, "ms_per_call_mean": tot_ms / len(pts), "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic (seeded center-mixture Q/K, Gaussian V)",
        "attention": {"tflops": tot_flops / (attn_ms * 1e-3) / 1e12,
                      "frac_of_burst": tot_flops / (attn_ms * 1e-3) / 1e12 / burst,
                      "peak": burst, "peak_kind": f"bf16 dense burst ({peak_src})"},
        "overhead_ratio": sum(p["stages_ms"]["cluster"] + p["stages_ms"]["mask_merge"] for p in pts) / attn_ms,
        "points": pts,
    }
    print(json.dumps(line), flush=True)
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
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=[WORKLOAD, "wan2.1-1.3b", "hunyuanvideo-13b", "sweep"],
                    help="configuration: the headline Wan2.1-14B step (default) or another config's line")
    ap.add_argument("--warm-iters", type=int, default=2,
                    help="k-means rounds of the warm-started next-timestep clustering the line reports")
    ap.add_argument("--cpu-threads", type=int, default=0,
                    help="host threads of the CPU-oracle sample (default: every core of this process)")
    args = ap.parse_args()
    if args.cluster_report:
        return run_cluster_report(args)
    if args.impl == "reference":
        return run_reference(args)
    if args.workload != WORKLOAD:
        return run_config(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
