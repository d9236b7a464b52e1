"""Python binding of libsvoo (online QK co-clustered block-sparse attention, sm_100a).

Argument marshalling only: every step runs in the library's CUDA kernels
(`csrc/`, C ABI in `include/svoo.h`). PyTorch provides device memory and the
current CUDA stream. If the compiled library is missing or no CUDA device is
present, calls raise; there is no CPU fallback.

Typical use (all tensors on one CUDA device, bf16 [B, H, N, d]):

    import free_sparse_attention_head_b200 as svoo
    cfg = svoo.Config(n_qc=256, n_kc=256, iters=10, block_q=128)
    out, plan = svoo.sparse_attention(q, k, v, keep, cfg)
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
from typing import Optional

import torch

__all__ = [
    "Config", "Shape", "Plan", "load", "lib_path", "cluster", "cluster_step", "build_mask",
    "permute", "sparse_attn", "sparse_attention", "check_device_errors", "workspace_sizes",
    "SvooError", "CLUSTER_WARM", "CLUSTER_IDENTITY", "PSA_INF", "psa_config", "psa_params",
    "psa_mask", "psa_attention", "snr_top_p", "cluster_outputs",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libsvoo.so")
_lib = None


class SvooError(RuntimeError):
    pass


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int), ("d", ctypes.c_int),
                ("n_text", ctypes.c_int)]


_PLAN_FIELDS = ["kmask", "q_label", "q_sizes", "stats", "q_perm", "q_off", "k_perm", "k_off",
                "tiles", "tile_count", "units", "unit_count"]


class _CPlan(ctypes.Structure):
    _fields_ = [(f, ctypes.c_void_p) for f in _PLAN_FIELDS]


_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t
_SP = ctypes.POINTER(Shape)
_PP = ctypes.POINTER(_CPlan)

_SIGS = {
    "svoo_status_string": (ctypes.c_char_p, [_I]),
    "svoo_version": (_I, []),
    "svoo_plan_counts": (_I, [_SP, _I, _I, _I, ctypes.POINTER(ctypes.c_int64)]),
    "svoo_cluster_workspace_size": (_SZ, [_SP, _I, _I]),
    "svoo_cluster": (_I, [_SP, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _SZ, _P, _P]),
    "svoo_cluster_step": (_I, [_SP, _P, _I, _P, _P, _P, _P, _P, _I, _P, _SZ, _P, _P]),
    "svoo_cluster_step_static": (_I, [_SP, _P, _I, _P, _P, _P, _P, _P, _I, _P, _P]),
    "svoo_mask_workspace_size": (_SZ, [_SP, _I, _I]),
    "svoo_build_mask": (_I, [_SP, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _PP, _P, _SZ,
                             _P, _P]),
    "svoo_permute": (_I, [_SP, _P, _P, _P, _P, _I, _I, _I, _PP, _P, _P, _P, _P, _P]),
    "svoo_sparse_attn": (_I, [_SP, _P, _P, _P, _PP, _I, _I, _I, _F, _P, _P, _P]),
    "svoo_psa_block_count": (_I, [_I, _I, _I, _I, _I, _I]),
    "svoo_psa_mask": (_I, [_SP, _I, _I, _I, _I, _I, _I, _P, _I, _PP, _P, _P, _P]),
    "svoo_snr_top_p": (_I, [_I, _I, ctypes.c_double, ctypes.c_double, ctypes.c_double, _P]),
}

EXPORTS = tuple(_SIGS)


def lib_path() -> str:
    return _LIB_PATH


def load(path: Optional[str] = None):
    """Loads libsvoo.so (built by `free_sparse_attention_head_b200.build`)."""
    global _lib
    if _lib is None:
        p = path or _LIB_PATH
        if not os.path.exists(p):
            raise SvooError(f"{p} is missing: run `python -m free_sparse_attention_head_b200.build`")
        L = ctypes.CDLL(p)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int, what: str):
    if status != 0:
        msg = load().svoo_status_string(status).decode()
        raise SvooError(f"{what}: {msg} (status {status})")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise SvooError("tensors must live on a CUDA device")
        if not t.is_contiguous():
            raise SvooError("tensors must be contiguous")


@dataclasses.dataclass
class Config:
    n_qc: int = 256
    n_kc: int = 256
    iters: int = 10
    block_q: int = 128
    select_mode: int = 0          # 0 keep ratio, 1 top-p
    merge_rounds: int = 2
    scale: Optional[float] = None  # default 1/sqrt(d)
    metric: int = 0               # 0 QK interaction (co-clustering), 1 identity (independent)


def make_shape(q: torch.Tensor, n_text: int = 0) -> Shape:
    if q.dim() != 4:
        raise SvooError("q/k/v must be [B, H, N, d]")
    B, H, N, d = q.shape
    return Shape(B, H, N, d, n_text)


class Plan:
    """Device buffers of one call's sparse plan (see svoo_plan in include/svoo.h)."""

    def __init__(self, shape: Shape, cfg: Config, device):
        counts = (ctypes.c_int64 * 12)()
        _check(load().svoo_plan_counts(ctypes.byref(shape), cfg.n_qc, cfg.n_kc, cfg.block_q, counts),
               "svoo_plan_counts")
        self.shape = shape
        self.cfg = cfg
        self.kmask = torch.zeros(counts[0], dtype=torch.int64, device=device)
        ints = {}
        for i, f in enumerate(_PLAN_FIELDS[1:], start=1):
            ints[f] = torch.zeros(counts[i], dtype=torch.int32, device=device)
        self.__dict__.update(ints)
        self._c = _CPlan(*[t.data_ptr() for t in [self.kmask] + [ints[f] for f in _PLAN_FIELDS[1:]]])

    @property
    def c(self):
        return ctypes.byref(self._c)

    @property
    def BH(self) -> int:
        return self.shape.B * self.shape.H

    @property
    def Gq(self) -> int:
        return self.cfg.n_qc + (1 if self.shape.n_text > 0 else 0)

    @property
    def Gk(self) -> int:
        return self.cfg.n_kc + (1 if self.shape.n_text > 0 else 0)

    @property
    def W(self) -> int:
        return (self.Gk + 63) // 64

    @property
    def tile_cap(self) -> int:
        return (self.shape.N + self.cfg.block_q - 1) // self.cfg.block_q + self.Gq

    @property
    def unit_cap(self) -> int:
        return (self.shape.N + 255) // 256 + self.Gq

    def views(self) -> dict:
        """Per-head views of the plan arrays (still on the device)."""
        BH, N = self.BH, self.shape.N
        return dict(
            kmask=self.kmask.view(BH, self.Gq, self.W),
            q_label=self.q_label.view(BH, N),
            q_sizes=self.q_sizes.view(BH, self.Gq),
            stats=self.stats.view(BH, 8),
            q_perm=self.q_perm.view(BH, N),
            q_off=self.q_off.view(BH, self.Gq + 1),
            k_perm=self.k_perm.view(BH, N),
            k_off=self.k_off.view(BH, self.Gk + 1),
            tiles=self.tiles.view(BH, self.tile_cap, 4),
            tile_count=self.tile_count.view(BH),
            units=self.units.view(BH, self.unit_cap, 4),
            unit_count=self.unit_count.view(BH),
        )


def workspace_sizes(shape: Shape, cfg: Config) -> tuple:
    L = load()
    c = L.svoo_cluster_workspace_size(ctypes.byref(shape), cfg.n_qc, cfg.n_kc)
    m = L.svoo_mask_workspace_size(ctypes.byref(shape), cfg.n_qc, cfg.n_kc)
    if c == 0 or m == 0:
        raise SvooError("unsupported shape or cluster counts")
    return int(c), int(m)


def _err_buf(dev_err, device):
    return dev_err if dev_err is not None else torch.zeros(1, dtype=torch.int32, device=device)


def check_device_errors(dev_err: torch.Tensor):
    """Raises if the device error word has bits set (synchronises the stream)."""
    v = int(dev_err.item())
    if v:
        names = {1: "attention wait timeout", 2: "clustering wait timeout", 4: "plan out of range",
                 8: "cluster label out of range"}
        raise SvooError("device error: " + ", ".join(n for b, n in names.items() if v & b))


CLUSTER_WARM = 1
CLUSTER_IDENTITY = 2


def _cluster_flags(cfg: Config, warm) -> int:
    if cfg.metric not in (0, 1):
        raise SvooError(f"Config.metric must be 0 (QK interaction) or 1 (identity), not {cfg.metric}")
    return (CLUSTER_WARM if warm is not None else 0) | (CLUSTER_IDENTITY if cfg.metric == 1 else 0)


_CLUSTER_OUT = ("q_assign", "k_assign", "q_cent", "k_cent", "q_sizes", "k_sizes")


def cluster_outputs(shape: Shape, cfg: Config, device) -> dict:
    """Device output buffers of `cluster` for a shape, to be reused across calls."""
    BH, nv, d = shape.B * shape.H, shape.N - shape.n_text, shape.d
    return dict(
        q_assign=torch.empty(BH, nv, dtype=torch.int32, device=device),
        k_assign=torch.empty(BH, nv, dtype=torch.int32, device=device),
        q_cent=torch.empty(BH, cfg.n_qc, d, dtype=torch.float32, device=device),
        k_cent=torch.empty(BH, cfg.n_kc, d, dtype=torch.float32, device=device),
        q_sizes=torch.zeros(BH, cfg.n_qc, dtype=torch.int32, device=device),
        k_sizes=torch.zeros(BH, cfg.n_kc, dtype=torch.int32, device=device),
    )


def cluster(q, k, cfg: Config, n_text=0, warm=None, workspace=None, dev_err=None, stream=None,
            out: Optional[dict] = None):
    """Co-clusters the video tokens of every head; returns a dict of device tensors.

    `out` (from cluster_outputs) is written in place instead of allocating new
    outputs. warm = (q_cent, k_cent, k_sizes) starts from those centroids
    (SVOO_CLUSTER_WARM); they may be out's own tensors (the previous call's
    result), in which case nothing is copied."""
    _need_cuda(q, k)
    sh = make_shape(q, n_text)
    dev = q.device
    if workspace is None:
        workspace = torch.empty(workspace_sizes(sh, cfg)[0], dtype=torch.uint8, device=dev)
    if out is None:
        out = cluster_outputs(sh, cfg, dev)
    else:
        missing = [f for f in _CLUSTER_OUT if f not in out]
        if missing:
            raise SvooError(f"cluster(out=...) lacks {missing}")
        _need_cuda(*(out[f] for f in _CLUSTER_OUT))
    if warm is not None:
        for dst, src in zip(("q_cent", "k_cent", "k_sizes"), warm):
            if out[dst].data_ptr() != src.data_ptr():
                out[dst].copy_(src)
    err = _err_buf(dev_err, dev)
    _check(load().svoo_cluster(ctypes.byref(sh), _ptr(q), _ptr(k), cfg.n_qc, cfg.n_kc, cfg.iters,
                               _cluster_flags(cfg, warm), _ptr(out["q_assign"]), _ptr(out["k_assign"]),
                               _ptr(out["q_cent"]), _ptr(out["k_cent"]), _ptr(out["q_sizes"]),
                               _ptr(out["k_sizes"]), _ptr(workspace), workspace.numel(), _ptr(err),
                               _stream(stream)), "svoo_cluster")
    out["dev_err"] = err
    return out


def cluster_step(x, cent, sizes, assign, metric_cent=None, metric_sizes=None, n_text=0,
                 workspace=None, dev_err=None, stream=None):
    """One assignment + update half-step (cent, sizes, assign are updated in place)."""
    _need_cuda(x, cent, sizes, assign, metric_cent, metric_sizes)
    sh = make_shape(x, n_text)
    C = cent.shape[-2]
    mC = metric_cent.shape[-2] if metric_cent is not None else 0
    cfg = Config(n_qc=max(C, mC, 1), n_kc=max(C, mC, 1))
    if workspace is None:
        workspace = torch.empty(workspace_sizes(sh, cfg)[0], dtype=torch.uint8, device=x.device)
    err = _err_buf(dev_err, x.device)
    _check(load().svoo_cluster_step(ctypes.byref(sh), _ptr(x), C, _ptr(cent), _ptr(sizes),
                                    _ptr(assign), _ptr(metric_cent), _ptr(metric_sizes), mC,
                                    _ptr(workspace), workspace.numel(), _ptr(err), _stream(stream)),
           "svoo_cluster_step")
    return err


def cluster_step_static(x, cent, sizes, assign, metric_cent=None, metric_sizes=None, n_text=0,
                        dev_err=None, stream=None):
    """cluster_step with the library's fixed device scratch instead of a
    workspace (for callers that may not allocate device memory)."""
    _need_cuda(x, cent, sizes, assign, metric_cent, metric_sizes)
    sh = make_shape(x, n_text)
    C = cent.shape[-2]
    mC = metric_cent.shape[-2] if metric_cent is not None else 0
    err = _err_buf(dev_err, x.device)
    _check(load().svoo_cluster_step_static(ctypes.byref(sh), _ptr(x), C, _ptr(cent), _ptr(sizes),
                                           _ptr(assign), _ptr(metric_cent), _ptr(metric_sizes), mC,
                                           _ptr(err), _stream(stream)), "svoo_cluster_step_static")
    return err


def build_mask(shape: Shape, cl: dict, keep: torch.Tensor, cfg: Config, plan: Optional[Plan] = None,
               workspace=None, dev_err=None, stream=None) -> Plan:
    """Pair masses, keep-ratio / top-p selection and tail merging into `plan`."""
    dev = cl["q_cent"].device
    keep = keep.to(device=dev, dtype=torch.float32).contiguous()
    _need_cuda(keep, cl["q_cent"], cl["k_cent"], cl["q_sizes"], cl["k_sizes"], cl["q_assign"])
    if plan is None:
        plan = Plan(shape, cfg, dev)
    if workspace is None:
        workspace = torch.empty(workspace_sizes(shape, cfg)[1], dtype=torch.uint8, device=dev)
    scale = cfg.scale if cfg.scale is not None else 1.0 / math.sqrt(shape.d)
    err = _err_buf(dev_err, dev)
    _check(load().svoo_build_mask(ctypes.byref(shape), _ptr(cl["q_cent"]), _ptr(cl["k_cent"]),
                                  _ptr(cl["q_sizes"]), _ptr(cl["k_sizes"]), _ptr(cl["q_assign"]),
                                  _ptr(keep), cfg.n_qc, cfg.n_kc, cfg.select_mode, cfg.block_q,
                                  cfg.merge_rounds, scale, plan.c, _ptr(workspace),
                                  workspace.numel(), _ptr(err), _stream(stream)), "svoo_build_mask")
    return plan


def permute(q, k, v, k_assign, plan: Plan, qp=None, kp=None, vp=None, dev_err=None, stream=None):
    """Cluster-order permutation, query tiles and gathered copies (qp, kp, vp)."""
    _need_cuda(q, k, v, k_assign)
    qp = torch.empty_like(q) if qp is None else qp
    kp = torch.empty_like(k) if kp is None else kp
    vp = torch.empty_like(v) if vp is None else vp
    err = _err_buf(dev_err, q.device)
    cfg = plan.cfg
    _check(load().svoo_permute(ctypes.byref(plan.shape), _ptr(q), _ptr(k), _ptr(v), _ptr(k_assign),
                               cfg.n_qc, cfg.n_kc, cfg.block_q, plan.c, _ptr(qp), _ptr(kp), _ptr(vp),
                               _ptr(err), _stream(stream)), "svoo_permute")
    return qp, kp, vp


def sparse_attn(qp, kp, vp, plan: Plan, out=None, dev_err=None, stream=None):
    """Block-sparse attention over the plan's kept tiles; returns O in token order."""
    _need_cuda(qp, kp, vp)
    out = torch.empty_like(qp) if out is None else out
    cfg = plan.cfg
    scale = cfg.scale if cfg.scale is not None else 1.0 / math.sqrt(plan.shape.d)
    err = _err_buf(dev_err, qp.device)
    _check(load().svoo_sparse_attn(ctypes.byref(plan.shape), _ptr(qp), _ptr(kp), _ptr(vp), plan.c,
                                   cfg.n_qc, cfg.n_kc, cfg.block_q, scale, _ptr(out), _ptr(err),
                                   _stream(stream)), "svoo_sparse_attn")
    return out


def sparse_attention(q, k, v, keep, cfg: Config, n_text=0, dev_err=None, stream=None):
    """The whole path: cluster -> mask + tail merge -> permute -> sparse attention."""
    sh = make_shape(q, n_text)
    err = _err_buf(dev_err, q.device)
    cl = cluster(q, k, cfg, n_text=n_text, dev_err=err, stream=stream)
    plan = build_mask(sh, cl, keep, cfg, dev_err=err, stream=stream)
    qp, kp, vp = permute(q, k, v, cl["k_assign"], plan, dev_err=err, stream=stream)
    out = sparse_attn(qp, kp, vp, plan, dev_err=err, stream=stream)
    return out, dict(cl=cl, plan=plan, dev_err=err)


# --------------------------------------------------------------------------- static stripe mask

PSA_INF = 2 ** 31 - 1   # SVOO_PSA_INF: infinite stride, one diagonal band on that axis


def psa_params(per_head, device) -> torch.Tensor:
    """int32 [B*H, 6] device tensor from per-head (Tw, To, Ts, Sw, So, Ss) tuples;
    None or math.inf for an infinite stride."""
    rows = []
    for prm in per_head:
        if len(prm) != 6:
            raise SvooError("a PSA mask has six parameters (Tw, To, Ts, Sw, So, Ss)")
        rows.append([PSA_INF if (i in (2, 5) and (v is None or v == math.inf)) else int(v)
                     for i, v in enumerate(prm)])
    return torch.tensor(rows, dtype=torch.int32).to(device)


def psa_config(grid, block, block_q: int = 128, scale: Optional[float] = None) -> Config:
    """The Config of a stripe-mask plan: one group per PSABlock on each side."""
    nb = load().svoo_psa_block_count(*grid, *block)
    if nb < 1 or nb > 256:
        raise SvooError(f"PSABlock grid of {grid} by {block} has {nb} blocks (1..256 supported)")
    return Config(n_qc=nb, n_kc=nb, iters=1, block_q=block_q, scale=scale)


def psa_mask(shape: Shape, grid, block, params: torch.Tensor, cfg: Config,
             plan: Optional[Plan] = None, k_assign: Optional[torch.Tensor] = None, dev_err=None,
             stream=None):
    """Plan of the PSA stripe mask (svoo_psa_mask): returns (plan, k_assign)."""
    _need_cuda(params)
    dev = params.device
    BH, nv = shape.B * shape.H, shape.N - shape.n_text
    if tuple(params.shape) != (BH, 6) or params.dtype != torch.int32 or not params.is_contiguous():
        raise SvooError("params must be a contiguous int32 [B*H, 6] tensor")
    if plan is None:
        plan = Plan(shape, cfg, dev)
    if k_assign is None:
        k_assign = torch.empty(BH, nv, dtype=torch.int32, device=dev)
    err = _err_buf(dev_err, dev)
    _check(load().svoo_psa_mask(ctypes.byref(shape), *grid, *block, _ptr(params), cfg.block_q, plan.c,
                                _ptr(k_assign), _ptr(err), _stream(stream)), "svoo_psa_mask")
    return plan, k_assign


def psa_attention(q, k, v, grid, block, params: torch.Tensor, n_text=0, block_q: int = 128,
                  scale: Optional[float] = None, dev_err=None, stream=None):
    """The stripe-mask path: PSA plan -> permute -> sparse attention."""
    sh = make_shape(q, n_text)
    cfg = psa_config(grid, block, block_q, scale)
    err = _err_buf(dev_err, q.device)
    plan, k_assign = psa_mask(sh, grid, block, params, cfg, dev_err=err, stream=stream)
    qp, kp, vp = permute(q, k, v, k_assign, plan, dev_err=err, stream=stream)
    out = sparse_attn(qp, kp, vp, plan, dev_err=err, stream=stream)
    return out, dict(plan=plan, k_assign=k_assign, dev_err=err, cfg=cfg)


# --------------------------------------------------------------------------- SNR-guided top-p


def snr_top_p(steps: int, warmup: int = 0, p_min: float = 0.7, tau: float = 0.999,
              shift: float = 1.0):
    """Top-p of each of `steps` denoising calls (svoo_snr_top_p), as a float32
    numpy array; feed p[t] to build_mask with Config(select_mode=1)."""
    import numpy as np
    p = np.empty(int(steps), dtype=np.float32)
    _check(load().svoo_snr_top_p(int(steps), int(warmup), float(p_min), float(tau), float(shift),
                                 p.ctypes.data_as(ctypes.c_void_p)), "svoo_snr_top_p")
    return p
