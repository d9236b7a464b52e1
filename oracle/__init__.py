"""CPU oracle of the online QK co-clustered block-sparse attention path.

TEST INFRASTRUCTURE ONLY. Only `tests/`, `__graft_entry__.smoke()` and the
benchmark's CPU-baseline leg may import this package. The CUDA library never
imports it and shares no code with it; the two meet only through the seeded
inputs of the `workload` package.

The arithmetic lives in `svoo_oracle.c` (plain single-threaded C, fp64 unless a
function states otherwise). This module compiles it on first use and wraps it
with numpy marshalling, looping over (batch, head).

Parity pins: every function here is pinned by `tests/test_oracle_pins.py`
against closed forms, brute force and invariants (see that file's docstrings).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "svoo_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile svoo_oracle.c into oracle/liboracle.so (gcc, no fast-math, no contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < max(
            os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "svoo_oracle.h"))):
        cc = os.environ.get("CC", "gcc")
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call([cc, *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float

_SIGS = {
    "oracle_version": (_I, []),
    "oracle_exp": (_F, [_F]),
    "oracle_metric": (None, [_P, _P, _I, _I, _I, _P]),
    "oracle_init_centroids": (None, [_P, _I, _I, _I, _P]),
    "oracle_assign": (None, [_P, _I, _I, _P, _I, _P, _P, _P, _P]),
    "oracle_update": (None, [_P, _I, _I, _P, _I, _P, _P, _P]),
    "oracle_cluster": (None, [_P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "oracle_pair_mass": (None, [_P, _P, _P, _P, _I, _I, _I, _F, _P, _P]),
    "oracle_select": (_I, [_P, _P, _I, _I, _I, _F, _F, _I, _P, _I]),
    "oracle_tail_merge": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "oracle_permute": (None, [_P, _I, _I, _P, _P]),
    "oracle_tiles": (_I, [_P, _I, _I, _P]),
    "oracle_attn_rows": (None, [_P, _P, _P, _I, _I, _F, _P, _P, _P, _I, _P, _I, _P, _P, _P]),
    "oracle_dense_attn_rows": (None, [_P, _P, _P, _I, _I, _F, _P, _I, _P]),
    "oracle_psa_attends": (_I, [ctypes.c_longlong, ctypes.c_longlong, ctypes.c_longlong, _P]),
    "oracle_psa_plan": (_I, [_I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P]),
    "oracle_snr_top_p": (_I, [_I, _I, ctypes.c_double, ctypes.c_double, ctypes.c_double, _P]),
}


def lib():
    global _lib
    if _lib is None:
        path = build()
        L = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def mask_words(n_kc: int, has_text: bool) -> int:
    return (n_kc + (1 if has_text else 0) + 63) // 64


# --------------------------------------------------------------------------- per-head wrappers

def exp(x: float) -> float:
    return lib().oracle_exp(float(x))


def metric(cent, sizes, identity=False):
    cent = _c(cent, np.float32)
    sizes = _c(sizes, np.int32)
    C, d = cent.shape
    M = np.empty((d, d), dtype=np.float64)
    lib().oracle_metric(_p(cent), _p(sizes), C, d, int(bool(identity)), _p(M))
    return M


def init_centroids(x, C):
    x = _c(x, np.uint16)
    n, d = x.shape
    cent = np.empty((C, d), dtype=np.float32)
    lib().oracle_init_centroids(_p(x), n, d, C, _p(cent))
    return cent


def assign(x, cent, M, with_dist=False):
    x = _c(x, np.uint16)
    cent = _c(cent, np.float32)
    M = _c(M, np.float64)
    n, d = x.shape
    C = cent.shape[0]
    a = np.empty(n, dtype=np.int32)
    b1 = np.empty(n, dtype=np.float64) if with_dist else None
    b2 = np.empty(n, dtype=np.float64) if with_dist else None
    lib().oracle_assign(_p(x), n, d, _p(cent), C, _p(M), _p(a), _p(b1), _p(b2))
    return (a, b1, b2) if with_dist else a


def update(x, labels, cent_old):
    x = _c(x, np.uint16)
    labels = _c(labels, np.int32)
    cent_old = _c(cent_old, np.float32)
    n, d = x.shape
    C = cent_old.shape[0]
    cent = np.empty((C, d), dtype=np.float32)
    sizes = np.empty(C, dtype=np.int32)
    lib().oracle_update(_p(x), n, d, _p(labels), C, _p(cent_old), _p(cent), _p(sizes))
    return cent, sizes


def cluster(q, k, n_qc, n_kc, iters, warm=None, identity=False):
    """One head. warm = (q_cent, k_cent, k_sizes) start state, or None;
    identity = True clusters queries and keys independently (M = I in every
    step)."""
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    n, d = q.shape
    qa = np.empty(n, dtype=np.int32)
    ka = np.empty(n, dtype=np.int32)
    qs = np.zeros(n_qc, dtype=np.int32)
    ks = np.zeros(n_kc, dtype=np.int32)
    if warm is None:
        qc = np.empty((n_qc, d), dtype=np.float32)
        kc = np.empty((n_kc, d), dtype=np.float32)
    else:
        qc = np.array(warm[0], dtype=np.float32, copy=True)
        kc = np.array(warm[1], dtype=np.float32, copy=True)
        ks[:] = warm[2]
    flags = int(warm is not None) | (2 if identity else 0)
    lib().oracle_cluster(_p(q), _p(k), n, d, n_qc, n_kc, iters, flags,
                         _p(qa), _p(ka), _p(qc), _p(kc), _p(qs), _p(ks))
    return dict(q_assign=qa, k_assign=ka, q_cent=qc, k_cent=kc, q_sizes=qs, k_sizes=ks)


def pair_mass(q_cent, k_cent, q_sizes, k_sizes, scale):
    q_cent = _c(q_cent, np.float32)
    k_cent = _c(k_cent, np.float32)
    q_sizes = _c(q_sizes, np.int32)
    k_sizes = _c(k_sizes, np.int32)
    Cq, d = q_cent.shape
    Ck = k_cent.shape[0]
    w = np.empty((Cq, Ck), dtype=np.float32)
    top1 = np.empty(Cq, dtype=np.int32)
    lib().oracle_pair_mass(_p(q_cent), _p(k_cent), _p(q_sizes), _p(k_sizes), Cq, Ck, d,
                           float(np.float32(scale)), _p(w), _p(top1))
    return w, top1


def select(w, top1, keep=0.0, mode=0, top_p=0.0, has_text=False):
    w = _c(w, np.float32)
    top1 = _c(top1, np.int32)
    Cq, Ck = w.shape
    W = mask_words(Ck, has_text)
    km = np.empty((Cq + (1 if has_text else 0), W), dtype=np.uint64)
    L = lib().oracle_select(_p(w), _p(top1), Cq, Ck, int(mode), float(keep), float(top_p),
                            int(bool(has_text)), _p(km), W)
    return km, L


def tail_merge(kmask, sizes, labels, block_q, rounds=2):
    """Returns (kmask', sizes', labels', nonempty, stats); inputs are not modified."""
    km = np.array(kmask, dtype=np.uint64, copy=True, order="C")
    sz = np.array(sizes, dtype=np.int32, copy=True)
    lb = np.array(labels, dtype=np.int32, copy=True)
    Cq = sz.shape[0]
    W = km.shape[1]
    st = np.zeros(6, dtype=np.int32)
    ne = lib().oracle_tail_merge(_p(km), _p(sz), _p(lb), lb.shape[0], Cq, W, int(block_q),
                                 int(rounds), _p(st))
    return km, sz, lb, ne, st


def permute(labels, G):
    labels = _c(labels, np.int32)
    n = labels.shape[0]
    perm = np.empty(n, dtype=np.int32)
    off = np.empty(G + 1, dtype=np.int32)
    lib().oracle_permute(_p(labels), n, G, _p(perm), _p(off))
    return perm, off


def tiles(off, block_q):
    off = _c(off, np.int32)
    G = off.shape[0] - 1
    cap = int(sum((int(off[g + 1] - off[g]) + block_q - 1) // block_q for g in range(G)))
    t = np.empty((max(cap, 1), 3), dtype=np.int32)
    c = lib().oracle_tiles(_p(off), G, int(block_q), _p(t))
    return t[:c]


def attn_rows(q, k, v, scale, q_label, k_label, kmask, rows):
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    q_label = _c(q_label, np.int32)
    k_label = _c(k_label, np.int32)
    kmask = _c(kmask, np.uint64)
    rows = _c(rows, np.int32)
    n, d = q.shape
    out = np.empty((rows.shape[0], d), dtype=np.float64)
    ps = np.empty(rows.shape[0], dtype=np.float64)
    nk = np.empty(rows.shape[0], dtype=np.int64)
    lib().oracle_attn_rows(_p(q), _p(k), _p(v), n, d, float(np.float32(scale)), _p(q_label),
                           _p(k_label), _p(kmask), kmask.shape[1], _p(rows), rows.shape[0],
                           _p(out), _p(ps), _p(nk))
    return out, ps, nk


def dense_attn_rows(q, k, v, scale, rows):
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    rows = _c(rows, np.int32)
    n, d = q.shape
    out = np.empty((rows.shape[0], d), dtype=np.float64)
    lib().oracle_dense_attn_rows(_p(q), _p(k), _p(v), n, d, float(np.float32(scale)), _p(rows),
                                 rows.shape[0], _p(out))
    return out


# --------------------------------------------------------------------------- whole path, one head

def plan_head(q, k, n_qc, n_kc, iters, keep, block_q, n_text=0, mode=0, top_p=0.0, scale=None,
              rounds=2, clusters=None):
    """Oracle of clustering -> mask -> tail merge -> permutation for one head.

    q, k: uint16 [N, d] including n_text trailing text tokens. `clusters` may
    carry a precomputed result of `cluster` (it is then not recomputed).
    """
    N, d = q.shape
    nv = N - n_text
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    cl = clusters if clusters is not None else cluster(q[:nv], k[:nv], n_qc, n_kc, iters)
    w, top1 = pair_mass(cl["q_cent"], cl["k_cent"], cl["q_sizes"], cl["k_sizes"], scale)
    km0, L = select(w, top1, keep=keep, mode=mode, top_p=top_p, has_text=n_text > 0)
    km, sz, lb, ne, st = tail_merge(km0, cl["q_sizes"], cl["q_assign"], block_q, rounds)
    has_text = n_text > 0
    q_label = np.concatenate([lb, np.full(n_text, n_qc, dtype=np.int32)])
    k_label = np.concatenate([cl["k_assign"], np.full(n_text, n_kc, dtype=np.int32)])
    Gq, Gk = n_qc + has_text, n_kc + has_text
    q_perm, q_off = permute(q_label, Gq)
    k_perm, k_off = permute(k_label, Gk)
    return dict(cl=cl, w=w, top1=top1, kmask_pre=km0, kept=L, kmask=km, q_sizes_merged=sz,
                q_label=q_label, k_label=k_label, nonempty=ne, merge_stats=st,
                q_perm=q_perm, q_off=q_off, k_perm=k_perm, k_off=k_off,
                tiles=tiles(q_off, block_q), scale=float(np.float32(scale)))


# --------------------------------------------------------------------------- PSA stripe mask

PSA_INF = 2 ** 31 - 1   # stride "infinity": one diagonal band, no wrap-around


def psa_params(prm):
    """(Tw, To, Ts, Sw, So, Ss) with None or math.inf for an infinite stride -> int32[6]."""
    out = []
    for i, v in enumerate(prm):
        if i in (2, 5) and (v is None or v == math.inf):
            v = PSA_INF
        out.append(int(v))
    return np.array(out, dtype=np.int32)


def psa_attends(i, j, HW, prm):
    return bool(lib().oracle_psa_attends(int(i), int(j), int(HW), _p(psa_params(prm))))


def psa_plan(T, H, W, block, n_text, prm):
    """Labels [N], block mask [G, Wd] and block sizes [G] of one head."""
    bt, bh, bw = block
    nb = -(-T // bt) * -(-H // bh) * -(-W // bw)
    G = nb + (1 if n_text > 0 else 0)
    Wd = (G + 63) // 64
    N = T * H * W + n_text
    label = np.empty(N, dtype=np.int32)
    kmask = np.empty((G, Wd), dtype=np.uint64)
    sizes = np.empty(G, dtype=np.int32)
    r = lib().oracle_psa_plan(T, H, W, bt, bh, bw, n_text, _p(psa_params(prm)), _p(label),
                              _p(kmask), _p(sizes))
    assert r == nb
    return dict(label=label, kmask=kmask, sizes=sizes, nb=nb, G=G)


def psa_plan_head(T, H, W, block, n_text, prm, block_q):
    """Oracle of the static stripe-mask path for one head: the PSA plan, then
    the same permutation and query tiles as the clustered path."""
    p = psa_plan(T, H, W, block, n_text, prm)
    q_perm, q_off = permute(p["label"], p["G"])
    return dict(kmask=p["kmask"], q_label=p["label"], k_label=p["label"], q_sizes=p["sizes"],
                nb=p["nb"], q_perm=q_perm, q_off=q_off, k_perm=q_perm, k_off=q_off,
                tiles=tiles(q_off, block_q))


# --------------------------------------------------------------------------- SNR-guided top-p

def snr_top_p(steps, warmup=0, p_min=0.7, tau=0.999, shift=1.0):
    """Top-p of each of `steps` denoising calls (fp32 [steps]); see oracle_snr_top_p."""
    p = np.empty(steps, dtype=np.float32)
    if lib().oracle_snr_top_p(int(steps), int(warmup), float(p_min), float(tau), float(shift), _p(p)) != 0:
        raise ValueError("bad SNR schedule arguments")
    return p
