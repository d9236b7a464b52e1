"""svoo_cluster_step_static: the clustering half-step for callers that may not
allocate device memory (a host framework that owns every device allocation
through its own pool, or a loop that forbids allocation after start-up). Its
scratch is a fixed array inside the library instead of a caller workspace.

The test calls it through the C ABI twice in a row (a query step in feature
space, then a key step under the query clusters' metric, so the second call
runs on scratch the first one left behind) and checks each result against the
workspace-based svoo_cluster_step on the same inputs: the same labels and
sizes, and centroids within twice the bound each call keeps from the exact
means (the fp32 member sums are added atomically, in no fixed order). It also
checks that a shape needing more than the fixed scratch is refused before any
launch.
This file sorts last so that a run stopping at its first failure has already
run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import workload
from workload import bf16_bits_to_f32
import free_sparse_attention_head_b200 as svoo
from free_sparse_attention_head_b200 import build as svoo_build

pytestmark = pytest.mark.gpu


def _dev_bf16(a, B, H):
    BH, N, d = a.shape
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16).view(B, H, N, d)


def _token_start(x, C):
    """Centroid j = token floor(j n / C), widened to fp32 (the library's cold start)."""
    BH, n, d = x.shape
    idx = [j * n // C for j in range(C)]
    f = (x[:, idx, :].astype(np.uint32) << 16).view(np.float32)
    return np.ascontiguousarray(f)


def _step_both(xd, cent0, metric=None):
    """Runs the workspace entry point and the static one on the same inputs."""
    outs = []
    for fn in (svoo.cluster_step, svoo.cluster_step_static):
        BH, C, _ = cent0.shape
        nv = xd.shape[2]
        cent = torch.from_numpy(cent0.copy()).cuda()
        sizes = torch.zeros(BH, C, dtype=torch.int32, device="cuda")
        assign = torch.full((BH, nv), -1, dtype=torch.int32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        mc, ms = (None, None) if metric is None else (metric[0], metric[1])
        fn(xd, cent, sizes, assign, metric_cent=mc, metric_sizes=ms, dev_err=err)
        torch.cuda.synchronize()
        svoo.check_device_errors(err)
        outs.append((assign, cent, sizes))
    return outs


def _same_means(c_a, c_b, x, labels):
    """Both centroid sets round the exact member means (the sums are exact),
    so they agree; the check allows the looser bound of fp32 sums,
    (n + 18) 2^-24 mean|x| + 2^-24 + 1 ulp from each, twice over."""
    a, b = c_a.cpu().numpy().astype(np.float64), c_b.cpu().numpy().astype(np.float64)
    lab = labels.cpu().numpy()
    xf = np.abs(bf16_bits_to_f32(x).astype(np.float64))
    for h in range(a.shape[0]):
        C = a.shape[1]
        n = np.bincount(lab[h], minlength=C)
        absum = np.zeros(a[h].shape)
        np.add.at(absum, lab[h], xf[h][: lab.shape[1]])
        mean_abs = absum / np.maximum(n, 1)[:, None]
        tol = 2 * ((n[:, None] + 18) * 2.0 ** -24 * mean_abs + 2.0 ** -24 +
                   np.spacing(np.abs(a[h]).astype(np.float32)).astype(np.float64))
        assert (np.abs(a[h] - b[h]) <= tol).all()


def test_static_scratch_step_matches_workspace_step():
    svoo_build.build()
    svoo.load()
    w = workload.get("wan2.1-1.3b")
    import dataclasses
    w = dataclasses.replace(w, H=2)
    q, k, _ = workload.make_qkv(w)
    qd, kd = _dev_bf16(q, w.B, w.H), _dev_bf16(k, w.B, w.H)
    # call 1: query step, feature space
    (a_ws, c_ws, s_ws), (a_st, c_st, s_st) = _step_both(qd, _token_start(q, w.n_qc))
    assert torch.equal(a_ws, a_st)
    assert torch.equal(s_ws, s_st)
    _same_means(c_ws, c_st, q, a_st)
    assert int(s_st.sum()) == w.B * w.H * w.n_video
    # call 2 (scratch still holds call 1's contents): key step under the query metric
    (b_ws, d_ws, t_ws), (b_st, d_st, t_st) = _step_both(kd, _token_start(k, w.n_kc), metric=(c_st, s_st))
    assert torch.equal(b_ws, b_st)
    assert torch.equal(t_ws, t_st)
    _same_means(d_ws, d_st, k, b_st)


def test_static_scratch_rejects_oversized_shape():
    lib = svoo.load()
    sh = svoo.Shape(1, 40, 75600, 128, 0)  # needs ~29 MB of scratch > 16 MiB
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: refused before any launch
    st = lib.svoo_cluster_step_static(ctypes.byref(sh), fake, 256, fake, fake, fake, None, None, 0,
                                      None, None)
    assert st == 2 and lib.svoo_status_string(st) == b"workspace too small"


def test_static_scratch_ignores_metric_count_without_metric():
    """With no metric (identity), metric_C plays no part: 32 heads, d = 128 and
    128 clusters fit the fixed scratch while 256 would not, so a leftover
    metric_C = 256 beside a NULL metric must neither be refused nor change the
    result (same labels and sizes as the workspace entry point)."""
    svoo_build.build()
    lib = svoo.load()
    B, H, N, d, C = 1, 32, 1024, 128, 128
    rng = np.random.Generator(np.random.PCG64(5))
    x = workload.f32_to_bf16_bits(rng.standard_normal((B * H, N, d), dtype=np.float32))
    xd = _dev_bf16(x, B, H)
    c0 = _token_start(x, C)
    res = []
    for static in (False, True):
        cent = torch.from_numpy(c0.copy()).cuda()
        sizes = torch.zeros(B * H, C, dtype=torch.int32, device="cuda")
        assign = torch.full((B * H, N), -1, dtype=torch.int32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        sh = svoo.Shape(B, H, N, d, 0)
        P = lambda t: ctypes.c_void_p(t.data_ptr())
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        if static:
            st = lib.svoo_cluster_step_static(ctypes.byref(sh), P(xd), C, P(cent), P(sizes), P(assign),
                                              None, None, 256, P(err), stream)
        else:
            ws_bytes = lib.svoo_cluster_workspace_size(ctypes.byref(sh), C, C)
            ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
            st = lib.svoo_cluster_step(ctypes.byref(sh), P(xd), C, P(cent), P(sizes), P(assign), None,
                                       None, 256, P(ws), ws_bytes, P(err), stream)
        assert st == 0, lib.svoo_status_string(st)
        torch.cuda.synchronize()
        svoo.check_device_errors(err)
        res.append((assign, sizes))
    assert torch.equal(res[0][0], res[1][0])
    assert torch.equal(res[0][1], res[1][1])
    assert int(res[1][1].sum()) == B * H * N
