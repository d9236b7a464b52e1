"""The C-ABI library: it builds, loads without a GPU, exports every entry point
that include/svoo.h declares, and rejects bad arguments on the host before any
launch (these calls never reach the device)."""
import ctypes
import os
import re

import pytest

import free_sparse_attention_head_b200 as svoo
from free_sparse_attention_head_b200 import build as svoo_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "svoo.h")


@pytest.fixture(scope="module")
def lib():
    svoo_build.build()
    return svoo.load()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(svoo_[a-z_]+)\s*\(", text)))


def test_header_declares_expected_entry_points():
    names = _declared()
    for n in ("svoo_cluster", "svoo_build_mask", "svoo_permute", "svoo_sparse_attn"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = os.popen(f"nm -D --defined-only {svoo.lib_path()}").read()
    exported = set(re.findall(r"\bT (svoo_\w+)", out))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    assert set(svoo.EXPORTS) <= exported


def test_cluster_flag_values_match_header():
    text = open(HEADER).read()
    macros = dict(re.findall(r"#define (SVOO_CLUSTER_\w+) (\d+)", text))
    assert int(macros["SVOO_CLUSTER_WARM"]) == svoo.CLUSTER_WARM
    assert int(macros["SVOO_CLUSTER_IDENTITY"]) == svoo.CLUSTER_IDENTITY
    assert svoo._cluster_flags(svoo.Config(metric=1), None) == svoo.CLUSTER_IDENTITY
    assert svoo._cluster_flags(svoo.Config(), (0, 0, 0)) == svoo.CLUSTER_WARM
    with pytest.raises(svoo.SvooError):
        svoo._cluster_flags(svoo.Config(metric=2), None)


def test_status_strings_and_version(lib):
    assert lib.svoo_status_string(0) == b"ok"
    assert lib.svoo_status_string(2) == b"workspace too small"
    assert lib.svoo_version() >= 1


def _shape(B=1, H=2, N=1024, d=64, n_text=0):
    return svoo.Shape(B, H, N, d, n_text)


def test_plan_counts(lib):
    sh = _shape(N=1000, d=128, n_text=24)
    counts = (ctypes.c_int64 * 12)()
    assert lib.svoo_plan_counts(ctypes.byref(sh), 16, 70, 64, counts) == 0
    Gq, Gk = 17, 71
    W = (Gk + 63) // 64
    cap = (1000 + 63) // 64 + Gq
    ucap = (1000 + 255) // 256 + Gq
    assert list(counts) == [2 * Gq * W, 2000, 2 * Gq, 16, 2000, 2 * (Gq + 1), 2000, 2 * (Gk + 1),
                            2 * cap * 4, 2, 2 * ucap * 4, 2]


@pytest.mark.parametrize("bad", [
    dict(d=96), dict(N=0), dict(B=0), dict(n_text=-1), dict(N=10, n_text=10),
    dict(B=70000, H=1), dict(H=65536),
])
def test_bad_shapes_rejected(lib, bad):
    sh = _shape(**bad)
    counts = (ctypes.c_int64 * 12)()
    assert lib.svoo_plan_counts(ctypes.byref(sh), 16, 16, 64, counts) == 1
    assert lib.svoo_cluster_workspace_size(ctypes.byref(sh), 16, 16) == 0


def test_compute_entry_points_validate_before_launch(lib):
    sh = _shape()
    P = ctypes.c_void_p
    fake = P(0x1000)   # never dereferenced: validation fails first
    odd = P(0x1001)    # misaligned
    ws = lib.svoo_cluster_workspace_size(ctypes.byref(sh), 16, 16)
    assert ws > 0
    # null inputs
    assert lib.svoo_cluster(ctypes.byref(sh), None, fake, 16, 16, 10, 0, fake, fake, fake, fake, fake,
                            fake, fake, ws, None, None) == 1
    # cluster counts out of range, iters < 1, unknown flag bits
    for nq, nk, it, flags in [(0, 16, 10, 0), (16, 300, 10, 0), (16, 16, 0, 0), (16, 16, 1, 4),
                              (16, 16, 1, -1), (16, 16, 1, 3 | 8)]:
        assert lib.svoo_cluster(ctypes.byref(sh), fake, fake, nq, nk, it, flags, fake, fake, fake, fake,
                                fake, fake, fake, ws, None, None) == 1
    # misaligned q
    assert lib.svoo_cluster(ctypes.byref(sh), odd, fake, 16, 16, 10, 0, fake, fake, fake, fake, fake,
                            fake, fake, ws, None, None) == 1
    # workspace too small
    assert lib.svoo_cluster(ctypes.byref(sh), fake, fake, 16, 16, 10, 0, fake, fake, fake, fake, fake,
                            fake, fake, ws - 1024, None, None) == 2
    plan = svoo._CPlan(*([0x1000] * 12))
    mws = lib.svoo_mask_workspace_size(ctypes.byref(sh), 16, 16)
    args = [ctypes.byref(sh), fake, fake, fake, fake, fake, fake, 16, 16]
    assert lib.svoo_build_mask(*args, 2, 64, 2, 0.125, ctypes.byref(plan), fake, mws, None, None) == 1
    assert lib.svoo_build_mask(*args, 0, 96, 2, 0.125, ctypes.byref(plan), fake, mws, None, None) == 1
    assert lib.svoo_build_mask(*args, 0, 64, 2, -1.0, ctypes.byref(plan), fake, mws, None, None) == 1
    assert lib.svoo_build_mask(*args, 0, 64, 2, 0.125, ctypes.byref(plan), fake, 8, None, None) == 2
    assert lib.svoo_permute(ctypes.byref(sh), fake, fake, fake, fake, 16, 16, 64, ctypes.byref(plan),
                            odd, fake, fake, None, None) == 1
    assert lib.svoo_sparse_attn(ctypes.byref(sh), fake, fake, fake, ctypes.byref(plan), 16, 16, 64,
                                float("nan"), fake, None, None) == 1
    assert lib.svoo_sparse_attn(ctypes.byref(sh), fake, fake, fake, None, 16, 16, 64, 0.125, fake,
                                None, None) == 1


def test_psa_block_count_and_mask_validation(lib):
    assert lib.svoo_psa_block_count(21, 45, 80, 3, 8, 16) == 7 * 6 * 5
    assert lib.svoo_psa_block_count(6, 10, 12, 2, 4, 5) == 27
    assert lib.svoo_psa_block_count(0, 10, 12, 2, 4, 5) == 0
    assert lib.svoo_psa_block_count(6, 10, 12, 2, 0, 5) == 0
    sh = _shape(B=1, H=2, N=6 * 10 * 12 + 4, d=128, n_text=4)
    P = ctypes.c_void_p
    fake = P(0x1000)
    plan = svoo._CPlan(*([0x1000] * 12))
    ok = (6, 10, 12, 2, 4, 5)
    args = lambda grid_block, params=fake, bq=128, pl=ctypes.byref(plan), ka=fake: (
        ctypes.byref(sh), *grid_block, params, bq, pl, ka, None, None)
    # grid does not cover the video tokens, too many blocks, bad block, block_q, nulls
    for gb in [(6, 10, 11, 2, 4, 5), (6, 10, 12, 1, 1, 1), (6, 10, 12, 0, 4, 5)]:
        assert lib.svoo_psa_mask(*args(gb)) == 1, gb
    assert lib.svoo_psa_mask(*args(ok, bq=96)) == 1
    assert lib.svoo_psa_mask(*args(ok, params=None)) == 1
    assert lib.svoo_psa_mask(*args(ok, ka=None)) == 1
    assert lib.svoo_psa_mask(*args(ok, pl=None)) == 1
    empty = svoo._CPlan(*([0] * 12))
    assert lib.svoo_psa_mask(*args(ok, pl=ctypes.byref(empty))) == 1


@pytest.mark.parametrize("args", [(50, 0, 0.7, 0.999, 1.0), (50, 5, 0.7, 0.999, 5.0),
                                  (30, 2, 0.5, 0.95, 3.0), (7, 0, 0.8, 0.8, 1.0)])
def test_snr_top_p_schedule_matches_oracle(lib, args):
    """svoo_snr_top_p is host code (no device work): the library's schedule
    equals the oracle's, written separately from the same reading of iCATS
    section 4.2, to one fp32 rounding."""
    import numpy as np
    import oracle
    got = svoo.snr_top_p(*args).astype(np.float64)
    want = oracle.snr_top_p(*args).astype(np.float64)
    assert np.all(np.abs(got - want) <= np.spacing(np.float32(1.0)))


def test_snr_top_p_rejects_bad_arguments(lib):
    for bad in [(0, 0, 0.7, 0.9, 1.0), (10, -1, 0.7, 0.9, 1.0), (10, 0, 0.9, 0.7, 1.0),
                (10, 0, 0.7, 1.5, 1.0), (10, 0, 0.7, 0.9, -2.0)]:
        with pytest.raises(svoo.SvooError):
            svoo.snr_top_p(*bad)
    assert lib.svoo_snr_top_p(5, 0, 0.7, 0.9, 1.0, None) == 1


def test_stall_library_exports_every_declared_symbol(lib):
    """The test-only build (SVOO_TEST_STALL) links with the same entry points."""
    out = os.popen(f"nm -D --defined-only {svoo_build.STALL_LIB}").read()
    exported = set(re.findall(r"\bT (svoo_\w+)", out))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
