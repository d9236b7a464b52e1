"""Pins of the oracle's static stripe mask (PSA sec. 3.2, Algorithm 1, masking
at PSABlock granularity) against what the pages and arithmetic fix: the SVG
special case is a plain band, the full window is dense attention, a finite
stride repeats with a closed-form count, an offset moves the diagonal, the
mirror symmetry of |.|, and the PSABlock-centric layout
(T', H', W', bt, bh, bw) of the permutation."""
import math

import numpy as np
import pytest

import oracle
from workload import f32_to_bf16_bits

INF = math.inf


def _coords(T, H, W, block):
    """Block (frame, in-frame) coordinates of every block in raster order."""
    bt, bh, bw = block
    Tb, Hb, Wb = -(-T // bt), -(-H // bh), -(-W // bw)
    a = np.arange(Tb * Hb * Wb)
    return a // (Hb * Wb), a % (Hb * Wb), (Tb, Hb, Wb)


def _bits(kmask, G):
    words = kmask[:, np.arange(G) // 64]
    return ((words >> (np.arange(G) % 64).astype(np.uint64)) & np.uint64(1)).astype(bool)


GRID = (6, 10, 12)       # T, H, W with ragged edge blocks below
BLOCK = (2, 4, 5)        # -> T' = 3, H' = 3, W' = 3: 27 blocks


@pytest.mark.parametrize("Tw,Sw", [(1, 1), (2, 3), (3, 9), (1, 4)])
def test_svg_special_case_is_a_band(Tw, Sw):
    """M(Tw, 0, inf, Sw, 0, inf) (SVG's pattern) keeps exactly the block pairs
    with |frame distance| < Tw and |in-frame distance| < Sw."""
    p = oracle.psa_plan(*GRID, BLOCK, 0, (Tw, 0, INF, Sw, 0, INF))
    t, s, _ = _coords(*GRID, BLOCK)
    want = (np.abs(t[None] - t[:, None]) < Tw) & (np.abs(s[None] - s[:, None]) < Sw)
    assert np.array_equal(_bits(p["kmask"], p["G"]), want)


def test_sta_special_case_repeats_along_the_frame():
    """M(Tw, 0, inf, Sw, 0, Ss) (STA's window): in-frame distance taken mod Ss."""
    Tw, Sw, Ss = 2, 1, 3
    p = oracle.psa_plan(*GRID, BLOCK, 0, (Tw, 0, INF, Sw, 0, Ss))
    t, s, _ = _coords(*GRID, BLOCK)
    ds = np.abs(s[None] - s[:, None])
    want = (np.abs(t[None] - t[:, None]) < Tw) & (ds % Ss == 0)
    assert np.array_equal(_bits(p["kmask"], p["G"]), want)


def test_full_window_is_dense_attention():
    rng = np.random.default_rng(21)
    T, H, W, d = 4, 6, 5, 16
    n = T * H * W
    q, k, v = (f32_to_bf16_bits(rng.standard_normal((n, d)).astype(np.float32)) for _ in range(3))
    block = (2, 3, 2)
    _, _, (Tb, Hb, Wb) = _coords(T, H, W, block)
    p = oracle.psa_plan(T, H, W, block, 0, (Tb, 0, INF, Hb * Wb, 0, INF))
    assert _bits(p["kmask"], p["G"]).all()
    rows = np.arange(0, n, 7, dtype=np.int32)
    out, ps, nk = oracle.attn_rows(q, k, v, 0.25, p["label"], p["label"], p["kmask"], rows)
    dense = oracle.dense_attn_rows(q, k, v, 0.25, rows)
    assert np.allclose(out, dense, rtol=0, atol=1e-12)
    assert (nk == n).all()


@pytest.mark.parametrize("Tw,Ts", [(1, 2), (2, 3), (1, 4), (3, 3), (4, 3)])
def test_finite_stride_count(Tw, Ts):
    """One spatial block per frame and To = 0: the first block row keeps the
    frame distances D in [0, T') with D mod Ts < Tw, i.e.
    floor(T'/Ts) min(Tw, Ts) + min(T' mod Ts, Tw) blocks; Tw >= Ts keeps all."""
    T = 11
    p = oracle.psa_plan(T, 1, 1, (1, 1, 1), 0, (Tw, 0, Ts, 1, 0, INF))
    row0 = _bits(p["kmask"], p["G"])[0]
    assert row0.sum() == (T // Ts) * min(Tw, Ts) + min(T % Ts, Tw)
    D = np.arange(T)
    assert np.array_equal(row0, D % Ts < Tw)
    if Tw >= Ts:
        assert row0.all()


@pytest.mark.parametrize("To", [-2, -1, 1, 2])
def test_offset_moves_the_diagonal(To):
    """Tw = 1, infinite stride: only frame distance exactly To is kept; with a
    full in-frame window every spatial block of that frame is kept."""
    T, H, W, block = 7, 4, 4, (1, 2, 2)
    t, s, (Tb, Hb, Wb) = _coords(T, H, W, block)
    p = oracle.psa_plan(T, H, W, block, 0, (1, To, INF, Hb * Wb, 0, INF))
    want = (t[None] - t[:, None]) == To
    assert np.array_equal(_bits(p["kmask"], p["G"]), want)


def test_mirror_symmetry():
    """|D - o| = |(-D) - (-o)|: the mask under offsets (To, So) is the transpose
    of the mask under (-To, -So) (strides infinite); with zero offsets it is
    symmetric."""
    prm = (2, 1, INF, 3, -1, INF)
    neg = (2, -1, INF, 3, 1, INF)
    a = _bits(oracle.psa_plan(*GRID, BLOCK, 0, prm)["kmask"], 27)
    b = _bits(oracle.psa_plan(*GRID, BLOCK, 0, neg)["kmask"], 27)
    assert np.array_equal(a, b.T)
    z = _bits(oracle.psa_plan(*GRID, BLOCK, 0, (2, 0, 2, 4, 0, 5))["kmask"], 27)
    assert np.array_equal(z, z.T)


def test_labels_sizes_and_block_centric_layout():
    """The stable sort by block label is the PSABlock-centric layout: pad the
    (T, H, W) index grid to whole blocks, view it as (T', bt, H', bh, W', bw),
    move to (T', H', W', bt, bh, bw) and drop the padding."""
    T, H, W = GRID
    bt, bh, bw = BLOCK
    n_text = 5
    res = oracle.psa_plan_head(T, H, W, BLOCK, n_text, (1, 0, INF, 1, 0, INF), 128)
    _, _, (Tb, Hb, Wb) = _coords(T, H, W, BLOCK)
    grid = np.full((Tb * bt, Hb * bh, Wb * bw), -1, dtype=np.int64)
    grid[:T, :H, :W] = np.arange(T * H * W).reshape(T, H, W)
    lay = grid.reshape(Tb, bt, Hb, bh, Wb, bw).transpose(0, 2, 4, 1, 3, 5).reshape(-1)
    lay = lay[lay >= 0]
    nv = T * H * W
    assert np.array_equal(res["q_perm"][:nv], lay)
    assert np.array_equal(res["q_perm"][nv:], np.arange(nv, nv + n_text))
    ext = lambda n, b: np.minimum(b, n - b * np.arange(-(-n // b)))
    sizes = (ext(T, bt)[:, None, None] * ext(H, bh)[None, :, None] * ext(W, bw)[None, None, :]).reshape(-1)
    assert np.array_equal(res["q_sizes"][:27], sizes)
    assert res["q_sizes"][27] == n_text
    # text: the text row attends everything, every row attends text
    bits = _bits(res["kmask"], 28)
    assert bits[27].all() and bits[:, 27].all()
    assert bits[:27, :27].sum() == 27   # Tw = Sw = 1, no stride: the diagonal only


def test_table7_configurations_on_the_wan_grid():
    """The Wan 2.1 grid (21 x 45 x 80, PSABlock 3 x 8 x 16: T' = 7, H' = 6,
    W' = 5). Under Algorithm 1 as printed, a stride no larger than the width
    keeps the whole axis, so e.g. (7, 0, inf)(3, 0, 3) is the full mask; the
    kept fractions of the other listed configurations follow the closed forms."""
    grid, block = (21, 45, 80), (3, 8, 16)
    t, s, (Tb, Hb, Wb) = _coords(*grid, block)
    assert (Tb, Hb, Wb) == (7, 6, 5)
    full = oracle.psa_plan(*grid, block, 0, (7, 0, INF, 3, 0, 3))
    assert _bits(full["kmask"], full["G"]).all()
    p = oracle.psa_plan(*grid, block, 0, (1, 0, INF, 5, 0, 6))
    want = (t[None] == t[:, None]) & (np.abs(s[None] - s[:, None]) % 6 < 5)
    assert np.array_equal(_bits(p["kmask"], p["G"]), want)


def test_seeded_strategies_are_deterministic_and_in_range():
    """The workload's per-head stripe parameters: the same draw every time,
    widths and strides in the appendix C.2 ranges, Table 7 rows or the full
    window on the Wan 2.1 14B block grid."""
    import workload
    w = workload.get("wan2.1-14b")
    a = workload.psa_strategies(w)
    assert a == workload.psa_strategies(w) and len(a) == w.B * w.H
    table7 = {c[0] + c[1] for c, _ in workload.PSA_TABLE7 if c is not None}
    full = (7, 0, INF, 30, 0, INF)
    for prm in a:
        Tw, To, Ts, Sw, So, Ss = prm
        assert 1 <= Tw <= 7 and To in (0, 1, -1, 2, -2) and Ts in (1, 2, 3, INF)
        assert 1 <= Sw <= 30 and So in (0, 1, -1) and Ss in (1, 3, 5, 6, INF)
        assert prm in table7 or prm == full or (Tw < 7 and Sw < 5)
