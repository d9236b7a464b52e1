"""Pins of the CPU oracle against things other than itself.

Each test checks one oracle function against a closed form, brute force on a
tiny input, an invariant the pages state, or a value the pages print, chosen so
that a plausible slip (dropped term, wrong sign, transposed operand, off-by-one
tie rule) fails at least one of them. No GPU and no CUDA library are involved.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
import workload
from workload import bf16_bits_to_f32, f32_to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_bf16(rng, shape, scale=1.0):
    return f32_to_bf16_bits((scale * rng.standard_normal(shape)).astype(np.float32))


# --------------------------------------------------------------------- exp


def test_exp_close_to_libm():
    """oracle_exp (Cody-Waite + Taylor) stays within a few ulp of libm's exp."""
    xs = np.concatenate([np.linspace(-87.0, 0.0, 20001), -np.logspace(-8, 1.9, 2000)])
    for x in xs:
        x = float(np.float32(x))
        got = oracle.exp(x)
        ref = math.exp(x)
        assert abs(got - ref) <= 4 * 2.0 ** -24 * ref, (x, got, ref)
    assert oracle.exp(0.0) == 1.0
    assert oracle.exp(-87.5) == 0.0 and oracle.exp(-1e4) == 0.0


# --------------------------------------------------------------------- metric


def test_metric_identity():
    cent = np.ones((3, 5), dtype=np.float32)
    M = oracle.metric(cent, np.array([1, 2, 3]), identity=True)
    assert np.array_equal(M, np.eye(5))


def test_metric_is_mean_squared_dot_error():
    """(q - mu)^T M (q - mu) equals the mean over all keys of ((q - mu).k)^2 when
    every key sits on its cluster centroid: the interaction error of iCATS 3.1."""
    rng = np.random.default_rng(1)
    C, d = 7, 6
    cent = rng.standard_normal((C, d)).astype(np.float32)
    sizes = np.array([3, 0, 5, 1, 2, 4, 6], dtype=np.int32)
    keys = np.concatenate([np.repeat(cent[b:b + 1].astype(np.float64), sizes[b], 0) for b in range(C)])
    M = oracle.metric(cent, sizes)
    for _ in range(5):
        e = rng.standard_normal(d)
        brute = np.mean((keys @ e) ** 2)
        assert abs(e @ M @ e - brute) <= 1e-12 * max(1.0, brute)
    assert np.allclose(M, M.T, atol=0)
    assert np.linalg.eigvalsh(M).min() > -1e-12


# --------------------------------------------------------------------- assign / update


def _direct_dist(x, cent, M):
    """D_j(x) = (x - mu_j)^T M (x - mu_j) by the unexpanded form."""
    diff = x[:, None, :] - cent[None, :, :].astype(np.float64)
    return np.einsum("njc,cd,njd->nj", diff, M, diff)


@pytest.mark.parametrize("identity", [True, False])
def test_assign_matches_brute_force(identity):
    rng = np.random.default_rng(2)
    n, d, C = 40, 8, 5
    xb = _rand_bf16(rng, (n, d), 2.0)
    x = bf16_bits_to_f32(xb).astype(np.float64)
    cent = (2 * rng.standard_normal((C, d))).astype(np.float32)
    if identity:
        M = np.eye(d)
    else:
        A = rng.standard_normal((d, d))
        M = A @ A.T / d
    a, b1, b2 = oracle.assign(xb, cent, M, with_dist=True)
    D = _direct_dist(x, cent, M)
    assert np.array_equal(a, np.argmin(D, axis=1))
    Ds = np.sort(D, axis=1)
    assert np.allclose(b1, Ds[:, 0], rtol=1e-10, atol=1e-10)
    assert np.allclose(b2, Ds[:, 1], rtol=1e-10, atol=1e-10)


def test_assign_tie_goes_to_smaller_id():
    x = f32_to_bf16_bits(np.array([[0.0, 0.0]], dtype=np.float32))
    cent = np.array([[1.0, 0.0], [0.0, 1.0], [-1.0, 0.0]], dtype=np.float32)
    a = oracle.assign(x, cent, np.eye(2))
    assert a[0] == 0
    a = oracle.assign(x, cent[::-1].copy(), np.eye(2))
    assert a[0] == 0


def test_update_is_exact_mean_and_keeps_empty():
    rng = np.random.default_rng(3)
    n, d, C = 200, 16, 6
    xb = _rand_bf16(rng, (n, d), 3.0)
    x = bf16_bits_to_f32(xb).astype(np.float64)
    labels = rng.integers(0, C - 1, size=n).astype(np.int32)  # cluster C-1 empty
    old = rng.standard_normal((C, d)).astype(np.float32)
    cent, sizes = oracle.update(xb, labels, old)
    for j in range(C):
        m = labels == j
        assert sizes[j] == m.sum()
        if m.any():
            assert np.array_equal(cent[j], np.mean(x[m], axis=0).astype(np.float32))
        else:
            assert np.array_equal(cent[j], old[j])


def test_update_drops_components_below_2_pow_minus_24():
    x = f32_to_bf16_bits(np.array([[2.0 ** -30, 1.0], [2.0 ** -24, 3.0]], dtype=np.float32))
    cent, sizes = oracle.update(x, np.array([0, 0], dtype=np.int32), np.zeros((1, 2), np.float32))
    assert sizes[0] == 2
    assert cent[0, 0] == np.float32(2.0 ** -25) and cent[0, 1] == 2.0


def _objective(x, labels, cent, M):
    D = _direct_dist(x, cent, M)
    return D[np.arange(x.shape[0]), labels].sum()


def test_half_step_is_descent():
    """Under a fixed PSD metric, the assignment and the update each never raise
    the k-means objective sum_i D(x_i, mu_a(i))."""
    rng = np.random.default_rng(4)
    n, d, C = 300, 8, 6
    xb = _rand_bf16(rng, (n, d), 2.0)
    x = bf16_bits_to_f32(xb).astype(np.float64)
    A = rng.standard_normal((d, d))
    M = A @ A.T / d
    cent = x[rng.choice(n, C, replace=False)].astype(np.float32)
    labels = rng.integers(0, C, size=n).astype(np.int32)
    for _ in range(4):
        j0 = _objective(x, labels, cent, M)
        labels = oracle.assign(xb, cent, M)
        j1 = _objective(x, labels, cent, M)
        cent, _ = oracle.update(xb, labels, cent)
        j2 = _objective(x, labels, cent, M)
        assert j1 <= j0 + 1e-9 * abs(j0)
        assert j2 <= j1 * (1 + 1e-6)  # fp32 rounding of the centroids


def test_first_round_query_step_is_lloyd():
    """Round 0's query step is feature-space k-means (iCATS 4.1) from the
    tokens at floor(j n / C): compare with a textbook Lloyd step."""
    rng = np.random.default_rng(5)
    n, d, C = 120, 8, 5
    q = _rand_bf16(rng, (n, d), 2.0)
    k = _rand_bf16(rng, (n, d), 2.0)
    res = oracle.cluster(q, k, C, C, iters=1)
    x = bf16_bits_to_f32(q).astype(np.float64)
    init = x[[j * n // C for j in range(C)]]
    lab = np.argmin(((x[:, None, :] - init[None]) ** 2).sum(-1), axis=1)
    assert np.array_equal(res["q_assign"], lab)
    means = np.stack([x[lab == j].mean(0) if (lab == j).any() else init[j] for j in range(C)])
    assert np.array_equal(res["q_cent"], means.astype(np.float32))
    assert np.array_equal(res["q_sizes"], np.bincount(lab, minlength=C))


def test_key_step_uses_query_metric():
    """The key step of round 0 assigns keys under M built from the freshly
    updated query clusters (the interaction error of the keys)."""
    rng = np.random.default_rng(6)
    n, d, C = 90, 6, 4
    q = _rand_bf16(rng, (n, d), 2.0)
    k = _rand_bf16(rng, (n, d), 2.0)
    res = oracle.cluster(q, k, C, C, iters=1)
    xq = bf16_bits_to_f32(q).astype(np.float64)
    xk = bf16_bits_to_f32(k).astype(np.float64)
    # M_Q as the mean of q q^T with each query replaced by its centroid
    Q_hat = res["q_cent"].astype(np.float64)[res["q_assign"]]
    M = Q_hat.T @ Q_hat / n
    kinit = xk[[j * n // C for j in range(C)]].astype(np.float32)
    lab = np.argmin(_direct_dist(xk, kinit, M), axis=1)
    assert np.array_equal(res["k_assign"], lab)
    assert np.abs(Q_hat - xq).max() > 0  # the metric is not the raw Gram matrix


def test_warm_start_equals_continuation():
    """Two rounds from cold equal one cold round followed by one warm round."""
    rng = np.random.default_rng(7)
    n, d, C = 150, 8, 5
    q = _rand_bf16(rng, (n, d), 2.0)
    k = _rand_bf16(rng, (n, d), 2.0)
    two = oracle.cluster(q, k, C, C, iters=2)
    one = oracle.cluster(q, k, C, C, iters=1)
    cont = oracle.cluster(q, k, C, C, iters=1, warm=(one["q_cent"], one["k_cent"], one["k_sizes"]))
    for key in ("q_assign", "k_assign", "q_cent", "k_cent", "q_sizes", "k_sizes"):
        assert np.array_equal(two[key], cont[key]), key


def _lloyd(x, init, iters):
    """Textbook Lloyd iterations in fp64 from `init` (fp32 centroids after each
    update, an empty cluster keeping its centroid)."""
    cent = init.astype(np.float32)
    for _ in range(iters):
        d2 = ((x[:, None, :] - cent.astype(np.float64)[None]) ** 2).sum(-1)
        lab = np.argmin(d2, axis=1)
        cent = np.stack([x[lab == j].mean(0).astype(np.float32) if (lab == j).any() else cent[j]
                         for j in range(cent.shape[0])])
    return lab, cent


def test_identity_mode_is_independent_lloyd():
    """Under the identity flag both sides run plain k-means of their own tokens
    (the independent Euclidean clustering of iCATS sec. 3.1 / App. D): several
    rounds equal separate textbook Lloyd runs of Q and of K."""
    rng = np.random.default_rng(11)
    n, d, Cq, Ck, iters = 160, 8, 6, 5, 3
    q = _rand_bf16(rng, (n, d), 2.0)
    k = _rand_bf16(rng, (n, d), 2.0)
    res = oracle.cluster(q, k, Cq, Ck, iters=iters, identity=True)
    for side, x_bits, C in (("q", q, Cq), ("k", k, Ck)):
        x = bf16_bits_to_f32(x_bits).astype(np.float64)
        assert (np.abs(x)[x != 0] >= 2.0 ** -24).all()   # no component the update drops
        lab, cent = _lloyd(x, x[[j * n // C for j in range(C)]], iters)
        assert np.array_equal(res[f"{side}_assign"], lab), side
        assert np.array_equal(res[f"{side}_cent"], cent), side
        assert np.array_equal(res[f"{side}_sizes"], np.bincount(lab, minlength=C)), side


def test_identity_mode_sides_do_not_interact():
    """Independent clustering: the key clusters do not depend on the queries
    (and vice versa), while under the interaction metric they do."""
    rng = np.random.default_rng(12)
    n, d, C = 140, 8, 5
    q = _rand_bf16(rng, (n, d), 2.0)
    k = _rand_bf16(rng, (n, d), 2.0)
    q2 = _rand_bf16(rng, (n, d), 2.0)
    a = oracle.cluster(q, k, C, C, iters=3, identity=True)
    b = oracle.cluster(q2, k, C, C, iters=3, identity=True)
    for key in ("k_assign", "k_cent", "k_sizes"):
        assert np.array_equal(a[key], b[key]), key
    ca = oracle.cluster(q, k, C, C, iters=3)
    cb = oracle.cluster(q2, k, C, C, iters=3)
    assert not np.array_equal(ca["k_assign"], cb["k_assign"])


def test_identity_warm_start_is_lloyd_from_given_centroids():
    rng = np.random.default_rng(13)
    n, d, C = 120, 6, 4
    q = _rand_bf16(rng, (n, d), 2.0)
    k = _rand_bf16(rng, (n, d), 2.0)
    qc0 = rng.standard_normal((C, d)).astype(np.float32)
    kc0 = rng.standard_normal((C, d)).astype(np.float32)
    res = oracle.cluster(q, k, C, C, iters=2, warm=(qc0, kc0, np.zeros(C, np.int32)), identity=True)
    for side, x_bits, c0 in (("q", q, qc0), ("k", k, kc0)):
        x = bf16_bits_to_f32(x_bits).astype(np.float64)
        lab, cent = _lloyd(x, c0, 2)
        assert np.array_equal(res[f"{side}_assign"], lab), side
        assert np.array_equal(res[f"{side}_cent"], cent), side


# --------------------------------------------------------------------- pair mass / selection


def test_pair_mass_is_cluster_softmax_mass():
    rng = np.random.default_rng(8)
    Cq, Ck, d = 9, 11, 16
    qc = rng.standard_normal((Cq, d)).astype(np.float32)
    kc = rng.standard_normal((Ck, d)).astype(np.float32)
    qs = rng.integers(0, 50, Cq).astype(np.int32)
    ks = rng.integers(0, 50, Ck).astype(np.int32)
    ks[3] = 0
    scale = 1.0 / math.sqrt(d)
    w, top1 = oracle.pair_mass(qc, kc, qs, ks, scale)
    s = (qc.astype(np.float64) @ kc.astype(np.float64).T) * scale
    ref = np.zeros_like(s)
    for a in range(Cq):
        live = ks > 0
        z = np.where(live, np.log(np.maximum(ks, 1)) + s[a], -np.inf)
        p = np.exp(z - z.max())
        ref[a] = qs[a] * p / p.sum()
    assert np.allclose(w, ref, rtol=2e-5, atol=1e-6 * qs.max())
    assert np.all(w[:, 3] == 0)
    assert np.allclose(w.sum(1), qs, rtol=1e-5)
    for a in range(Cq):
        assert top1[a] == int(np.argmax(w[a]))


def _kept_pairs(km, Cq, Ck):
    kept = np.zeros((Cq, Ck), dtype=bool)
    for a in range(Cq):
        for b in range(Ck):
            kept[a, b] = (int(km[a, b // 64]) >> (b % 64)) & 1
    return kept


@pytest.mark.parametrize("keep", [0.01, 0.05, 0.25, 0.6, 1.0])
def test_select_keep_ratio(keep):
    rng = np.random.default_rng(9)
    Cq, Ck = 20, 70
    w = rng.random((Cq, Ck)).astype(np.float32)
    w[3, :] = 0.5  # a row of exact ties
    top1 = np.argmax(w, axis=1).astype(np.int32)
    km, L = oracle.select(w, top1, keep=keep)
    K = math.ceil(np.float32(keep) * np.float32(Cq * Ck))
    assert L == max(K, Cq)
    kept = _kept_pairs(km, Cq, Ck)
    assert kept.sum() == L
    assert all(kept[a, top1[a]] for a in range(Cq))
    forced = np.zeros_like(kept)
    forced[np.arange(Cq), top1] = True
    free_kept = w[kept & ~forced]
    dropped = w[~kept]
    if free_kept.size and dropped.size:
        assert free_kept.min() >= dropped.max()
    # ties broken by (a asc, b asc): among equal weights at the threshold the kept are first
    if free_kept.size and dropped.size and free_kept.min() == dropped.max():
        t = free_kept.min()
        ka = [(a, b) for a, b in zip(*np.nonzero(kept & ~forced & (w == t)))]
        da = [(a, b) for a, b in zip(*np.nonzero(~kept & (w == t)))]
        assert max(ka) < min(da)


def test_select_top_p():
    rng = np.random.default_rng(10)
    Cq, Ck = 12, 30
    w = (rng.random((Cq, Ck)) ** 4).astype(np.float32)
    top1 = np.argmax(w, axis=1).astype(np.int32)
    for p in (0.3, 0.7, 0.95):
        km, L = oracle.select(w, top1, mode=1, top_p=p)
        kept = _kept_pairs(km, Cq, Ck)
        fx = np.floor(w.astype(np.float64) * 2.0 ** 32)
        target = math.ceil(p * fx.sum())
        assert fx[kept].sum() >= target
        forced = np.zeros_like(kept)
        forced[np.arange(Cq), top1] = True
        free = kept & ~forced
        if free.any():  # dropping the lightest free pair falls below the target
            a, b = min(zip(*np.nonzero(free)), key=lambda ab: (w[ab], -ab[0], -ab[1]))
            assert fx[kept].sum() - fx[a, b] < target
        assert (w[~kept].max() if (~kept).any() else 0) <= (w[free].min() if free.any() else np.inf)


def test_select_text_bits():
    w = np.ones((3, 4), dtype=np.float32)
    km, L = oracle.select(w, np.zeros(3, np.int32), keep=0.25, has_text=True)
    assert km.shape == (4, 1)
    assert L == 3
    for a in range(3):
        assert (int(km[a, 0]) >> 4) & 1
    assert int(km[3, 0]) == 0b11111


# --------------------------------------------------------------------- tail merging


def test_tail_merge_golden_case():
    g = json.load(open(os.path.join(GOLDEN, "tail_merge_case1.json")))
    km = np.array(g["kmask"], dtype=np.uint64)[:, None]
    labels = np.array(g["labels"], dtype=np.int32)
    sizes = np.bincount(labels, minlength=km.shape[0]).astype(np.int32)
    km2, sz, lb, ne, st = oracle.tail_merge(km, sizes, labels, g["block_q"], g["rounds"])
    assert km2[:, 0].tolist() == g["expected_kmask"]
    assert sz.tolist() == g["expected_sizes"]
    assert lb.tolist() == g["expected_labels"]
    assert ne == g["expected_nonempty"]
    assert st.tolist() == g["expected_stats"]


def _random_plan(seed, n=600, Cq=24, Ck=40, bq=16):
    rng = np.random.default_rng(seed)
    labels = rng.integers(0, Cq, n).astype(np.int32)
    labels[labels == 5] = 6  # an empty cluster
    sizes = np.bincount(labels, minlength=Cq).astype(np.int32)
    base = rng.random((4, Ck)) < 0.3
    km = np.zeros((Cq, 1), dtype=np.uint64)
    for a in range(Cq):
        bits = base[a % 4] ^ (rng.random(Ck) < 0.05)
        km[a, 0] = np.uint64(sum(1 << b for b in range(Ck) if bits[b]))
    return km, sizes, labels, bq


@pytest.mark.parametrize("seed", [11, 12, 13])
def test_tail_merge_invariants(seed):
    km, sizes, labels, bq = _random_plan(seed)
    km2, sz, lb, ne, st = oracle.tail_merge(km, sizes, labels, bq)
    assert sz.sum() == sizes.sum()
    assert np.array_equal(np.bincount(lb, minlength=sz.shape[0]), sz)
    for i in range(labels.shape[0]):  # every token keeps at least its keys
        old, new = int(km[labels[i], 0]), int(km2[lb[i], 0])
        assert old & ~new == 0
    assert st[4] <= st[3]
    assert ne == int((sz > 0).sum())
    assert st[4] == sum(-(-int(s) // bq) for s in sz)


def test_identical_mask_merge_keeps_attention():
    """Step (i) alone (rounds=0) does not change any row's attention output."""
    rng = np.random.default_rng(14)
    n, d, Cq, Ck = 96, 8, 6, 5
    q = _rand_bf16(rng, (n, d))
    k = _rand_bf16(rng, (n, d))
    v = _rand_bf16(rng, (n, d))
    ql = rng.integers(0, Cq, n).astype(np.int32)
    kl = rng.integers(0, Ck, n).astype(np.int32)
    km = np.array([[0b00011], [0b00110], [0b00011], [0b11000], [0b00110], [0b00001]], dtype=np.uint64)
    sizes = np.bincount(ql, minlength=Cq).astype(np.int32)
    km2, sz, lb, ne, st = oracle.tail_merge(km, sizes, ql, 4, rounds=0)
    assert st[0] == 2 and st[1] == 0 and st[2] == 0
    rows = np.arange(n, dtype=np.int32)
    o1, _, _ = oracle.attn_rows(q, k, v, 0.35, ql, kl, km, rows)
    o2, _, _ = oracle.attn_rows(q, k, v, 0.35, lb, kl, km2, rows)
    assert np.array_equal(o1, o2)


# --------------------------------------------------------------------- permutation and tiles


def test_permute_stable_bijection():
    rng = np.random.default_rng(15)
    n, G = 500, 13
    lab = rng.integers(0, G, n).astype(np.int32)
    lab[lab == 4] = 5
    perm, off = oracle.permute(lab, G)
    assert np.array_equal(np.sort(perm), np.arange(n))
    assert off[0] == 0 and off[-1] == n
    assert np.array_equal(np.diff(off), np.bincount(lab, minlength=G))
    for g in range(G):
        seg = perm[off[g]:off[g + 1]]
        assert np.all(lab[seg] == g)
        assert np.all(np.diff(seg) > 0)


def test_tiles_cover_groups():
    off = np.array([0, 5, 5, 21, 22], dtype=np.int32)
    t = oracle.tiles(off, 8)
    assert t.tolist() == [[0, 0, 5], [2, 5, 8], [2, 13, 8], [3, 21, 1]]


# --------------------------------------------------------------------- attention


def _numpy_attention(q, k, v, scale, allowed):
    qf = bf16_bits_to_f32(q).astype(np.float64)
    kf = bf16_bits_to_f32(k).astype(np.float64)
    vf = bf16_bits_to_f32(v).astype(np.float64)
    s = scale * (qf @ kf.T)
    s = np.where(allowed, s, -np.inf)
    m = s.max(1, keepdims=True)
    p = np.exp(s - m)
    p = p / p.sum(1, keepdims=True)
    return p @ vf


def test_full_mask_equals_dense_attention():
    rng = np.random.default_rng(16)
    n, d = 70, 16
    q, k, v = (_rand_bf16(rng, (n, d), 2.0) for _ in range(3))
    scale = float(np.float32(1 / math.sqrt(d)))
    ql = rng.integers(0, 3, n).astype(np.int32)
    kl = rng.integers(0, 4, n).astype(np.int32)
    km = np.full((3, 1), 0b1111, dtype=np.uint64)
    rows = np.arange(n, dtype=np.int32)
    o, ps, nk = oracle.attn_rows(q, k, v, scale, ql, kl, km, rows)
    od = oracle.dense_attn_rows(q, k, v, scale, rows)
    ref = _numpy_attention(q, k, v, scale, np.ones((n, n), bool))
    assert np.abs(o - ref).max() <= 1e-12
    assert np.abs(od - ref).max() <= 1e-12
    assert np.abs(ps - 1).max() <= 1e-12
    assert np.all(nk == n)


def test_masked_attention_brute_force():
    rng = np.random.default_rng(17)
    n, d, Cq, Ck = 80, 8, 4, 6
    q, k, v = (_rand_bf16(rng, (n, d), 2.0) for _ in range(3))
    ql = rng.integers(0, Cq, n).astype(np.int32)
    kl = rng.integers(0, Ck, n).astype(np.int32)
    km = np.array([[0b000001], [0b101010], [0b111111], [0]], dtype=np.uint64)
    allowed = np.array([[(int(km[ql[i], 0]) >> kl[j]) & 1 for j in range(n)] for i in range(n)], bool)
    rows = np.arange(n, dtype=np.int32)
    o, ps, nk = oracle.attn_rows(q, k, v, 0.3, ql, kl, km, rows)
    live = allowed.any(1)
    ref = _numpy_attention(q[live], k, v, float(np.float32(0.3)), allowed[live])
    assert np.abs(o[live] - ref).max() <= 1e-12
    assert np.all(o[~live] == 0) and np.all(nk[~live] == 0)
    assert np.abs(ps[live] - 1).max() <= 1e-12
    assert np.array_equal(nk, allowed.sum(1))


# --------------------------------------------------------------------- whole path on the tiny case


def test_tiny_plan_invariants():
    w = workload.get("tiny")
    q, k, _ = workload.make_qkv(w, heads=[0])
    p = oracle.plan_head(q[0], k[0], w.n_qc, w.n_kc, w.iters, 0.25, w.block_q)
    assert p["kept"] == math.ceil(0.25 * w.n_qc * w.n_kc)
    assert p["cl"]["q_sizes"].sum() == w.N and p["cl"]["k_sizes"].sum() == w.N
    assert np.array_equal(np.sort(p["q_perm"]), np.arange(w.N))
    assert np.array_equal(np.sort(p["k_perm"]), np.arange(w.N))
    assert p["tiles"][:, 2].sum() == w.N
    assert p["merge_stats"][4] <= p["merge_stats"][3]


def test_generator_deterministic_and_subsettable():
    w = workload.get("tiny")
    q, k, v = workload.make_qkv(w)
    q1, k1, v1 = workload.make_qkv(w, heads=[1])
    assert np.array_equal(q[1], q1[0]) and np.array_equal(v[1], v1[0])
    f = bf16_bits_to_f32(q)
    assert abs(f.std() - math.sqrt(4 + 0.25)) < 0.5
    assert f32_to_bf16_bits(np.array([1.0 + 2 ** -8], np.float32))[0] == 0x3F80  # tie to even
    assert f32_to_bf16_bits(np.array([1.0 + 3 * 2 ** -8], np.float32))[0] == 0x3F82


# ----------------------------------------------------------------------------- SNR-guided top-p
# iCATS section 4.2 / appendix A give the shape of the schedule only (dense
# before the first sparse call, steady early and late, falling in the middle,
# a smooth function of log SNR, parameters tau and p_min); the formula is a
# reading, so these pins check the stated properties and the closed-form
# points of that reading, not values printed on the pages (parity unpinned).


def test_snr_schedule_warmup_dense_and_starts_at_tau():
    p = oracle.snr_top_p(50, warmup=4, p_min=0.7, tau=0.999)
    assert (p[:4] == 1.0).all()
    q = oracle.snr_top_p(50, warmup=0, p_min=0.7, tau=0.999)
    assert q[0] == np.float32(0.999)          # pure noise: SNR = 0
    assert np.array_equal(p[4:], q[4:])         # warm-up does not shift the schedule


@pytest.mark.parametrize("shift", [1.0, 3.0, 5.0])
def test_snr_schedule_monotone_between_p_min_and_tau(shift):
    p = oracle.snr_top_p(200, warmup=0, p_min=0.6, tau=0.99, shift=shift).astype(np.float64)
    assert (np.diff(p) <= 0).all()
    assert p.min() > 0.6 - 1e-7 and p.max() <= 0.99 + 1e-7
    # noise-free limit: the last of many steps is close to p_min
    assert oracle.snr_top_p(100000, 0, 0.6, 0.99, shift)[-1] < 0.6 + 1e-6


@pytest.mark.parametrize("steps,shift,t_mid", [(50, 1.0, 25), (40, 3.0, 30), (60, 5.0, 50)])
def test_snr_schedule_midpoint_where_snr_is_one(steps, shift, t_mid):
    """SNR = 1 where the shifted noise level is 1/2, i.e. s = 1 / (1 + shift),
    t = steps (1 - s): there p is the mean of tau and p_min."""
    p = oracle.snr_top_p(steps, 0, 0.7, 0.999, shift)
    assert abs(float(p[t_mid]) - (0.7 + 0.999) / 2) < 1e-7
    assert p[t_mid - 1] > p[t_mid] > p[t_mid + 1]


def test_snr_schedule_is_logistic_in_log_snr():
    """Equal steps in log SNR away from SNR = 1 give mirror-image distances
    from the midpoint (the logistic's odd symmetry)."""
    steps = 1000
    p = oracle.snr_top_p(steps, 0, 0.5, 0.9).astype(np.float64)
    sigma = 1.0 - np.arange(steps) / steps
    lam = 2.0 * np.log((1.0 - sigma[1:]) / sigma[1:])
    for a, b in [(100, 900), (250, 750), (400, 600)]:   # lambda(b) = -lambda(a)
        assert abs(lam[a - 1] + lam[b - 1]) < 1e-9
        assert abs((p[a] - 0.7) + (p[b] - 0.7)) < 1e-6


def test_snr_schedule_flat_when_tau_equals_p_min_and_rejects_bad_args():
    assert (oracle.snr_top_p(30, 0, 0.8, 0.8) == np.float32(0.8)).all()
    for bad in [(0, 0, 0.7, 0.9, 1.0), (10, -1, 0.7, 0.9, 1.0), (10, 0, 0.9, 0.7, 1.0),
                (10, 0, 0.7, 1.5, 1.0), (10, 0, 0.7, 0.9, 0.0), (10, 0, -0.1, 0.9, 1.0)]:
        with pytest.raises(ValueError):
            oracle.snr_top_p(*bad)
