"""Seeded synthetic inputs for the online co-clustered block-sparse attention path.

This module is shared by the CUDA library's tests/bench and by the CPU oracle's
tests. It holds no arithmetic of the method itself: it only draws Q, K, V
tensors (rounded to bf16) and per-head keep ratios with the shapes of the video
DiT attention calls that the SVOO / iCATS / PSA pages evaluate (Wan2.1-1.3B,
Wan2.1-14B, HunyuanVideo-13B) plus a tiny case and a sequence-length sweep.

Recipe (stand-in for real Wan / HunyuanVideo activations, which need trained
models and prompt suites):

* tokens sit on a (t, y, x) grid in row-major order, i = t*Y*X + y*X + x;
* per head h, C_c centers are drawn from N(0, 4 I_d);
* the grid is cut into cells of (ct, cy, cx) tokens; each cell takes one center,
  chosen by splitmix64(cell_id ^ head_seed) mod C_c, or, for the Zipf-skewed
  sweep, drawn from a Zipf(1.2) popularity over the centers;
* Q = center + 0.5 N(0, I), K = center + 0.5 N(0, I) (independent noise),
  V ~ N(0, I);
* optional text tokens (HunyuanVideo) are appended after the video tokens with
  Q, K ~ N(0, 4 I) and V ~ N(0, I);
* every value is drawn as float32 and rounded to bf16 with round-to-nearest-even
  by integer bit operations; arrays are returned as uint16 bit patterns.

Head h of batch b uses the NumPy PCG64 stream seeded with seed*1000 + b*H + h, so
any subset of heads can be generated alone and matches the full tensor.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "get", "splitmix64", "f32_to_bf16_bits",
    "bf16_bits_to_f32", "make_qkv", "cell_centers", "sweep_workload", "psa_strategies",
    "PSA_BLOCKS", "next_timestep",
]

_MASK64 = np.uint64(0xFFFFFFFFFFFFFFFF)


def splitmix64(x: np.ndarray) -> np.ndarray:
    """SplitMix64 finaliser (Steele, Lea, Flood 2014) on uint64 arrays."""
    with np.errstate(over="ignore"):
        z = (np.asarray(x, dtype=np.uint64) + np.uint64(0x9E3779B97F4A7C15)) & _MASK64
        z = ((z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)) & _MASK64
        z = ((z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)) & _MASK64
        return z ^ (z >> np.uint64(31))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even) -> uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention-call shape plus the hyper-parameters of the sparse path."""
    name: str
    B: int
    H: int
    d: int
    grid: tuple            # (T, Y, X) video token grid
    n_text: int            # always-kept text tokens appended after the video tokens
    n_centers: int         # mixture centers per head
    cell: tuple            # (ct, cy, cx) tokens per cell
    n_qc: int              # query clusters
    n_kc: int              # key clusters
    iters: int             # k-means iterations (each = one Q step + one K step)
    block_q: int           # query block (tail-merge / padding granularity)
    block_kv: int          # key/value block
    keep_kind: str         # "const", "choice", "linspace", "schedule"
    keep_args: tuple
    zipf: bool = False
    seed: int = 0

    @property
    def n_video(self) -> int:
        T, Y, X = self.grid
        return T * Y * X

    @property
    def N(self) -> int:
        return self.n_video + self.n_text

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def keep_ratios(self, t: int = 0) -> np.ndarray:
        """Per-(batch, head) keep ratio, float32 [B*H].

        const: one value for every head; choice: uniform draw per head from a
        set; linspace: a seeded shuffle of linspace(lo, hi, H) (a per-layer
        profile standing in for SVOO's offline levels); schedule: the
        SNR-style r(t) = lo + (hi - lo) * (1 - t / T) of call t, same for all
        heads.
        """
        BH = self.B * self.H
        kind, args = self.keep_kind, self.keep_args
        if kind == "const":
            r = np.full(BH, args[0], dtype=np.float64)
        elif kind == "choice":
            rng = np.random.Generator(np.random.PCG64(self.seed * 1000 + 999_983))
            r = rng.choice(np.asarray(args, dtype=np.float64), size=BH)
        elif kind == "linspace":
            lo, hi = args
            rng = np.random.Generator(np.random.PCG64(self.seed * 1000 + 999_979))
            prof = np.linspace(lo, hi, self.H)
            r = np.concatenate([rng.permutation(prof) for _ in range(self.B)])
        elif kind == "schedule":
            lo, hi, steps = args
            r = np.full(BH, lo + (hi - lo) * (1.0 - t / steps), dtype=np.float64)
        else:
            raise ValueError(kind)
        return r.astype(np.float32)


def cell_centers(w: Workload, head_seed: int, rng: np.random.Generator) -> np.ndarray:
    """Center id of every video token (int64 [n_video])."""
    T, Y, X = w.grid
    ct, cy, cx = w.cell
    nyc, nxc = -(-Y // cy), -(-X // cx)
    ntc = -(-T // ct)
    t = np.arange(T)[:, None, None] // ct
    y = np.arange(Y)[None, :, None] // cy
    x = np.arange(X)[None, None, :] // cx
    cell = ((t * nyc + y) * nxc + x).reshape(-1).astype(np.uint64)
    n_cells = ntc * nyc * nxc
    if w.zipf:
        pop = (np.arange(w.n_centers, dtype=np.float64) + 1.0) ** -1.2
        pop /= pop.sum()
        cmap = rng.choice(w.n_centers, size=n_cells, p=pop)
        return cmap[cell.astype(np.int64)]
    h = splitmix64(cell ^ np.uint64(head_seed))
    return (h % np.uint64(w.n_centers)).astype(np.int64)


def make_qkv(w: Workload, heads: Optional[Sequence[int]] = None):
    """Draw Q, K, V as bf16 bit patterns, uint16 arrays [len(heads), N, d].

    `heads` are flat (batch*H + head) indices; default: all B*H heads.
    """
    if heads is None:
        heads = range(w.B * w.H)
    heads = list(heads)
    N, d, nv = w.N, w.d, w.n_video
    q = np.empty((len(heads), N, d), dtype=np.uint16)
    k = np.empty_like(q)
    v = np.empty_like(q)
    for i, hh in enumerate(heads):
        head_seed = w.seed * 1000 + hh
        rng = np.random.Generator(np.random.PCG64(head_seed))
        centers = (2.0 * rng.standard_normal((w.n_centers, d), dtype=np.float32)).astype(np.float32)
        cid = cell_centers(w, head_seed, rng)
        cq = centers[cid]
        nq = rng.standard_normal((nv, d), dtype=np.float32)
        q[i, :nv] = f32_to_bf16_bits(cq + np.float32(0.5) * nq)
        del nq
        nk = rng.standard_normal((nv, d), dtype=np.float32)
        k[i, :nv] = f32_to_bf16_bits(cq + np.float32(0.5) * nk)
        del nk, cq
        v[i, :nv] = f32_to_bf16_bits(rng.standard_normal((nv, d), dtype=np.float32))
        if w.n_text:
            nt = w.n_text
            q[i, nv:] = f32_to_bf16_bits(np.float32(2.0) * rng.standard_normal((nt, d), dtype=np.float32))
            k[i, nv:] = f32_to_bf16_bits(np.float32(2.0) * rng.standard_normal((nt, d), dtype=np.float32))
            v[i, nv:] = f32_to_bf16_bits(rng.standard_normal((nt, d), dtype=np.float32))
    return q, k, v


def next_timestep(x: np.ndarray, sigma: float = 0.1, seed: int = 1) -> np.ndarray:
    """Inputs of the next denoising call, standing in for the slow drift of a
    layer's Q or K from one timestep to the next: x + sigma N(0, I) per token,
    drawn from PCG64(seed) as float32 and rounded to bf16 (uint16 bits, same
    shape as x)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    noise = rng.standard_normal(x.shape, dtype=np.float32)
    return f32_to_bf16_bits(bf16_bits_to_f32(x) + np.float32(sigma) * noise)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 64, (4, 16, 16), 0, 32, (2, 4, 4), 16, 16, 10, 64, 64,
                     "const", (0.25,)),
    "wan2.1-1.3b": Workload("wan2.1-1.3b", 1, 12, 128, (21, 30, 52), 0, 256, (3, 5, 5), 128, 128,
                            10, 128, 128, "choice", (0.1, 0.2, 0.3, 0.5)),
    "wan2.1-14b": Workload("wan2.1-14b", 1, 40, 128, (21, 45, 80), 0, 512, (3, 5, 5), 256, 256,
                           10, 128, 128, "linspace", (0.05, 0.6)),
    "hunyuanvideo-13b": Workload("hunyuanvideo-13b", 1, 24, 128, (33, 45, 80), 256, 512, (3, 5, 5),
                                 256, 256, 10, 128, 128, "schedule", (0.1, 0.5, 50)),
}


def sweep_workload(n_tokens: int, keep: float) -> Workload:
    """Sweep point: H=24, d=128, N tokens on an (N/2048, 32, 64) grid, Zipf-skewed cells."""
    if n_tokens % 2048:
        raise ValueError("sweep sizes are multiples of 2048 tokens")
    return Workload(f"sweep-{n_tokens}-{keep}", 1, 24, 128, (n_tokens // 2048, 32, 64), 0, 512,
                    (3, 5, 5), 256, 256, 10, 128, 128, "const", (keep,), zipf=True)


def get(name: str) -> Workload:
    return WORKLOADS[name]


# --------------------------------------------------------------------------- stripe-mask strategies

# PSABlock per workload for the static stripe mask: 3 x 8 x 16 as the PSA pages
# use for Wan 2.1 (appendix C.2); the HunyuanVideo grid takes 3 x 16 x 16, since
# 3 x 8 x 16 would give 330 blocks and the plan holds at most 256 groups.
PSA_BLOCKS = {"tiny": (2, 4, 4), "wan2.1-1.3b": (3, 8, 16), "wan2.1-14b": (3, 8, 16),
              "hunyuanvideo-13b": (3, 16, 16)}

# The ten most frequent (Tw, To, Ts), (Sw, So, Ss) of PSA-Search on Wan 2.1 14B
# (PSA appendix C.3, Table 7) with their head counts; None = the full window,
# math.inf = an infinite stride. The remaining 27.02% of heads (the table's
# remainder row) are drawn from the candidate ranges of appendix C.2.
PSA_TABLE7 = (
    (None, 32000), (((7, 0, math.inf), (3, 0, 3)), 25257), (((1, 0, math.inf), (5, 0, 6)), 11778),
    (((7, 0, math.inf), (1, 0, 3)), 11069), (((7, 0, math.inf), (3, 0, 1)), 9014),
    (((7, 0, math.inf), (3, 0, 5)), 6810), (((7, 0, math.inf), (1, 0, 5)), 5655),
    (((7, 0, math.inf), (5, 0, 3)), 5470), (((1, 0, 3), (5, 0, 6)), 5088),
    (((3, 0, math.inf), (5, 0, 6)), 4622),
)
PSA_OTHER = 43237


def psa_strategies(w: Workload, block: Optional[tuple] = None) -> list:
    """Per-(batch, head) stripe-mask parameters (Tw, To, Ts, Sw, So, Ss) for a
    workload, drawn (seeded) from the Table 7 head-count distribution, the rest
    uniformly from the appendix C.2 candidate ranges (Tw in [1, T'), To in
    {0, +-1, +-2}, Ts in {1, 2, 3, inf}, Sw in [1, W'), So in {0, +-1}, Ss in
    {1, 3, 5, 6, inf}); the full window is (T', 0, inf, H'W', 0, inf)."""
    block = block or PSA_BLOCKS[w.name]
    T, Y, X = w.grid
    Tb, Yb, Xb = -(-T // block[0]), -(-Y // block[1]), -(-X // block[2])
    rng = np.random.Generator(np.random.PCG64(w.seed * 1000 + 999_971))
    counts = np.array([c for _, c in PSA_TABLE7] + [PSA_OTHER], dtype=np.float64)
    pick = rng.choice(len(counts), size=w.B * w.H, p=counts / counts.sum())
    out = []
    for k in pick:
        if k < len(PSA_TABLE7):
            cfg = PSA_TABLE7[k][0]
            out.append((Tb, 0, math.inf, Yb * Xb, 0, math.inf) if cfg is None else cfg[0] + cfg[1])
        else:
            out.append((int(rng.integers(1, max(Tb, 2))), int(rng.choice([0, 1, -1, 2, -2])),
                        [1, 2, 3, math.inf][rng.integers(4)], int(rng.integers(1, max(Xb, 2))),
                        int(rng.choice([0, 1, -1])), [1, 3, 5, 6, math.inf][rng.integers(5)]))
    return out
