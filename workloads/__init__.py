"""Seeded synthetic inputs for partition attention over a DiT token sequence.

This module only *generates data*: configuration records, Gaussian draws, the shared
3-D sinusoidal positional embedding that gives the inputs their spatial locality,
partition / group boundary tables and the static reuse masks that the workloads
prescribe.  It holds none of the attention, merge or importance arithmetic; both the
CUDA path and the fp64 oracle consume what it returns.

Sources (web-page summaries of DiTango, "Cost-Effective Parallel Diffusion Generation
with Selective Attention State Reuse", and SwiftFusion, "Scalable Sequence Parallelism
for Distributed Inference of Diffusion Transformers on GPUs"):

* partitions of the spatiotemporal sequence and the observation that spatially near
  partitions dominate a query's attention -- DiTango, Methodology (spatial locality);
* group-wise decisions over spatially adjacent partitions -- DiTango, Methodology 1
  (group-wise strategy);
* states from an earlier denoising step reused for distant partitions -- DiTango,
  Methodology 1-2 (anchor steps, state composition);
* a sequence-major layout that a chunked all-to-all turns head-major -- SwiftFusion,
  Methodology 2 (Torus Attention).

Readings where the pages are silent:

* tokens are ordered t-major: n = (t*Hh + h)*W + w;
* partition p covers [p*S, min((p+1)*S, N)) with S = ceil(N/P); the last one may be short;
* a group is G consecutive partitions, for queries and keys alike;
* the positional embedding gives each of t, h, w a block of d_a = 2*floor(D/6) channels,
  [sin(pos*om_k) for k < d_a/2] then [cos(pos*om_k)], om_k = 10000**(-2k/d_a); the rest
  of the D channels are zero; the same [N, D] table is added (times alpha) to Q, K and V
  of every batch and head;
* "spatially nearest" groups are ranked by the Euclidean distance between the groups'
  mean (t, h, w) token coordinates, ties to the lower group index.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

__all__ = [
    "Workload", "WORKLOADS", "workload", "part_offsets", "group_row_bounds",
    "pe_3d", "token_coords", "make_qkv", "make_cached_kv", "drift_kv",
    "reuse_mask", "sample_rows", "to_f64", "small_variant",
]


@dataclass(frozen=True)
class Workload:
    """One synthetic workload.  Sizes follow the configurations the pages motivate."""

    name: str
    index: int                   # seeds derive from it: 1000+, 2000+ (cache), 3000+step (drift)
    B: int
    H: int
    grid: tuple                  # (T, Hh, W) latent grid; N = T*Hh*W
    D: int
    dtype: str                   # "f32" or "bf16"
    P: int                       # KV partitions
    G: int = 1                   # partitions per group
    alpha: float = 1.0           # positional-embedding weight
    cache_sigma: float = 0.0     # K_prev = K + sigma*N(0,1), V likewise (0: no cache)
    mask: str = "all"            # "all" | "neighbours" | "nearest"
    mask_keep: int = 0           # fresh KV groups per query group for mask == "nearest"
    steps: int = 1               # denoising-trajectory steps
    drift: float = 0.0           # K_s = K_{s-1} + drift*N(0,1), V likewise
    anchors: tuple = ()          # anchor steps (all partitions fresh, importance refreshed)
    threshold: float = 0.0       # reuse partitions whose stored importance is below it
    chunks: int = 1              # sequence chunks of the seq-major -> head-major relayout
    seq_major: bool = False      # inputs start as [N][H][D] (B == 1)

    @property
    def N(self) -> int:
        t, h, w = self.grid
        return t * h * w

    @property
    def S(self) -> int:
        return -(-self.N // self.P)

    @property
    def QG(self) -> int:
        return -(-self.P // self.G)

    @property
    def KG(self) -> int:
        return self.QG

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2


WORKLOADS = {
    0: Workload("tiny full recompute", 0, B=1, H=2, grid=(4, 16, 16), D=64, dtype="f32", P=4),
    1: Workload("image DiT with reuse", 1, B=1, H=24, grid=(1, 64, 64), D=128, dtype="bf16",
                P=8, cache_sigma=0.05, mask="neighbours"),
    2: Workload("720p video DiT", 2, B=1, H=40, grid=(21, 45, 80), D=128, dtype="bf16",
                P=32, G=4, cache_sigma=0.03, mask="nearest", mask_keep=2),
    3: Workload("denoising trajectory", 3, B=1, H=24, grid=(1, 64, 64), D=128, dtype="bf16",
                P=8, steps=10, drift=0.02, anchors=(0, 5), threshold=0.05, mask="weights"),
    4: Workload("long-sequence Ulysses layout", 4, B=1, H=24, grid=(8, 90, 160), D=128,
                dtype="bf16", P=64, chunks=16, seq_major=True),
}


def workload(i: int) -> Workload:
    return WORKLOADS[i]


def small_variant(wl: Workload, grid: tuple, H: int, **kw) -> Workload:
    """Same recipe on a smaller grid / fewer heads (oracle-sized parity cases)."""
    d = dict(wl.__dict__)
    d.update(grid=tuple(grid), H=H, name=wl.name + f" (grid {grid}, H={H})")
    d.update(kw)
    return Workload(**d)


def part_offsets(N: int, P: int) -> np.ndarray:
    """int32[P+1]: partition p covers tokens [off[p], off[p+1])."""
    S = -(-N // P)
    return np.array([min(p * S, N) for p in range(P + 1)], dtype=np.int32)


def group_row_bounds(part_off: np.ndarray, G: int) -> np.ndarray:
    """int32[QG+1]: group g covers tokens [b[g], b[g+1]) (G consecutive partitions)."""
    P = len(part_off) - 1
    QG = -(-P // G)
    return np.array([part_off[min(g * G, P)] for g in range(QG + 1)], dtype=np.int32)


def token_coords(grid: tuple) -> np.ndarray:
    """float64[N, 3]: (t, h, w) of each token in t-major flattened order."""
    T, Hh, W = grid
    t, h, w = np.meshgrid(np.arange(T), np.arange(Hh), np.arange(W), indexing="ij")
    return np.stack([t.ravel(), h.ravel(), w.ravel()], axis=1).astype(np.float64)


def pe_3d(grid: tuple, D: int) -> np.ndarray:
    """float32[N, D] shared 3-D sinusoidal positional embedding (reading in module doc)."""
    coords = token_coords(grid)
    N = coords.shape[0]
    d_a = 2 * (D // 6)
    half = d_a // 2
    omega = 10000.0 ** (-2.0 * np.arange(half) / d_a)
    pe = np.zeros((N, D), dtype=np.float64)
    for axis in range(3):
        ang = coords[:, axis:axis + 1] * omega[None, :]
        pe[:, axis * d_a: axis * d_a + half] = np.sin(ang)
        pe[:, axis * d_a + half: (axis + 1) * d_a] = np.cos(ang)
    return pe.astype(np.float32)


def _normal(seed: int, shape) -> np.ndarray:
    return np.random.default_rng(seed).standard_normal(size=shape, dtype=np.float32)


def make_qkv(wl: Workload) -> dict:
    """Q, K, V as CPU torch tensors in the workload dtype.

    Head-major [B, H, N, D], or sequence-major [N, H, D] when ``wl.seq_major`` (B == 1).
    Draw order from seed 1000+index: Q, then K, then V, each ~N(0, 1) in fp32, plus
    alpha * PE broadcast over batch and heads, then rounded (round-to-nearest-even).
    """
    rng = np.random.default_rng(1000 + wl.index)
    pe = pe_3d(wl.grid, wl.D)
    out = {}
    for name in ("q", "k", "v"):
        if wl.seq_major:
            assert wl.B == 1
            x = rng.standard_normal(size=(wl.N, wl.H, wl.D), dtype=np.float32)
            x += wl.alpha * pe[:, None, :]
        else:
            x = rng.standard_normal(size=(wl.B, wl.H, wl.N, wl.D), dtype=np.float32)
            x += wl.alpha * pe[None, None, :, :]
        out[name] = torch.from_numpy(x).to(wl.torch_dtype)
    return out


def make_cached_kv(wl: Workload, k: torch.Tensor, v: torch.Tensor):
    """K_prev, V_prev = K + sigma*N(0,1), V + sigma*N(0,1) (fp32, then rounded).

    Seed 2000+index; K's noise is drawn before V's.  Q_prev = Q.
    """
    rng = np.random.default_rng(2000 + wl.index)
    outs = []
    for x in (k, v):
        n = rng.standard_normal(size=tuple(x.shape), dtype=np.float32)
        outs.append((x.float() + wl.cache_sigma * torch.from_numpy(n)).to(wl.torch_dtype))
    return outs[0], outs[1]


def drift_kv(wl: Workload, k: torch.Tensor, v: torch.Tensor, step: int):
    """One trajectory step of drift: X_s = X_{s-1} + drift*N(0,1), seed 3000+step."""
    rng = np.random.default_rng(3000 + step)
    outs = []
    for x in (k, v):
        n = rng.standard_normal(size=tuple(x.shape), dtype=np.float32)
        outs.append((x.float() + wl.drift * torch.from_numpy(n)).to(wl.torch_dtype))
    return outs[0], outs[1]


def reuse_mask(wl: Workload) -> np.ndarray:
    """uint8[QG, KG] static reuse mask prescribed by the workload (1 = compute fresh).

    * "all": every pair fresh;
    * "neighbours": query partition q recomputes KV partitions q-1, q, q+1 (no wrap);
    * "nearest": each query group recomputes its ``mask_keep`` spatially nearest KV
      groups (centroid distance, ties to the lower index).
    Trajectory workloads ("weights") choose their masks from stored importance at run
    time; their static mask is all ones (the anchor step).
    """
    QG, KG = wl.QG, wl.KG
    if wl.mask in ("all", "weights"):
        return np.ones((QG, KG), dtype=np.uint8)
    if wl.mask == "neighbours":
        m = np.zeros((QG, KG), dtype=np.uint8)
        for q in range(QG):
            for k in range(max(0, q - 1), min(KG, q + 2)):
                m[q, k] = 1
        return m
    if wl.mask == "nearest":
        bounds = group_row_bounds(part_offsets(wl.N, wl.P), wl.G)
        coords = token_coords(wl.grid)
        cent = np.stack([coords[bounds[g]:bounds[g + 1]].mean(axis=0) for g in range(KG)])
        m = np.zeros((QG, KG), dtype=np.uint8)
        for q in range(QG):
            d = np.sqrt(((cent - cent[q]) ** 2).sum(axis=1))
            order = sorted(range(KG), key=lambda g: (d[g], g))
            for g in order[:wl.mask_keep]:
                m[q, g] = 1
        return m
    raise ValueError(wl.mask)


def sample_rows(wl: Workload, n_random: int = 512, seed: int = 77) -> np.ndarray:
    """Sorted int64 query rows for full-size spot checks.

    ``n_random`` seeded random rows plus every row of the first and the last query
    partition (the ragged tail included).
    """
    off = part_offsets(wl.N, wl.P)
    rng = np.random.default_rng(seed)
    r = rng.choice(wl.N, size=min(n_random, wl.N), replace=False)
    first = np.arange(off[0], off[1])
    last = np.arange(off[-2], off[-1])
    return np.unique(np.concatenate([r, first, last])).astype(np.int64)


def to_f64(x: torch.Tensor) -> np.ndarray:
    """Exact upcast of a (CPU) input tensor to float64 numpy."""
    return x.detach().to("cpu").double().numpy()
