"""Seeded synthetic inputs for the submanifold 3x3x3 sparse convolution.

This module only draws inputs: voxel coordinate sets, features and KRSC weights.
It holds none of the convolution's arithmetic (no neighbour lookup, no
contraction), so both the CPU oracle and the CUDA path can be fed from it.

The five workloads stand in for the pages' "128^3/128ch" layer and for real
V-VAE activations, neither of which is available (trellis_sparse_mrp_mlx
commit log, closing paragraph; lato.2_mrp_mlx CLAUDE.md, "Key facts").  The
surface-shell shapes follow the structure-stage occupancy the Pixal3D pages
report (a few percent of a 64^3 grid, pixal3d_mrp_mlx sampler.py commit log).

Coordinates are int32 rows (b, z, y, x) in raster order (b, z, y, x
lexicographic); the weight layout is spconv's KRSC [Cout, kz, ky, kx, Cin]
(lato.2_mrp_mlx CLAUDE.md, "Key facts").
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "make_workload", "tiny_coords", "random_coords", "shell_coords",
    "headline_coords", "dense_coords", "batched_coords", "make_features",
    "make_weight", "permute_rows", "to_bf16_values",
]


def _raster(occ: np.ndarray, b: int = 0) -> np.ndarray:
    """Occupied cells of a [G,G,G] bool grid as int32 (b,z,y,x) rows, raster order."""
    z, y, x = np.nonzero(occ)
    out = np.empty((z.size, 4), np.int32)
    out[:, 0] = b
    out[:, 1] = z
    out[:, 2] = y
    out[:, 3] = x
    return out


def _add_shell(occ: np.ndarray, r: float, c, half: float) -> None:
    """Mark every integer point p of the grid with | |p - c| - r | <= half."""
    g = occ.shape[0]
    lo = [max(0, int(np.floor(ci - r - half))) for ci in c]
    hi = [min(g, int(np.ceil(ci + r + half)) + 1) for ci in c]
    if any(h <= l for l, h in zip(lo, hi)):
        return
    z, y, x = np.meshgrid(np.arange(lo[0], hi[0]), np.arange(lo[1], hi[1]),
                          np.arange(lo[2], hi[2]), indexing="ij")
    d = np.sqrt((z - c[0]) ** 2 + (y - c[1]) ** 2 + (x - c[2]) ** 2)
    occ[lo[0]:hi[0], lo[1]:hi[1], lo[2]:hi[2]] |= np.abs(d - r) <= half


def tiny_coords(seed: int = 0, grid: int = 16, p: float = 0.3) -> np.ndarray:
    """Batch 1, 16^3 grid, each cell occupied i.i.d. with probability p (1,223 voxels at seed 0)."""
    occ = np.random.default_rng(seed).random((grid, grid, grid)) < p
    return _raster(occ)


def random_coords(seed: int, grid: int, batch: int, p: float) -> np.ndarray:
    """`batch` grids of grid^3 cells, each cell occupied i.i.d. with probability
    p; rows in raster order (b, z, y, x)."""
    rng = np.random.default_rng(seed)
    parts = [_raster(rng.random((grid, grid, grid)) < p, b) for b in range(batch)]
    return np.concatenate(parts) if parts else np.empty((0, 4), np.int32)


def shell_coords(grid: int = 64, radius: float = 24.0, half: float = 1.0) -> np.ndarray:
    """One sphere shell | |p - (32,32,32)| - 24 | <= 1 in a 64^3 grid (14,534 voxels)."""
    occ = np.zeros((grid,) * 3, bool)
    ctr = grid / 2.0
    _add_shell(occ, radius, (ctr, ctr, ctr), half)
    return _raster(occ)


def headline_coords(seed: int = 0, grid: int = 128, n_shells: int = 8,
                    half: float = 2.0) -> np.ndarray:
    """Union of 8 shells in a 128^3 grid: r ~ U[12,40], centre ~ U[r+2, 125-r]^3,
    half-width 2 (329,839 voxels at seed 0)."""
    rng = np.random.default_rng(seed)
    occ = np.zeros((grid,) * 3, bool)
    for _ in range(n_shells):
        r = rng.uniform(12, 40)
        c = rng.uniform(r + 2, 125 - r, size=3)
        _add_shell(occ, r, c, half)
    return _raster(occ)


def dense_coords(grid: int = 128, batch: int = 1) -> np.ndarray:
    """Every cell of a grid^3 volume, for each batch element (2,097,152 voxels at 128^3)."""
    occ = np.ones((grid,) * 3, bool)
    return np.concatenate([_raster(occ, b) for b in range(batch)])


def batched_coords(batch: int = 4, grid: int = 256, min_voxels: int = 250_000,
                   seed0: int = 100, half: float = 1.0, r_lo: float = 16.0,
                   r_hi: float = 48.0) -> np.ndarray:
    """Batch of independent shell sets in a 256^3 grid.  Element b draws from
    rng(100+b) and adds shells r ~ U[16,48], centre ~ U[r+1, grid-2-r]^3,
    half-width 1, until it holds at least 250k voxels (1,135,307 in total)."""
    parts = []
    for b in range(batch):
        rng = np.random.default_rng(seed0 + b)
        occ = np.zeros((grid,) * 3, bool)
        while int(occ.sum()) < min_voxels:
            r = rng.uniform(r_lo, r_hi)
            c = rng.uniform(r + 1, grid - 2 - r, size=3)
            _add_shell(occ, r, c, half)
        parts.append(_raster(occ, b))
    return np.concatenate(parts)


def make_features(n: int, c: int, seed: int) -> np.ndarray:
    """float32 features ~ N(0, 1), shape [n, c]."""
    return np.random.default_rng(seed).standard_normal((n, c), dtype=np.float32)


def make_weight(cout: int, cin: int, seed: int) -> np.ndarray:
    """KRSC weight [Cout, 3, 3, 3, Cin] ~ N(0, std = 1/sqrt(27*Cin)), float32."""
    w = np.random.default_rng(seed).standard_normal((cout, 3, 3, 3, cin), dtype=np.float32)
    return (w * np.float32(1.0 / np.sqrt(27.0 * cin))).astype(np.float32)


def permute_rows(n: int, seed: int) -> np.ndarray:
    """A seeded random permutation of the row order (int64)."""
    return np.random.default_rng(seed).permutation(n)


def to_bf16_values(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round-to-nearest-even) and return them
    as float32, i.e. the exact values a bf16 tensor holds.  Done with torch's
    float32 -> bfloat16 cast, which is a single RNE rounding."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16).float().numpy()


@dataclass
class Workload:
    """One synthetic workload: a coordinate set plus the layer shapes run on it."""
    name: str
    coords: np.ndarray          # int32 [N, 4] (b, z, y, x)
    grid_dim: int
    batch: int
    channels: list              # [C0, C1, ...]: layer l maps C_l -> C_{l+1}
    dtype: str                  # "f32" or "bf16"
    gelu_between: bool = False  # exact-erf GELU after every layer but the last
    seed: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def n(self) -> int:
        return int(self.coords.shape[0])

    def features(self) -> np.ndarray:
        x = make_features(self.n, self.channels[0], self.seed + 1)
        return to_bf16_values(x) if self.dtype == "bf16" else x

    def weights(self) -> list:
        ws = []
        for l in range(len(self.channels) - 1):
            w = make_weight(self.channels[l + 1], self.channels[l], self.seed + 2 + l)
            ws.append(to_bf16_values(w) if self.dtype == "bf16" else w)
        return ws


WORKLOADS = ("tiny", "shell", "shell_bf16", "headline", "dense", "batched")


def make_workload(name: str) -> Workload:
    """The synthetic workloads by name (sizes in the docstrings above)."""
    if name == "tiny":
        return Workload("tiny 16^3 p=0.3 8->8 f32", tiny_coords(), 16, 1, [8, 8], "f32")
    if name == "shell":
        return Workload("shell 64^3 r=24 64->64 f32", shell_coords(), 64, 1, [64, 64], "f32")
    if name == "shell_bf16":
        return Workload("shell 64^3 r=24 64->64 bf16", shell_coords(), 64, 1, [64, 64], "bf16")
    if name == "headline":
        return Workload("headline 128^3 8 shells 128->128 bf16", headline_coords(), 128, 1,
                        [128, 128], "bf16")
    if name == "dense":
        return Workload("dense 128^3 128->128 bf16", dense_coords(), 128, 1, [128, 128], "bf16")
    if name == "batched":
        return Workload("batched 4x256^3 shells 64->128->128->128->64 bf16 GELU",
                        batched_coords(), 256, 4, [64, 128, 128, 128, 64], "bf16",
                        gelu_between=True)
    raise KeyError(name)
