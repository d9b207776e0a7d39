"""Pure-Python oracle for the submanifold 3x3x3 sparse convolution.

TEST INFRASTRUCTURE ONLY: only tests/, the smoke check and the benchmark's
CPU-baseline leg may import this.  It shares no code with the CUDA path.

The op, as the pages define it (lato.2_mrp_mlx, commit 97dcdfb54a message and
CLAUDE.md "Key facts"): every SparseConv3d is a submanifold 3x3x3 convolution
with stride 1 whose output sites are the input sites, weights in spconv's KRSC
layout [Cout, kz, ky, kx, Cin].  The map is a lookup over the coordinate set
(27 lookups per voxel); here it is a Python dict keyed by (b, z, y, x).

Readings of points the pages leave open (each also listed in the design notes):
  * offset order kz-major, k = 9*(dz+1) + 3*(dy+1) + (dx+1): KRSC index order;
  * W[:, kz, ky, kx, :] multiplies the voxel at (z+kz-1, y+ky-1, x+kx-1):
    correlation, torch Conv3d's convention; ``flip`` selects the mirrored
    slice W[:, 26-k, :] (the --flip-kernel A/B of the same commit message);
  * neighbours outside the grid are absent (no wrap); a coordinate outside
    [0, batch) x [0, grid_dim)^3 or given twice is an error;
  * the batch index is part of the key, so batch elements never touch.

This module runs the tiny cases; oracle/cpp.py wraps the C++ oracle, built
from the same definition, for larger ones.  The two are cross-checked.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = ["OFFSETS", "OracleError", "build_map", "forward", "backward_data", "backward_weight",
           "gelu", "silu", "round_bf16",
           "brute_force_map"]

# (dz, dy, dx) for k = 0..26, kz-major: dz slowest, dx fastest.
OFFSETS = [(dz, dy, dx) for dz in (-1, 0, 1) for dy in (-1, 0, 1) for dx in (-1, 0, 1)]


class OracleError(ValueError):
    """A coordinate set the op does not accept (out of range or duplicated)."""


def build_map(coords, grid_dim: int, batch: int = 1) -> np.ndarray:
    """nbr[i, k] = row of the voxel at p_i + d_k, or -1 (int32 [N, 27])."""
    coords = np.asarray(coords)
    table = {}
    for i, (b, z, y, x) in enumerate(coords.tolist()):
        if not (0 <= b < batch and 0 <= z < grid_dim and 0 <= y < grid_dim
                and 0 <= x < grid_dim):
            raise OracleError(f"coordinate {(b, z, y, x)} of row {i} is out of range")
        if (b, z, y, x) in table:
            raise OracleError(f"coordinate {(b, z, y, x)} occurs twice")
        table[(b, z, y, x)] = i
    nbr = np.full((coords.shape[0], 27), -1, np.int32)
    for i, (b, z, y, x) in enumerate(coords.tolist()):
        for k, (dz, dy, dx) in enumerate(OFFSETS):
            nbr[i, k] = table.get((b, z + dz, y + dy, x + dx), -1)
    return nbr


def brute_force_map(coords) -> np.ndarray:
    """The map by an all-pairs scan, with no lookup structure at all: j is the
    k-neighbour of i when both share b and p_j - p_i = d_k.  O(N^2)."""
    c = np.asarray(coords, np.int64)
    n = c.shape[0]
    nbr = np.full((n, 27), -1, np.int32)
    for i in range(n):
        d = c - c[i]                              # [N, 4]
        near = (d[:, 0] == 0) & (np.abs(d[:, 1:]) <= 1).all(axis=1)
        for j in np.nonzero(near)[0]:
            dz, dy, dx = (int(v) for v in d[j, 1:])
            nbr[i, 9 * (dz + 1) + 3 * (dy + 1) + (dx + 1)] = j
    return nbr


def forward(nbr, x, w, flip: bool = False, act: str | None = None,
            round_to_bf16: bool = False, rows=None, bias=None, residual=None) -> np.ndarray:
    """out[i] = act(sum_k Wf[:, k, :] @ x[nbr[i, k]] + bias) + residual[i], in fp64.

    The sum runs over nbr[i, k] != -1.  x: [N, Cin]; w: KRSC [Cout, 3, 3, 3, Cin]
    (or [Cout, 27, Cin]).  Wf[:, k] = w[:, k] (correlation) or w[:, 26 - k] (flip).
    bias: optional [Cout], added to the sum.  act: None, "gelu" (exact erf form)
    or "silu" (v * sigmoid(v)), applied after the bias.  residual: optional
    [N, Cout], added after the activation -- the epilogue of a sparse residual
    block's second convolution (conv + bias + skip).
    round_to_bf16: round the result to bf16 (RNE) once, as a bf16 output would be.
    rows: optional subset of output rows (the result then has len(rows) rows).
    """
    nbr = np.asarray(nbr)
    x = np.asarray(x, np.float64)
    w = np.asarray(w, np.float64)
    cout = w.shape[0]
    w27 = w.reshape(cout, 27, -1)
    rows = range(nbr.shape[0]) if rows is None else [int(r) for r in rows]
    out = np.zeros((len(rows), cout), np.float64)
    for p, i in enumerate(rows):
        acc = np.zeros(cout, np.float64)
        for k in range(27):
            j = int(nbr[i, k])
            if j < 0:
                continue
            kw = 26 - k if flip else k
            acc += w27[:, kw, :] @ x[j]
        out[p] = acc
    if bias is not None:
        out = out + np.asarray(bias, np.float64)[None, :]
    if act == "gelu":
        out = gelu(out)
    elif act == "silu":
        out = silu(out)
    elif act is not None:
        raise ValueError(f"unknown activation {act!r}")
    if residual is not None:
        out = out + np.asarray(residual, np.float64)[list(rows)]
    if round_to_bf16:
        out = round_bf16(out)
    return out


def backward_data(nbr, dy, w, flip: bool = False) -> np.ndarray:
    """Gradient of the forward's output with respect to its input features, in
    fp64, by scattering every term of the forward back to its source row:

        dx[j] += Wf[:, k, :]^T @ dy[i]   for every (i, k) with nbr[i, k] = j.

    dy: [N, Cout]; w: KRSC [Cout, 3, 3, 3, Cin]; returns [N, Cin].  (No
    activation: this is the backward of the convolution itself.)
    """
    nbr = np.asarray(nbr)
    dy = np.asarray(dy, np.float64)
    w = np.asarray(w, np.float64)
    cout = w.shape[0]
    w27 = w.reshape(cout, 27, -1)
    dx = np.zeros((nbr.shape[0], w27.shape[2]), np.float64)
    for i in range(nbr.shape[0]):
        for k in range(27):
            j = int(nbr[i, k])
            if j < 0:
                continue
            kw = 26 - k if flip else k
            dx[j] += w27[:, kw, :].T @ dy[i]
    return dx


def backward_weight(nbr, x, dy, flip: bool = False) -> np.ndarray:
    """Gradient of the forward's output with respect to the KRSC weight, in fp64:

        dW[:, kw, :] += outer(dy[i], x[nbr[i, k]])   for every (i, k), nbr[i, k] != -1,

    kw = k (correlation) or 26 - k (flip).  Returns [Cout, 3, 3, 3, Cin].
    """
    nbr = np.asarray(nbr)
    x = np.asarray(x, np.float64)
    dy = np.asarray(dy, np.float64)
    dw = np.zeros((dy.shape[1], 27, x.shape[1]), np.float64)
    for i in range(nbr.shape[0]):
        for k in range(27):
            j = int(nbr[i, k])
            if j < 0:
                continue
            kw = 26 - k if flip else k
            dw[:, kw, :] += np.outer(dy[i], x[j])
    return dw.reshape(dy.shape[1], 3, 3, 3, x.shape[1])


def gelu(v) -> np.ndarray:
    """Exact-erf GELU, 0.5 * v * (1 + erf(v / sqrt(2))), element-wise in fp64."""
    v = np.asarray(v, np.float64)
    erf = np.vectorize(math.erf, otypes=[np.float64])
    return 0.5 * v * (1.0 + erf(v / math.sqrt(2.0)))


def silu(v) -> np.ndarray:
    """SiLU, v * sigmoid(v) = v / (1 + exp(-v)), element-wise in fp64."""
    v = np.asarray(v, np.float64)
    with np.errstate(over="ignore"):
        return v / (1.0 + np.exp(-v))


def round_bf16(v) -> np.ndarray:
    """Round fp64 values to the nearest bfloat16 value, ties to even.

    bfloat16 keeps 8 significant bits with float32's exponent range: for a
    value in [2^(e-1), 2^e) the spacing is 2^(e-8), never finer than the
    subnormal spacing 2^-133.  np.rint rounds halves to even.
    """
    v = np.asarray(v, np.float64)
    out = v.copy()
    nz = np.isfinite(v) & (v != 0)
    _, e = np.frexp(v[nz])
    q = np.maximum(e.astype(np.int64) - 8, -133)
    r = np.ldexp(np.rint(np.ldexp(v[nz], -q)), q)
    max_bf16 = math.ldexp(255.0, 120)
    r = np.where(np.abs(r) > max_bf16, np.copysign(np.inf, v[nz]), r)
    out[nz] = r
    return out
