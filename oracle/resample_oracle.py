"""Oracle for the resolution changes around the sparse convolution: subdivide,
masked upsample, channel2spatial, spatial2channel and downsample.

TEST INFRASTRUCTURE ONLY: only tests/, the smoke check and the benchmark's
CPU-baseline leg may import this.  It shares no code with the CUDA path.

What the pages fix (trellis_sparse_mrp_mlx commit log; lato.2_mrp_mlx notes):
  * upsampling is SparseSubdivide: coords * 2 + the unit cube, features
    replicated to the 8 children (lato.2 notes "Key facts");
  * upsample is a MASKED expansion: subdivision.feats is an [N, 8] 0/1 mask and
    a voxel emits only its flagged children; the child index decodes
    axis 0 fastest, offset_i = subidx // 2**i % 2 -- the reverse of subdivide's
    C order (trellis_sparse commit log, "upsample is a MASKED expansion");
  * spatial2channel / channel2spatial are sparse space-to-depth and its inverse
    with the slot index sum_i (coord[i] % 2) * 2**i, axis 0 fastest
    (trellis_sparse commit log, "Completes the sparse op surface");
  * downsample is mode 'max' or 'mean' over the children of parent
    coord // 2 (trellis_sparse commit log, "downsample now takes mode").
Readings where the pages are silent (each listed in the design notes):
  * the spatial axes are the coordinate columns (z, y, x) = axes 0, 1, 2; the
    batch index is carried unchanged;
  * expansions list children parent-major, by ascending child index;
  * upsample's children carry the parent's features (replicated, as subdivide);
  * pooled parents come in raster order of (b, z, y, x); spatial2channel puts
    zeros in the channel slots of absent children.
Factor 2 throughout (the pages' decoders double the resolution per stage).
"""
from __future__ import annotations

import numpy as np

__all__ = ["subdivide", "upsample", "channel2spatial", "spatial2channel", "downsample",
           "slot_offsets_c_order", "slot_offsets_axis0_fastest"]


def slot_offsets_c_order(s: int):
    """(dz, dy, dx) of child s of subdivide: C order, x fastest."""
    return (s >> 2) & 1, (s >> 1) & 1, s & 1


def slot_offsets_axis0_fastest(s: int):
    """(dz, dy, dx) of child s of upsample / channel2spatial: offset_i = s // 2**i % 2."""
    return s & 1, (s >> 1) & 1, (s >> 2) & 1


def _expand(coords, feats, mask, offsets, slice_channels):
    coords = np.asarray(coords, np.int64)
    feats = np.asarray(feats)
    n = coords.shape[0]
    c_child = feats.shape[1] // 8 if slice_channels else feats.shape[1]
    out_c, out_f = [], []
    for i in range(n):
        b, z, y, x = (int(v) for v in coords[i])
        for s in range(8):
            if mask is not None and not mask[i, s]:
                continue
            dz, dy, dx = offsets(s)
            out_c.append((b, 2 * z + dz, 2 * y + dy, 2 * x + dx))
            out_f.append(feats[i, s * c_child:(s + 1) * c_child] if slice_channels else feats[i])
    oc = np.array(out_c, np.int32).reshape(-1, 4)
    of = np.array(out_f, feats.dtype).reshape(-1, c_child)
    return oc, of


def subdivide(coords, feats):
    """Every voxel -> its 8 children at 2 * coord + (dz, dy, dx), C order
    (s = 4 dz + 2 dy + dx); features replicated.  Rows: parent-major."""
    return _expand(coords, feats, None, slot_offsets_c_order, False)


def upsample(coords, feats, mask):
    """Masked expansion: voxel i emits child s only where mask[i, s] != 0, child
    offsets decoded axis 0 fastest; features replicated."""
    return _expand(coords, feats, np.asarray(mask), slot_offsets_axis0_fastest, False)


def channel2spatial(coords, feats, mask=None):
    """feats [N, 8 C] -> child s (axis 0 fastest) gets channels [s C, (s + 1) C);
    all 8 children, or only the flagged ones."""
    m = None if mask is None else np.asarray(mask)
    return _expand(coords, feats, m, slot_offsets_axis0_fastest, True)


def _parents(coords):
    """Unique parents coord // 2 in raster order, and each row's parent index
    and child slot (axis 0 fastest)."""
    coords = np.asarray(coords, np.int64)
    par = coords.copy()
    par[:, 1:] //= 2
    keys = [tuple(int(v) for v in p) for p in par]
    uniq = sorted(set(keys))
    index = {k: t for t, k in enumerate(uniq)}
    pid = np.array([index[k] for k in keys], np.int64)
    r = coords[:, 1:] % 2
    slot = r[:, 0] + 2 * r[:, 1] + 4 * r[:, 2]
    return np.array(uniq, np.int32).reshape(-1, 4), pid, slot


def spatial2channel(coords, feats):
    """Children -> parents coord // 2 (raster order); parent channel slot s =
    sum_i (coord[i] % 2) 2**i holds that child's features, zeros where absent."""
    feats = np.asarray(feats)
    pc, pid, slot = _parents(coords)
    c = feats.shape[1]
    out = np.zeros((pc.shape[0], 8 * c), feats.dtype)
    for i in range(feats.shape[0]):
        out[pid[i], slot[i] * c:(slot[i] + 1) * c] = feats[i]
    return pc, out


def downsample(coords, feats, mode: str):
    """Parents coord // 2 in raster order; features: 'max' or 'mean' over the
    children present, in fp64."""
    if mode not in ("max", "mean"):
        raise ValueError("mode must be 'max' or 'mean'")
    feats = np.asarray(feats, np.float64)
    pc, pid, _ = _parents(coords)
    m = pc.shape[0]
    if mode == "max":
        out = np.full((m, feats.shape[1]), -np.inf)
        for i in range(feats.shape[0]):
            out[pid[i]] = np.maximum(out[pid[i]], feats[i])
    else:
        out = np.zeros((m, feats.shape[1]))
        cnt = np.zeros(m)
        for i in range(feats.shape[0]):
            out[pid[i]] += feats[i]
            cnt[pid[i]] += 1
        out /= cnt[:, None]
    return pc, out
