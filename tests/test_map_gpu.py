"""Neighbour-map build on the GPU vs the CPU oracle: bit-exact on every
workload, under raster and random row order, for both key forms, plus the
per-tile offset masks and the device-detected data errors."""
import os

import numpy as np
import pytest
import torch

import workloads as WL
from oracle import cpp as C
from tests.helpers import masks_from_nbr

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    import sparse_voxel_conv_b200 as S
    return S


@pytest.fixture(params=["auto", "direct", "brick", "hash"])
def kind(request, monkeypatch):
    """auto: the library's choice (the direct table for small or dense volumes,
    the brick table for sparser ones, the hash table beyond both); direct /
    brick / hash: that table wherever it fits (testing knob SUBM3D_MAP_KIND)."""
    if request.param == "auto":
        monkeypatch.delenv("SUBM3D_MAP_KIND", raising=False)
    else:
        monkeypatch.setenv("SUBM3D_MAP_KIND", request.param)
    return request.param


def _gpu_map(S, coords, grid, batch):
    """The GPU map, and its tile masks as whole unsigned 32-bit words: compared
    with the oracle's 27-bit masks, the five high bits must be zero too."""
    h = S.build_map(torch.from_numpy(np.ascontiguousarray(coords)).cuda(), grid, batch)
    words = S.tile_mask_tensor(h).cpu().numpy().view(np.uint32).astype(np.int64)
    return h, h.nbr.cpu().numpy(), words


@pytest.mark.parametrize("name", ["tiny", "shell", "headline", "dense", "batched"])
def test_map_bit_exact(S, kind, name):
    wl = WL.make_workload(name)
    h, nbr, masks = _gpu_map(S, wl.coords, wl.grid_dim, wl.batch)
    ref = C.build_map(wl.coords, wl.grid_dim, wl.batch)
    assert nbr.shape == ref.shape
    assert np.array_equal(nbr, ref)
    assert np.array_equal(masks, masks_from_nbr(ref))


@pytest.mark.parametrize("name,seed", [("shell", 1), ("headline", 2), ("batched", 3)])
def test_map_bit_exact_random_row_order(S, kind, name, seed):
    wl = WL.make_workload(name)
    c = wl.coords[WL.permute_rows(wl.n, seed)]
    _, nbr, masks = _gpu_map(S, c, wl.grid_dim, wl.batch)
    ref = C.build_map(c, wl.grid_dim, wl.batch)
    assert np.array_equal(nbr, ref)
    assert np.array_equal(masks, masks_from_nbr(ref))


@pytest.mark.parametrize("grid,batch,shift", [(2048, 1, 1900), (64, 6, 0), (65535, 9, 65500)])
def test_map_wide_keys(S, kind, grid, batch, shift):
    # batch > 4 or grid_dim > 1024 takes the 64-bit key form
    rng = np.random.default_rng(grid + batch)
    parts = []
    for b in range(batch):
        c = WL.tiny_coords(seed=b)
        c[:, 0] = b
        c[:, 1:] += shift
        parts.append(c)
    c = np.concatenate(parts)[WL.permute_rows(sum(len(p) for p in parts), 4)]
    del rng
    _, nbr, masks = _gpu_map(S, c, grid, batch)
    ref = C.build_map(c, grid, batch)
    assert np.array_equal(nbr, ref)
    assert np.array_equal(masks, masks_from_nbr(ref))


def test_map_table_choice(S, monkeypatch):
    """The table each set gets (subm3d_map_table): direct for the headline and
    the dense sets (small or dense volumes), brick for the decoder-stack set (60
    cells per voxel); the testing knob forces the hash table."""
    A = S._abi
    monkeypatch.delenv("SUBM3D_MAP_KIND", raising=False)
    want = {"headline": A.SUBM3D_TABLE_DIRECT, "dense": A.SUBM3D_TABLE_DIRECT,
            "batched": A.SUBM3D_TABLE_BRICK}
    for name, table in want.items():
        wl = WL.make_workload(name)
        h = S.build_map(torch.from_numpy(wl.coords).cuda(), wl.grid_dim, wl.batch)
        assert A.subm3d_map_table(h) == table, name
    monkeypatch.setenv("SUBM3D_MAP_KIND", "hash")
    wl = WL.make_workload("shell")
    h = S.build_map(torch.from_numpy(wl.coords).cuda(), wl.grid_dim, wl.batch)
    assert A.subm3d_map_table(h) == A.SUBM3D_TABLE_HASH


@pytest.fixture(scope="module")
def large_sparse():
    """Two 512^3 grids of large shells: 615,658 voxels, 441 cells per voxel, so
    the direct table (1.09 GB) exceeds the budget and the library's choice is the
    brick table (a 17 MB directory)."""
    c = WL.batched_coords(batch=2, grid=512, min_voxels=120_000, seed0=7, r_lo=40.0, r_hi=120.0)
    return c, C.build_map(c, 512, 2)


def test_map_large_sparse_volume(S, kind, large_sparse):
    c, ref = large_sparse
    _, nbr, masks = _gpu_map(S, c, 512, 2)
    assert np.array_equal(nbr, ref)
    assert np.array_equal(masks, masks_from_nbr(ref))


def test_map_edge_sizes(S, kind):
    for c in (np.zeros((0, 4), np.int32), np.array([[0, 3, 3, 3]], np.int32),
              WL.dense_coords(5)[:129], WL.dense_coords(2)):
        grid = 5
        h, nbr, masks = _gpu_map(S, c, grid, 1)
        ref = C.build_map(c, grid, 1)
        assert np.array_equal(nbr, ref)
        assert np.array_equal(masks, masks_from_nbr(ref))


def test_map_grid_boundary_no_wrap(S, kind):
    # voxels on opposite faces of the grid are not neighbours (no wrap-around)
    g = 8
    c = np.array([[0, 0, 0, 0], [0, g - 1, 0, 0], [0, 0, g - 1, 0], [0, 0, 0, g - 1],
                  [0, g - 1, g - 1, g - 1]], np.int32)
    _, nbr, _ = _gpu_map(S, c, g, 1)
    assert np.array_equal(nbr, C.build_map(c, g, 1))
    assert ((nbr >= 0).sum(axis=1) == 1).all()


@pytest.mark.parametrize("bad,status", [([0, 0, 0, 16], 2), ([0, -1, 3, 3], 2), ([1, 1, 1, 1], 2),
                                        (None, 3)])
def test_map_data_errors(S, kind, bad, status):
    base = WL.tiny_coords()
    extra = base[700:701] if bad is None else np.array([bad], np.int32)  # None: a duplicate
    c = np.concatenate([base, extra])
    with pytest.raises(S.Subm3dError) as e:
        S.build_map(torch.from_numpy(c).cuda(), 16, 1)
    assert e.value.status == status


def test_map_table_full_is_reported_not_spun(S, monkeypatch):
    monkeypatch.setenv("SUBM3D_TABLE_CAPACITY", "64")
    c = torch.from_numpy(WL.tiny_coords()).cuda()
    with pytest.raises(S.Subm3dError) as e:
        S.build_map(c, 16, 1)
    assert e.value.status == 4
    monkeypatch.delenv("SUBM3D_TABLE_CAPACITY")
    h = S.build_map(c, 16, 1)
    assert np.array_equal(h.nbr.cpu().numpy(), C.build_map(WL.tiny_coords(), 16, 1))


def test_map_async_status_and_reuse(S):
    # build twice into the same buffers; the second build fully overwrites the first
    c1 = torch.from_numpy(WL.shell_coords()).cuda()
    h1 = S.build_map(c1, 64, 1, check=False)
    assert S.map_status(h1) == 0
    c2 = torch.from_numpy(WL.tiny_coords()).cuda()
    nbr = torch.empty((c2.shape[0], 27), dtype=torch.int32, device="cuda")
    h2 = S.build_map(c2, 16, 1, nbr=nbr, workspace=h1.workspace)
    assert np.array_equal(h2.nbr.cpu().numpy(), C.build_map(WL.tiny_coords(), 16, 1))


def _check_run_layout(S, coords, grid, batch):
    """Every voxel sits at one position p of the x-run layout, its run's pads
    beside it, and for each of its 27 offsets (dz, dy, dx) the E index entry of
    (tile, dz-dy) at row p+dx is its neighbour nbr[v][k] -- the property the
    x-run forward relies on.  Every other entry of the used tiles is empty or
    a valid row, so no gather can leave the feature array."""
    coords = np.ascontiguousarray(coords, dtype=np.int32)
    h = S.build_map(torch.from_numpy(coords).cuda(), grid, batch)
    pos, et, hdr = (t.cpu().numpy() for t in S.run_layout_tensors(h))
    ref = C.build_map(coords, grid, batch)
    n = coords.shape[0]
    c = coords.astype(np.int64)
    same = (c[1:, 0] == c[:-1, 0]) & (c[1:, 1] == c[:-1, 1]) & (c[1:, 2] == c[:-1, 2]) & \
        (c[1:, 3] == c[:-1, 3] + 1)
    starts = np.concatenate([[True], ~same])
    ends = np.concatenate([~same, [True]])
    runs = int(starts.sum())
    positions = n + 2 * runs
    assert hdr[0] == runs and hdr[2] == positions and hdr[1] == (positions + 255) // 256
    assert pos.shape[0] == 256 * hdr[1] and et.shape == (9, 256 * hdr[1] + 2)
    voxel_pos = np.nonzero((pos >= 0) & ((pos & 3) == 0))[0]
    assert np.array_equal(pos[voxel_pos] >> 2, np.arange(n))      # every row once, in order
    assert np.array_equal(voxel_pos, np.arange(n) + 2 * np.cumsum(starts))
    left = np.nonzero((pos >= 0) & ((pos & 3) == 1))[0]
    assert np.array_equal(left + 1, voxel_pos[starts]) and np.array_equal(pos[left] >> 2,
                                                                           np.nonzero(starts)[0])
    right = np.nonzero((pos >= 0) & ((pos & 3) == 2))[0]
    inside = voxel_pos[ends] + 1 < pos.shape[0]          # the last right pad may sit past the tiles
    assert np.array_equal(right, (voxel_pos[ends] + 1)[inside])
    assert pos[0] == -1 and (pos[positions + 1:] == -1).all()
    assert ((pos >= 0) | (pos == -1)).all()
    assert (et >= -1).all() and (et < n).all()   # every entry a tile reads is written
    for k in range(27):
        dzdy, dx = k // 3, k % 3 - 1
        got = et[dzdy, voxel_pos + dx + 1]
        assert np.array_equal(got, ref[:, k]), f"offset {k}"
    # E rows that are not a voxel's neighbour row: positions -1 and 0, and the
    # tail after the last right pad, are empty
    assert (et[:, :2] == -1).all() and (et[:, positions + 2:] == -1).all()


@pytest.mark.parametrize("name", ["tiny", "shell", "headline", "batched"])
def test_run_layout_invariant(S, kind, name):
    wl = WL.make_workload(name)
    _check_run_layout(S, wl.coords, wl.grid_dim, wl.batch)


def test_run_layout_edges(S, kind):
    """Tiny maps, a last tile ending on a position-tile boundary (one run of
    252 to 255 voxels puts the last right pad at 255, 256 or beyond), and
    random row order (short runs, many pads)."""
    rng = np.random.default_rng(17)
    for n in (1, 2, 127, 128, 129, 300):
        cells = rng.choice(8 ** 3, n, replace=False)
        zyx = np.stack(np.unravel_index(np.sort(cells), (8, 8, 8)), 1)
        _check_run_layout(S, np.concatenate([np.zeros((n, 1), np.int64), zyx], 1), 8, 1)
    for length in (252, 253, 254, 255, 510, 511):
        line = np.array([[0, 3, 5, x] for x in range(length)])
        _check_run_layout(S, line, 512, 1)
    wl = WL.make_workload("shell")
    _check_run_layout(S, wl.coords[WL.permute_rows(wl.n, 5)], wl.grid_dim, wl.batch)
