"""Pins for the resample oracle (subdivide, masked upsample, channel2spatial,
spatial2channel, downsample): hand-worked cases from the pages' definitions,
round trips, and numpy's own unique / reduction routines.  CPU only."""
import numpy as np
import pytest

from oracle import resample_oracle as R


def _rand_set(rng, n, grid, batch=2):
    cells = rng.choice(batch * grid ** 3, size=n, replace=False)
    b, rem = np.divmod(cells, grid ** 3)
    z, rem = np.divmod(rem, grid * grid)
    y, x = np.divmod(rem, grid)
    return np.stack([b, z, y, x], 1).astype(np.int32)


def test_subdivide_hand_worked():
    # voxel (b=1, z=2, y=0, x=5): children 2*coord + (dz, dy, dx), x fastest (C order)
    c = np.array([[1, 2, 0, 5]], np.int32)
    f = np.array([[3.0, -1.0]])
    oc, of = R.subdivide(c, f)
    expect = [(1, 4 + dz, 0 + dy, 10 + dx) for dz in (0, 1) for dy in (0, 1) for dx in (0, 1)]
    assert [tuple(r) for r in oc] == expect
    assert np.array_equal(of, np.repeat(f, 8, axis=0))


def test_upsample_mask_decodes_axis0_fastest():
    # mask bit s -> offsets (s % 2, s // 2 % 2, s // 4 % 2) along (z, y, x); slot 1 is +z,
    # slot 4 is +x -- the reverse of subdivide's C order, where slot 1 is +x
    c = np.array([[0, 3, 3, 3], [0, 7, 7, 7]], np.int32)
    f = np.array([[1.0], [2.0]])
    mask = np.zeros((2, 8), np.uint8)
    mask[0, [1, 4, 7]] = 1          # voxel 0: +z, +x, +z+y+x
    oc, of = R.upsample(c, f, mask)  # voxel 1 has no flagged child: contributes nothing
    assert [tuple(r) for r in oc] == [(0, 7, 6, 6), (0, 6, 6, 7), (0, 7, 7, 7)]
    assert np.array_equal(of, [[1.0], [1.0], [1.0]])
    sub, _ = R.subdivide(c[:1], f[:1])
    assert tuple(sub[1]) == (0, 6, 6, 7)   # subdivide's slot 1 is +x


def test_channel2spatial_slices_channels():
    c = np.array([[0, 1, 1, 1]], np.int32)
    f = np.arange(16, dtype=np.float64)[None, :]          # 8 children x 2 channels
    oc, of = R.channel2spatial(c, f)
    for s in range(8):
        dz, dy, dx = s & 1, (s >> 1) & 1, (s >> 2) & 1
        assert tuple(oc[s]) == (0, 2 + dz, 2 + dy, 2 + dx)
        assert np.array_equal(of[s], [2 * s, 2 * s + 1])


def test_round_trips_and_all_ones_mask():
    rng = np.random.default_rng(5)
    c = _rand_set(rng, 200, 9)
    order = np.lexsort(c.T[::-1])                 # raster order of the parents
    f = rng.standard_normal((200, 3))
    sub_c, sub_f = R.subdivide(c, f)
    for mode in ("max", "mean"):
        pc, pf = R.downsample(sub_c, sub_f, mode)
        assert np.array_equal(pc, c[order]) and np.allclose(pf, f[order], rtol=0, atol=1e-15)
    f8 = rng.standard_normal((200, 24))
    c2s_c, c2s_f = R.channel2spatial(c, f8)
    pc, pf = R.spatial2channel(c2s_c, c2s_f)
    assert np.array_equal(pc, c[order]) and np.array_equal(pf, f8[order])
    up_c, up_f = R.upsample(c, f, np.ones((200, 8), np.uint8))
    key = lambda a: np.lexsort(a.T[::-1])
    assert np.array_equal(up_c[key(up_c)], sub_c[key(sub_c)])
    assert np.array_equal(up_f[key(up_c)], sub_f[key(sub_c)])


def test_downsample_against_numpy_unique_and_reductions():
    rng = np.random.default_rng(6)
    c = _rand_set(rng, 500, 10)
    f = rng.standard_normal((500, 4))
    par = c.astype(np.int64).copy()
    par[:, 1:] //= 2
    uniq, inv = np.unique(par, axis=0, return_inverse=True)   # lexicographic = raster order
    inv = inv.reshape(-1)
    mx = np.full((uniq.shape[0], 4), -np.inf)
    np.maximum.at(mx, inv, f)
    sm = np.zeros((uniq.shape[0], 4))
    np.add.at(sm, inv, f)
    cnt = np.bincount(inv, minlength=uniq.shape[0])[:, None]
    pc, pmax = R.downsample(c, f, "max")
    _, pmean = R.downsample(c, f, "mean")
    assert np.array_equal(pc, uniq) and np.array_equal(pmax, mx)
    assert np.allclose(pmean, sm / cnt, rtol=1e-15, atol=1e-15)
    assert not np.allclose(pmax, pmean)          # the two modes differ
    # spatial2channel: each child's row lands in its parent's slot, zeros elsewhere
    pc2, s2c = R.spatial2channel(c, f)
    assert np.array_equal(pc2, uniq)
    r = c[:, 1:] % 2
    slot = r[:, 0] + 2 * r[:, 1] + 4 * r[:, 2]
    filled = np.zeros((uniq.shape[0], 8), bool)
    filled[inv, slot] = True
    for i in range(500):
        assert np.array_equal(s2c[inv[i], 4 * slot[i]:4 * slot[i] + 4], f[i])
    assert np.all(s2c.reshape(-1, 8, 4)[~filled] == 0)


def test_downsample_rejects_unknown_mode():
    with pytest.raises(ValueError):
        R.downsample(np.zeros((1, 4), np.int32), np.zeros((1, 1)), "sum")


def test_batches_never_share_a_parent():
    # the same spatial child in two batch elements: two parents, one per element
    c = np.array([[0, 2, 3, 4], [1, 2, 3, 4], [1, 3, 3, 5]], np.int32)
    f = np.array([[1.0], [5.0], [7.0]])
    pc, pmax = R.downsample(c, f, "max")
    assert [tuple(r) for r in pc] == [(0, 1, 1, 2), (1, 1, 1, 2)]
    assert np.array_equal(pmax, [[1.0], [7.0]])
    _, pmean = R.downsample(c, f, "mean")
    assert np.array_equal(pmean, [[1.0], [6.0]])
    _, s2c = R.spatial2channel(c, f)
    # child (2,3,4) sits in slot 0 + 2*1 + 4*0 = 2; child (3,3,5) in 1 + 2 + 4 = 7
    assert s2c[0, 2] == 1.0 and s2c[1, 2] == 5.0 and s2c[1, 7] == 7.0
    assert np.count_nonzero(s2c) == 3


def test_empty_and_all_zero_mask():
    c = np.zeros((0, 4), np.int32)
    oc, of = R.subdivide(c, np.zeros((0, 3)))
    assert oc.shape == (0, 4) and of.shape == (0, 3)
    c = np.array([[0, 1, 2, 3], [0, 4, 4, 4]], np.int32)
    oc, of = R.upsample(c, np.ones((2, 3)), np.zeros((2, 8), np.uint8))
    assert oc.shape[0] == 0 and of.shape == (0, 3)
    oc, of = R.channel2spatial(c, np.ones((2, 16)), np.zeros((2, 8), np.uint8))
    assert oc.shape[0] == 0 and of.shape == (0, 2)
