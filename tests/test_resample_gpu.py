"""Resolution changes on the GPU (through the C ABI) vs the resample oracle.

Coordinates, subdivide / upsample / channel2spatial / spatial2channel features
and max pooling are copies or exact selections: compared bit for bit.  Mean
pooling sums at most 8 children in fp32 (one rounding of a bf16 output): bar
1e-5 (fp32) / 2e-2 (bf16) of |ref| + rms(ref).
"""
import numpy as np
import pytest
import torch

import workloads as WL
from oracle import resample_oracle as R
from tests.helpers import RTOL_BF16, RTOL_F32, assert_close

pytestmark = pytest.mark.gpu
DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


@pytest.fixture(scope="module")
def S():
    import sparse_voxel_conv_b200 as S
    return S


@pytest.fixture(params=["auto", "brick", "hash"])
def kind(request, monkeypatch):
    if request.param == "auto":
        monkeypatch.delenv("SUBM3D_MAP_KIND", raising=False)
    else:
        monkeypatch.setenv("SUBM3D_MAP_KIND", request.param)
    return request.param


def _rand_set(n, grid, batch, seed):
    rng = np.random.default_rng(seed)
    cells = rng.choice(batch * grid ** 3, size=n, replace=False)
    b, rem = np.divmod(cells, grid ** 3)
    z, rem = np.divmod(rem, grid * grid)
    y, x = np.divmod(rem, grid)
    return np.stack([b, z, y, x], 1).astype(np.int32)


def _st(S, coords, feats, grid, batch, dtype):
    f = torch.from_numpy(np.ascontiguousarray(feats, np.float32)).cuda().to(DTYPES[dtype])
    return S.SparseTensor(torch.from_numpy(coords).cuda(), f, grid, batch)


def _np(t):
    return t.float().cpu().numpy() if t.is_floating_point() else t.cpu().numpy()


def _feats(n, c, dtype, seed):
    f = WL.make_features(n, c, seed)
    return WL.to_bf16_values(f) if dtype == "bf16" else f


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_subdivide_exact(S, dtype):
    c = _rand_set(3000, 20, 2, 1)
    f = _feats(3000, 24, dtype, 2)
    out = S.subdivide(_st(S, c, f, 20, 2, dtype))
    rc, rf = R.subdivide(c, f)
    assert out.grid_dim == 40
    assert np.array_equal(_np(out.coords), rc) and np.array_equal(_np(out.feats), rf)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_upsample_exact(S, dtype):
    c = _rand_set(2500, 16, 1, 3)
    f = _feats(2500, 16, dtype, 4)
    rng = np.random.default_rng(5)
    mask = (rng.random((2500, 8)) < 0.4).astype(np.uint8)
    mask[:50] = 0                                  # voxels with no flagged child
    out = S.upsample(_st(S, c, f, 16, 1, dtype), torch.from_numpy(mask).cuda())
    rc, rf = R.upsample(c, f, mask)
    assert out.coords.shape[0] == int(mask.sum())
    assert np.array_equal(_np(out.coords), rc) and np.array_equal(_np(out.feats), rf)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("masked", [False, True])
def test_channel2spatial_exact(S, dtype, masked):
    c = _rand_set(1800, 14, 3, 6)
    f = _feats(1800, 8 * 6, dtype, 7)              # 6 channels per child (12 B bf16 rows)
    mask = (np.random.default_rng(8).random((1800, 8)) < 0.5).astype(np.uint8) if masked else None
    out = S.channel2spatial(_st(S, c, f, 14, 3, dtype),
                            None if mask is None else torch.from_numpy(mask).cuda())
    rc, rf = R.channel2spatial(c, f, mask)
    assert np.array_equal(_np(out.coords), rc) and np.array_equal(_np(out.feats), rf)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_pooling_matches_oracle(S, kind, dtype):
    c = _rand_set(4000, 17, 2, 9)                  # odd grid: parents on the ragged edge too
    f = _feats(4000, 20, dtype, 10)
    st = _st(S, c, f, 17, 2, dtype)
    for mode in ("max", "mean"):
        out = S.downsample(st, mode)
        rc, rf = R.downsample(c, f, mode)
        assert out.grid_dim == 9
        assert np.array_equal(_np(out.coords), rc), mode
        if mode == "max":                          # a selection: exact
            assert np.array_equal(_np(out.feats), rf.astype(np.float32)), mode
        else:
            ref = WL.to_bf16_values(rf.astype(np.float32)) if dtype == "bf16" else rf
            assert_close(_np(out.feats), ref, RTOL_BF16 if dtype == "bf16" else RTOL_F32, mode)
    out = S.spatial2channel(st)
    rc, rf = R.spatial2channel(c, f)
    assert np.array_equal(_np(out.coords), rc) and np.array_equal(_np(out.feats), rf)
    assert list(st.cache) == ["subm0"]             # one map of the fine set, built once


def test_round_trips(S):
    wl = WL.make_workload("shell")
    f = _feats(wl.n, 16, "bf16", 11)
    st = _st(S, wl.coords, f, wl.grid_dim, 1, "bf16")
    order = np.lexsort(wl.coords.T[::-1])
    for mode in ("max", "mean"):
        back = S.downsample(S.subdivide(st), mode)
        assert np.array_equal(_np(back.coords), wl.coords[order])
        assert np.array_equal(_np(back.feats), f[order])
    f8 = _feats(wl.n, 64, "bf16", 12)
    st8 = _st(S, wl.coords, f8, wl.grid_dim, 1, "bf16")
    back = S.spatial2channel(S.channel2spatial(st8))
    assert np.array_equal(_np(back.coords), wl.coords[order])
    assert np.array_equal(_np(back.feats), f8[order])


def test_empty_and_argument_errors(S):
    st = S.SparseTensor(torch.zeros((0, 4), dtype=torch.int32, device="cuda"),
                        torch.zeros((0, 8), device="cuda"), 8, 1)
    assert S.subdivide(st).coords.shape[0] == 0
    assert S.downsample(st, "mean").coords.shape[0] == 0
    c = _rand_set(10, 4, 1, 13)
    st = _st(S, c, np.zeros((10, 8), np.float32), 4, 1, "f32")
    with pytest.raises(ValueError):
        S.downsample(st, "sum")
    with pytest.raises(ValueError):
        S.upsample(st, torch.zeros((10, 7), dtype=torch.uint8, device="cuda"))
    A = S._abi
    ws = torch.empty(4096, dtype=torch.uint8, device="cuda")
    cnt = __import__("ctypes").c_int64(0)
    # subdivide takes no mask; upsample needs one
    assert A.lib.subm3d_expand(st.coords.data_ptr(), st.feats.data_ptr(), ws.data_ptr(), 10, 8,
                               A.SUBM3D_F32, A.SUBM3D_EXPAND_SUBDIVIDE, ws.data_ptr(),
                               ws.data_ptr(), ws.data_ptr(), 4096,
                               __import__("ctypes").byref(cnt), None) == A.SUBM3D_E_INVALID
    assert A.lib.subm3d_expand(st.coords.data_ptr(), st.feats.data_ptr(), None, 10, 8,
                               A.SUBM3D_F32, A.SUBM3D_EXPAND_UPSAMPLE, ws.data_ptr(),
                               ws.data_ptr(), ws.data_ptr(), 4096,
                               __import__("ctypes").byref(cnt), None) == A.SUBM3D_E_INVALID
