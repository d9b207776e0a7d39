"""Parity at the sizes bench.py times, on the headline set (329,839 voxels,
128^3 grid) with 128 bf16 channels.

The oracle cannot redo these full-size calls in seconds, so each check takes
a property that holds entry by entry:
  * subdivide is per parent: the children of a sample of parents (rows 8i..8i+7
    of the output) must equal the oracle's subdivide of those parents alone;
  * pooling is per parent: the pooled row of a sample of parents must equal the
    oracle's max / mean over those parents' children alone;
  * weight-gradient entry dW[o][k][c] depends on dy[:, o] and x[:, c] only: the
    full 128 -> 128 gradient's rows and columns for a subset of o and c must
    equal the oracle's gradient computed from those columns alone.
"""
import numpy as np
import pytest
import torch

import workloads as WL
from oracle import cpp as C
from oracle import resample_oracle as R
from tests.helpers import RTOL_BF16, assert_close, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    import sparse_voxel_conv_b200 as S
    return S


@pytest.fixture(scope="module")
def headline():
    wl = WL.make_workload("headline")
    f = WL.to_bf16_values(WL.make_features(wl.n, 128, 21))
    return wl, f


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda().to(torch.bfloat16)


def test_subdivide_headline_128ch(S, headline):
    wl, f = headline
    st = S.SparseTensor(torch.from_numpy(wl.coords).cuda(), _bf16(f), wl.grid_dim, 1)
    out = S.subdivide(st)
    assert out.coords.shape[0] == 8 * wl.n and out.grid_dim == 2 * wl.grid_dim
    parents = sample_rows(wl.n, 3000, seed=22)
    rows = (8 * parents[:, None] + np.arange(8)[None, :]).reshape(-1)
    idx = torch.from_numpy(rows).cuda()
    got_c = out.coords.index_select(0, idx).cpu().numpy()
    got_f = out.feats.index_select(0, idx).float().cpu().numpy()
    rc, rf = R.subdivide(wl.coords[parents], f[parents])
    assert np.array_equal(got_c, rc)
    assert np.array_equal(got_f, rf)


@pytest.mark.parametrize("mode", ["max", "mean"])
def test_pooling_headline_children_128ch(S, headline, mode):
    """Mean / max pooling of the subdivided headline set (2.64 M children) back
    to its parents, with random child features so that the reduction matters."""
    wl, _ = headline
    fine_c = R.subdivide(wl.coords, np.zeros((wl.n, 1), np.float32))[0]
    g = torch.Generator(device="cuda").manual_seed(23)
    fine_f = torch.randn((fine_c.shape[0], 128), generator=g, device="cuda").to(torch.bfloat16)
    fine = S.SparseTensor(torch.from_numpy(fine_c).cuda(), fine_f, 2 * wl.grid_dim, 1)
    out = S.downsample(fine, mode)
    # the headline set is in raster order, so parent i is output row i
    assert out.coords.shape[0] == wl.n
    assert np.array_equal(out.coords.cpu().numpy(), wl.coords)
    parents = sample_rows(wl.n, 2000, seed=24)
    rows = (8 * parents[:, None] + np.arange(8)[None, :]).reshape(-1)
    child_f = fine_f.index_select(0, torch.from_numpy(rows).cuda()).float().cpu().numpy()
    rc, rf = R.downsample(fine_c[rows], child_f, mode)
    assert np.array_equal(rc, wl.coords[parents])
    got = out.feats.index_select(0, torch.from_numpy(parents).cuda()).float().cpu().numpy()
    if mode == "max":
        assert np.array_equal(got, rf.astype(np.float32))
    else:
        assert_close(got, WL.to_bf16_values(rf.astype(np.float32)), RTOL_BF16, "mean")


def test_weight_gradient_headline_128x128(S, headline):
    wl, x = headline
    h = S.build_map(torch.from_numpy(wl.coords).cuda(), wl.grid_dim, 1)
    dy = WL.to_bf16_values(WL.make_features(wl.n, 128, 25))
    dw = S.backward_weight(h, _bf16(x), _bf16(dy)).cpu().numpy()   # tcgen05 over the x-run layout
    assert dw.shape == (128, 3, 3, 3, 128)
    osel = np.r_[0:16, 56:72, 112:128]
    csel = np.r_[0:16, 64:80, 120:128]
    nbr = C.build_map(wl.coords, wl.grid_dim, 1)
    ref = C.backward_weight(nbr, x[:, csel].astype(np.float64), dy[:, osel].astype(np.float64))
    got = dw[osel][:, :, :, :, csel]
    scale = np.abs(ref) + np.sqrt(np.mean(ref ** 2))
    assert np.all(np.abs(got - ref) <= 1e-4 * scale), float(np.max(np.abs(got - ref) / scale))
