"""A seeded random sweep through the map build, the forward kernels, the
gradients and the resolution changes.

Small random coordinate sets -- several grid sizes (odd ones included), batch
sizes, densities and row orders (raster, permuted, reversed) -- with channel
pairs that reach every forward kernel: the x-run bf16 kernel (Cin >= 48, whole
and partial 64-channel chunks, Cout below, at and above 128), the per-offset
bf16 kernel (Cin < 48) and the fp32 kernel (any size), some with a bias and a
residual in the fused epilogue.  nbr must equal the
oracle's bit for bit and every output row must meet the path's bar against the
oracle (bf16 2e-2, fp32 1e-5 of |ref| + rms ref).
"""
import numpy as np
import pytest
import torch

import workloads as WL
from oracle import cpp as C
from tests.helpers import RTOL_BF16, RTOL_F32, assert_close

pytestmark = pytest.mark.gpu

_CHANNELS = [(16, 16, "bf16"), (32, 48, "bf16"), (48, 32, "bf16"), (64, 64, "bf16"),
             (80, 144, "bf16"), (128, 128, "bf16"), (96, 16, "bf16"), (8, 24, "f32"),
             (20, 12, "f32")]


def _cases(count=45, seed=2024):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(count):
        grid = int(rng.choice([5, 9, 17, 24, 33]))
        batch = int(rng.integers(1, 4))
        p = float(rng.choice([0.03, 0.15, 0.4]))
        order = ["raster", "permuted", "reversed"][i % 3]
        cin, cout, dtype = _CHANNELS[i % len(_CHANNELS)]
        act = [None, "gelu", "silu"][int(rng.integers(0, 3))]
        flip = bool(rng.integers(0, 2))
        out.append((1000 + i, grid, batch, p, order, cin, cout, dtype, act, flip))
    return out


@pytest.fixture(scope="module")
def S():
    import sparse_voxel_conv_b200 as S
    return S


def _case_id(c):
    return f"s{c[0]}-g{c[1]}b{c[2]}-{c[4]}-{c[5]}x{c[6]}{c[7]}"


@pytest.mark.parametrize("case", _cases(), ids=_case_id)
def test_random_sets_against_oracle(S, case):
    seed, grid, batch, p, order, cin, cout, dtype, act, flip = case
    coords, n = _case_inputs(case)
    x = WL.make_features(n, cin, seed + 1)
    w = WL.make_weight(cout, cin, seed + 2)
    if dtype == "bf16":
        x, w = WL.to_bf16_values(x), WL.to_bf16_values(w)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    # the fused epilogue's inputs on some of the sets: a bias on odd seeds, a
    # residual on every third (fp32 staging in the bf16 kernels then)
    bias = WL.make_features(1, cout, seed + 9)[0] if seed % 2 else None
    res = WL.make_features(n, cout, seed + 10) if seed % 3 == 0 else None
    if dtype == "bf16":
        bias = None if bias is None else WL.to_bf16_values(bias)
        res = None if res is None else WL.to_bf16_values(res)
    t = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda().to(tdt)

    h = S.build_map(torch.from_numpy(coords).cuda(), grid, batch)
    want_nbr = C.build_map(coords, grid, batch)
    assert np.array_equal(h.nbr.cpu().numpy(), want_nbr), case

    y = S.forward(h, t(x), t(w), flip=flip, act=act, bias=t(bias), residual=t(res))
    torch.cuda.synchronize()
    assert S._abi.subm3d_device_status() == 0
    ref = C.forward(want_nbr, np.asarray(x, np.float64), np.asarray(w, np.float64), flip=flip,
                    act=act, round_to_bf16=(dtype == "bf16"),
                    bias=None if bias is None else np.asarray(bias, np.float64),
                    residual=None if res is None else np.asarray(res, np.float64))
    assert_close(y.float().cpu().numpy(), ref, RTOL_BF16 if dtype == "bf16" else RTOL_F32,
                 f"random set {case}")


RTOL_WGRAD = 1e-4  # fp32 weight gradient: fp32 atomics over up to N terms per entry


def _case_inputs(case):
    seed, grid, batch, p, order, cin, cout, dtype, act, flip = case
    coords = WL.random_coords(seed, grid, batch, p)
    n = coords.shape[0]
    if order == "permuted":
        coords = coords[WL.permute_rows(n, seed)]
    elif order == "reversed":
        coords = coords[::-1]
    return np.ascontiguousarray(coords), n


@pytest.mark.parametrize("case", _cases(count=18, seed=77), ids=_case_id)
def test_random_sets_gradients_against_oracle(S, case):
    """Input and weight gradients on random sets (the input gradient is a forward
    Cout -> Cin, so the channel pairs reach the x-run and per-offset kernels in
    that direction too)."""
    seed, grid, batch, p, order, cin, cout, dtype, act, flip = case
    coords, n = _case_inputs(case)
    x = WL.make_features(n, cin, seed + 3)
    w = WL.make_weight(cout, cin, seed + 4)
    dy = WL.make_features(n, cout, seed + 5)
    if dtype == "bf16":
        x, w, dy = WL.to_bf16_values(x), WL.to_bf16_values(w), WL.to_bf16_values(dy)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(tdt)
    h = S.build_map(torch.from_numpy(coords).cuda(), grid, batch)
    dx = S.backward_data(h, t(dy), t(w), flip=flip)
    dw = S.backward_weight(h, t(x), t(dy), flip=flip)
    torch.cuda.synchronize()
    assert S._abi.subm3d_device_status() == 0
    nbr = C.build_map(coords, grid, batch)
    ref_dx = C.backward_data(nbr, np.asarray(dy, np.float64), np.asarray(w, np.float64), flip=flip)
    if dtype == "bf16":
        ref_dx = C.round_bf16(ref_dx)
    assert_close(dx.float().cpu().numpy(), ref_dx, RTOL_BF16 if dtype == "bf16" else RTOL_F32,
                 f"input gradient {case}")
    ref_dw = C.backward_weight(nbr, np.asarray(x, np.float64), np.asarray(dy, np.float64),
                               flip=flip)
    assert_close(dw.cpu().numpy(), ref_dw, RTOL_WGRAD, f"weight gradient {case}")


@pytest.mark.parametrize("case", _cases(count=12, seed=99),
                         ids=lambda c: f"s{c[0]}-g{c[1]}b{c[2]}-{c[4]}-{c[7]}")
def test_random_sets_resampling_against_oracle(S, case):
    """Subdivide, max / mean downsample and spatial2channel on random sets, every
    row against the resampling oracle."""
    from oracle import resample_oracle as R
    seed, grid, batch, p, order, cin, cout, dtype, act, flip = case
    coords, n = _case_inputs(case)
    # the pooling oracle and kernels take raster-ordered parents from any child order
    f = WL.make_features(n, cin, seed + 6)
    if dtype == "bf16":
        f = WL.to_bf16_values(f)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    st = S.SparseTensor(torch.from_numpy(coords).cuda(), torch.from_numpy(f).cuda().to(tdt),
                        grid_dim=grid, batch=batch)
    npf = lambda t: t.float().cpu().numpy() if t.is_floating_point() else t.cpu().numpy()
    fine = S.subdivide(st)
    rc, rf = R.subdivide(coords, f)
    assert np.array_equal(npf(fine.coords), rc) and np.array_equal(npf(fine.feats), rf), case
    for mode in ("max", "mean"):
        out = S.downsample(st, mode)
        rc, rf = R.downsample(coords, f, mode)
        assert np.array_equal(npf(out.coords), rc), (case, mode)
        if mode == "max":
            assert np.array_equal(npf(out.feats), rf.astype(np.float32)), (case, mode)
        else:
            ref = WL.to_bf16_values(rf.astype(np.float32)) if dtype == "bf16" else rf
            assert_close(npf(out.feats), ref, RTOL_BF16 if dtype == "bf16" else RTOL_F32,
                         f"mean pooling {case}")
    out = S.spatial2channel(st)
    rc, rf = R.spatial2channel(coords, f)
    assert np.array_equal(npf(out.coords), rc) and np.array_equal(npf(out.feats), rf), case
    torch.cuda.synchronize()
    assert S._abi.subm3d_device_status() == 0


@pytest.mark.parametrize("kind", ["brick", "hash"])
@pytest.mark.parametrize("case", _cases(count=15, seed=123), ids=_case_id)
def test_random_sets_table_kinds(S, case, kind, monkeypatch):
    """The brick and hash tables (forced with the testing knob SUBM3D_MAP_KIND)
    give the oracle's nbr, and the forward on their maps equals, bit for bit,
    the forward on the direct table's map: the map, and the x-run layout built
    from it, do not depend on the table."""
    seed, grid, batch, p, order, cin, cout, dtype, act, flip = case
    coords, n = _case_inputs(case)
    x = WL.make_features(n, cin, seed + 7)
    w = WL.make_weight(cout, cin, seed + 8)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    xt = torch.from_numpy(x).cuda().to(tdt)
    wt = torch.from_numpy(w).cuda().to(tdt)
    ct = torch.from_numpy(coords).cuda()
    monkeypatch.delenv("SUBM3D_MAP_KIND", raising=False)
    h_direct = S.build_map(ct, grid, batch)
    y_direct = S.forward(h_direct, xt, wt, flip=flip, act=act)
    monkeypatch.setenv("SUBM3D_MAP_KIND", kind)
    h = S.build_map(ct, grid, batch)
    y = S.forward(h, xt, wt, flip=flip, act=act)
    torch.cuda.synchronize()
    assert S._abi.subm3d_device_status() == 0
    want = {"brick": S._abi.SUBM3D_TABLE_BRICK, "hash": S._abi.SUBM3D_TABLE_HASH}[kind]
    assert S._abi.subm3d_map_table(h) == want
    assert np.array_equal(h.nbr.cpu().numpy(), C.build_map(coords, grid, batch)), case
    assert torch.equal(y, y_direct), case


@pytest.mark.parametrize("kind", ["auto", "brick", "hash"])
@pytest.mark.parametrize("seed,grid,batch,p", [(2001, 7, 5, 0.3), (2002, 12, 6, 0.1),
                                              (2003, 20, 7, 0.05)])
def test_random_sets_wide_keys(S, seed, grid, batch, p, kind, monkeypatch):
    """Batches above 4 take the wide (64-bit) keys in the hash table and more
    grids in the direct and brick tables: nbr against the oracle, in permuted
    row order, and the x-run forward against the oracle."""
    if kind == "auto":
        monkeypatch.delenv("SUBM3D_MAP_KIND", raising=False)
    else:
        monkeypatch.setenv("SUBM3D_MAP_KIND", kind)
    coords = WL.random_coords(seed, grid, batch, p)
    n = coords.shape[0]
    coords = np.ascontiguousarray(coords[WL.permute_rows(n, seed)])
    h = S.build_map(torch.from_numpy(coords).cuda(), grid, batch)
    nbr = C.build_map(coords, grid, batch)
    assert np.array_equal(h.nbr.cpu().numpy(), nbr)
    x = WL.to_bf16_values(WL.make_features(n, 64, seed + 1))
    w = WL.to_bf16_values(WL.make_weight(64, 64, seed + 2))
    y = S.forward(h, torch.from_numpy(x).cuda().to(torch.bfloat16),
                  torch.from_numpy(w).cuda().to(torch.bfloat16))
    torch.cuda.synchronize()
    assert S._abi.subm3d_device_status() == 0
    ref = C.forward(nbr, np.asarray(x, np.float64), np.asarray(w, np.float64), round_to_bf16=True)
    assert_close(y.float().cpu().numpy(), ref, RTOL_BF16, f"wide keys {kind} b={batch}")
