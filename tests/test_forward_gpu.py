"""Forward on the GPU (through the C ABI) vs the CPU oracle, element by element.

Bars: fp32 path |y-ref| <= 1e-5 (|ref| + rms ref); bf16 path (bf16 inputs,
fp32 accumulation, bf16 output) 2e-2 on the same scale.  The oracle sees the
exact bf16 input values widened to fp64.  Small workloads are compared on
every output; the large ones on the full output where the oracle finishes in
seconds (headline) and on sampled rows otherwise (dense, batched stack).
"""
import numpy as np
import pytest
import torch

import workloads as WL
from oracle import cpp as C
from tests.helpers import RTOL_BF16, RTOL_F32, assert_close, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    import sparse_voxel_conv_b200 as S
    return S


def _run(S, coords, grid, batch, x, w, dtype, flip=False, act=None, use_mask=True):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    h = S.build_map(torch.from_numpy(np.ascontiguousarray(coords)).cuda(), grid, batch)
    xt = torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda().to(tdt)
    wt = torch.from_numpy(np.ascontiguousarray(w, np.float32)).cuda().to(tdt)
    y = S.forward(h, xt, wt, flip=flip, act=act, use_tile_mask=use_mask)
    torch.cuda.synchronize()
    assert S._abi.subm3d_device_status() == 0
    return h, y.float().cpu().numpy()


def _oracle(coords, grid, batch, x, w, flip=False, act=None, bf16_out=False, rows=None):
    nbr = C.build_map(coords, grid, batch)
    return C.forward(nbr, np.asarray(x, np.float64), np.asarray(w, np.float64), flip=flip,
                     act=act, round_to_bf16=bf16_out, rows=rows)


def _inputs(coords, cin, cout, dtype, seed=0):
    x = WL.make_features(coords.shape[0], cin, seed + 1)
    w = WL.make_weight(cout, cin, seed + 2)
    if dtype == "bf16":
        x, w = WL.to_bf16_values(x), WL.to_bf16_values(w)
    return x, w


# ------------------------------------------------------------------ fp32 ----

@pytest.mark.parametrize("flip", [False, True])
@pytest.mark.parametrize("act", [None, "gelu"])
def test_f32_tiny_full(S, flip, act):
    wl = WL.make_workload("tiny")
    x, w = wl.features(), wl.weights()[0]
    _, y = _run(S, wl.coords, 16, 1, x, w, "f32", flip, act)
    assert_close(y, _oracle(wl.coords, 16, 1, x, w, flip, act), RTOL_F32, "tiny f32")


@pytest.mark.parametrize("flip", [False, True])
def test_f32_shell_full(S, flip):
    wl = WL.make_workload("shell")
    x, w = wl.features(), wl.weights()[0]
    _, y = _run(S, wl.coords, 64, 1, x, w, "f32", flip)
    assert_close(y, _oracle(wl.coords, 64, 1, x, w, flip), RTOL_F32, "shell f32")


@pytest.mark.parametrize("cin,cout", [(1, 1), (3, 5), (70, 130), (17, 64)])
def test_f32_odd_shapes(S, cin, cout):
    c = WL.shell_coords()
    x, w = _inputs(c, cin, cout, "f32", seed=cin)
    _, y = _run(S, c, 64, 1, x, w, "f32")
    assert_close(y, _oracle(c, 64, 1, x, w), RTOL_F32, f"f32 {cin}->{cout}")


def test_f32_without_tile_mask(S):
    c = WL.tiny_coords()
    x, w = _inputs(c, 8, 8, "f32")
    _, y = _run(S, c, 16, 1, x, w, "f32", use_mask=False)
    assert_close(y, _oracle(c, 16, 1, x, w), RTOL_F32, "f32 no mask")


def test_f32_headline_full(S):
    # the size bench.py times: 2,577 tiles of 128 rows (the last one 111 rows),
    # 128 -> 128, every output against the oracle
    wl = WL.make_workload("headline")
    x, w = wl.features(), wl.weights()[0]
    _, y = _run(S, wl.coords, 128, 1, x, w, "f32")
    assert_close(y, _oracle(wl.coords, 128, 1, x, w), RTOL_F32, "headline f32")


def test_f32_headline_flip_gelu_sampled(S):
    wl = WL.make_workload("headline")
    x, w = wl.features(), wl.weights()[0]
    _, y = _run(S, wl.coords, 128, 1, x, w, "f32", flip=True, act="gelu")
    rows = sample_rows(wl.n, 4000, seed=3)  # includes the first and the ragged last tiles
    ref = _oracle(wl.coords, 128, 1, x, w, flip=True, act="gelu", rows=rows)
    assert_close(y[rows], ref, RTOL_F32, "headline f32 flip gelu")


# ------------------------------------------------------------------ bf16 ----

@pytest.mark.parametrize("flip", [False, True])
@pytest.mark.parametrize("act", [None, "gelu"])
def test_bf16_shell_full(S, flip, act):
    wl = WL.make_workload("shell_bf16")
    x, w = wl.features(), wl.weights()[0]
    _, y = _run(S, wl.coords, 64, 1, x, w, "bf16", flip, act)
    ref = _oracle(wl.coords, 64, 1, x, w, flip, act, bf16_out=True)
    assert_close(y, ref, RTOL_BF16, "shell bf16")


@pytest.mark.parametrize("cin,cout", [(16, 16), (80, 48), (128, 272), (256, 256), (64, 128),
                                      (32, 512), (192, 80)])
def test_bf16_shapes(S, cin, cout):
    # partial 64-channel chunks, several column blocks, the widest N
    c = WL.shell_coords()
    x, w = _inputs(c, cin, cout, "bf16", seed=cin + cout)
    _, y = _run(S, c, 64, 1, x, w, "bf16")
    assert_close(y, _oracle(c, 64, 1, x, w, bf16_out=True), RTOL_BF16, f"bf16 {cin}->{cout}")


def test_bf16_random_row_order_and_no_mask(S):
    c = WL.shell_coords()[WL.permute_rows(14534, 6)]
    x, w = _inputs(c, 64, 64, "bf16", seed=3)
    ref = _oracle(c, 64, 1, x, w, bf16_out=True)
    for use_mask in (True, False):
        _, y = _run(S, c, 64, 1, x, w, "bf16", use_mask=use_mask)
        assert_close(y, ref, RTOL_BF16, f"bf16 permuted mask={use_mask}")


def test_bf16_edge_sets(S):
    # one voxel; a 129-voxel set (one full tile + a 1-row tail); isolated voxels
    lattice = np.array([(0, z, y, x) for z in range(0, 16, 2) for y in range(0, 16, 2)
                        for x in range(0, 16, 2)], np.int32)
    for c in (np.array([[0, 7, 7, 7]], np.int32), WL.dense_coords(6)[:129], lattice):
        x, w = _inputs(c, 32, 48, "bf16", seed=len(c))
        _, y = _run(S, c, 16, 1, x, w, "bf16")
        assert_close(y, _oracle(c, 16, 1, x, w, bf16_out=True), RTOL_BF16, f"edge n={len(c)}")
    # isolated voxels see only the centre slice
    x, w = _inputs(lattice, 32, 48, "bf16", seed=9)
    _, y = _run(S, lattice, 16, 1, x, w, "bf16")
    centre = np.asarray(x, np.float64) @ np.asarray(w, np.float64)[:, 1, 1, 1, :].T
    assert_close(y, C.round_bf16(centre), RTOL_BF16, "isolated")


@pytest.mark.parametrize("flip", [False, True])
def test_bf16_runs_edge_layouts(S, flip):
    """The x-run kernel (Cin % 64 == 0) on the layouts whose edges matter: one
    voxel; isolated voxels (every voxel its own run); 129 voxels of a dense
    block; runs of 255 and 511 voxels along x (the last right pad lands on or
    past a 256-position tile boundary, read through the next tile's edge rows);
    random sets in 8^3."""
    rng = np.random.default_rng(23)
    lattice = np.array([(0, z, y, x) for z in range(0, 16, 2) for y in range(0, 16, 2)
                        for x in range(0, 16, 2)], np.int32)
    sets = [(np.array([[0, 7, 7, 7]], np.int32), 16), (lattice, 16),
            (WL.dense_coords(6)[:129], 16)]
    for length in (255, 511):
        sets.append((np.array([[0, 3, 5, x] for x in range(length)] +
                              [[0, 4, 5, x] for x in range(0, length, 3)], np.int32), 512))
    for n in (2, 300):
        cells = np.sort(rng.choice(8 ** 3, n, replace=False))
        zyx = np.stack(np.unravel_index(cells, (8, 8, 8)), 1)
        sets.append((np.concatenate([np.zeros((n, 1), np.int64), zyx], 1).astype(np.int32), 8))
    for c, grid in sets:
        x, w = _inputs(c, 64, 48, "bf16", seed=len(c))
        _, y = _run(S, c, grid, 1, x, w, "bf16", flip=flip)
        ref = _oracle(c, grid, 1, x, w, flip=flip, bf16_out=True)
        assert_close(y, ref, RTOL_BF16, f"x-run n={len(c)} flip={flip}")


def test_bf16_empty(S):
    c = np.zeros((0, 4), np.int32)
    h = S.build_map(torch.from_numpy(c).cuda(), 8, 1)
    y = S.forward(h, torch.zeros((0, 16), dtype=torch.bfloat16, device="cuda"),
                  torch.zeros((16, 3, 3, 3, 16), dtype=torch.bfloat16, device="cuda"))
    assert y.shape == (0, 16)


def test_bf16_headline_full(S):
    wl = WL.make_workload("headline")
    x, w = wl.features(), wl.weights()[0]
    _, y = _run(S, wl.coords, 128, 1, x, w, "bf16")
    assert_close(y, _oracle(wl.coords, 128, 1, x, w, bf16_out=True), RTOL_BF16, "headline")


def test_bf16_headline_flip_sampled(S):
    wl = WL.make_workload("headline")
    x, w = wl.features(), wl.weights()[0]
    _, y = _run(S, wl.coords, 128, 1, x, w, "bf16", flip=True)
    rows = sample_rows(wl.n, 4000, seed=1)
    ref = _oracle(wl.coords, 128, 1, x, w, flip=True, bf16_out=True, rows=rows)
    assert_close(y[rows], ref, RTOL_BF16, "headline flip")


@pytest.mark.parametrize("cin,cout", [(80, 128), (48, 48)])
def test_bf16_headline_partial_chunk_sampled(S, cin, cout):
    # the x-run kernel with a partial last 64-channel chunk, over all 1,567 tiles
    wl = WL.make_workload("headline")
    x, w = _inputs(wl.coords, cin, cout, "bf16", seed=cin)
    _, y = _run(S, wl.coords, 128, 1, x, w, "bf16", act="gelu")
    rows = sample_rows(wl.n, 4000, seed=cin)
    ref = _oracle(wl.coords, 128, 1, x, w, act="gelu", bf16_out=True, rows=rows)
    assert_close(y[rows], ref, RTOL_BF16, f"headline {cin}->{cout}")


def test_bf16_dense_sampled_and_vs_conv3d(S):
    wl = WL.make_workload("dense")
    x, w = wl.features(), wl.weights()[0]
    _, y = _run(S, wl.coords, 128, 1, x, w, "bf16")
    rows = sample_rows(wl.n, 20000, seed=2)
    ref = _oracle(wl.coords, 128, 1, x, w, bf16_out=True, rows=rows)
    assert_close(y[rows], ref, RTOL_BF16, "dense sampled")
    # On a fully occupied grid the op is a dense zero-padded Conv3d: compare
    # every output with torch's conv3d run in fp32 on the same bf16 values.
    xd = torch.from_numpy(x).cuda().view(128, 128, 128, 128).permute(3, 0, 1, 2)[None]
    wd = torch.from_numpy(w).cuda().permute(0, 4, 1, 2, 3)
    with torch.backends.cudnn.flags(enabled=True, allow_tf32=False):
        ref_all = torch.nn.functional.conv3d(xd.contiguous(), wd.contiguous(), padding=1)
    ref_all = ref_all[0].permute(1, 2, 3, 0).reshape(-1, 128).double().cpu().numpy()
    assert_close(y, ref_all, RTOL_BF16, "dense vs conv3d")


def test_bf16_batched_stack_per_layer(S):
    # 4 chained layers 64->128->128->128->64 with GELU between, one cached map.
    # Each layer is checked on sampled rows against the oracle fed with that
    # layer's actual (bf16) GPU input.
    wl = WL.make_workload("batched")
    coords = torch.from_numpy(wl.coords).cuda()
    x = wl.features()
    ws = wl.weights()
    st = S.SparseTensor(coords, torch.from_numpy(x).cuda().to(torch.bfloat16), 256, 4)
    nbr_ref = C.build_map(wl.coords, 256, 4)
    rows = sample_rows(wl.n, 8000, seed=5)
    for l, w in enumerate(ws):
        act = "gelu" if l < len(ws) - 1 else None
        h = st.get_map("subm_stack")
        xin = st.feats.float().cpu().numpy().astype(np.float64)
        y = S.forward(h, st.feats, torch.from_numpy(w).cuda().to(torch.bfloat16), act=act)
        ref = C.forward(nbr_ref, xin, np.asarray(w, np.float64), act=act, round_to_bf16=True,
                        rows=rows)
        assert_close(y.float().cpu().numpy()[rows], ref, RTOL_BF16, f"stack layer {l}")
        st = st.replace(y)
    assert len(st.cache) == 1


def test_bf16_stack_end_to_end_small(S):
    # the same 4-layer stack on a small batched set, checked end to end
    c = WL.batched_coords(batch=2, grid=48, min_voxels=3000, seed0=7, r_lo=6, r_hi=16)
    chans = [64, 128, 128, 128, 64]
    x = WL.to_bf16_values(WL.make_features(c.shape[0], 64, 11))
    ws = [WL.to_bf16_values(WL.make_weight(chans[l + 1], chans[l], 20 + l)) for l in range(4)]
    mod = [S.SubMConv3d(chans[l], chans[l + 1], "k", act="gelu" if l < 3 else None,
                        device="cuda") for l in range(4)]
    for m, w in zip(mod, ws):
        m.weight.data.copy_(torch.from_numpy(w).cuda().to(torch.bfloat16))
    st = S.SparseTensor(torch.from_numpy(c).cuda(), torch.from_numpy(x).cuda().to(torch.bfloat16),
                        48, 2)
    for m in mod:
        st = m(st)
    nbr = C.build_map(c, 48, 2)
    ref = np.asarray(x, np.float64)
    for l, w in enumerate(ws):
        ref = C.forward(nbr, ref, np.asarray(w, np.float64), act="gelu" if l < 3 else None,
                        round_to_bf16=True)
    assert_close(st.feats.float().cpu().numpy(), ref, RTOL_BF16, "stack e2e")


@pytest.mark.parametrize("name", ["shell_bf16", "headline"])
@pytest.mark.parametrize("flip", [False, True])
def test_bf16_both_kernels_agree_with_oracle(S, name, flip):
    """The x-run kernel (subm3d_forward_map) and the per-offset gather kernel
    (subm3d_forward) on the same map and inputs, both against the oracle."""
    wl = WL.make_workload(name)
    x, w = wl.features(), wl.weights()[0]
    h = S.build_map(torch.from_numpy(wl.coords).cuda(), wl.grid_dim, wl.batch)
    xt = torch.from_numpy(x).cuda().to(torch.bfloat16)
    wt = torch.from_numpy(w).cuda().to(torch.bfloat16)
    rows = sample_rows(wl.n, 6000, seed=4)
    ref = _oracle(wl.coords, wl.grid_dim, wl.batch, x, w, flip=flip, bf16_out=True, rows=rows)
    for kernel in ("auto", "gather"):
        y = S.forward(h, xt, wt, flip=flip, kernel=kernel).float().cpu().numpy()
        assert S._abi.subm3d_device_status() == 0
        assert_close(y[rows], ref, RTOL_BF16, f"{name} {kernel} flip={flip}")


def test_kernel_choice_and_knob(S, monkeypatch):
    """subm3d_forward_map runs the x-run kernel wherever its layout applies and
    Cin >= 48, on short runs too (the 64^3 shell: runs of ~4 voxels, 1.50 N
    positions); at 48 and 80 input channels its last 64-channel chunk is partial
    (zero-filled past Cin).  Below 48 channels it takes the per-offset kernel of
    subm3d_forward, and SUBM3D_FORWARD_KERNEL=gather does so everywhere.  Each
    kernel is deterministic, so results match bit for bit the kernel that ran."""
    wl = WL.make_workload("shell_bf16")
    c = torch.from_numpy(wl.coords).cuda()
    h = S.build_map(c, wl.grid_dim, wl.batch)
    hdr = S.run_layout_tensors(h)[2].cpu().numpy()
    assert hdr[2] > 1.45 * wl.n
    for cin in (32, 48, 64, 80, 128):
        xt = torch.from_numpy(WL.to_bf16_values(WL.make_features(wl.n, cin, 41))).cuda().to(
            torch.bfloat16)
        wt = torch.from_numpy(WL.to_bf16_values(WL.make_weight(64, cin, 42))).cuda().to(
            torch.bfloat16)
        auto = S.forward(h, xt, wt)
        gather = S.forward(h, xt, wt, kernel="gather")       # subm3d_forward on nbr
        monkeypatch.setenv("SUBM3D_FORWARD_KERNEL", "gather")
        knob = S.forward(h, xt, wt)
        monkeypatch.delenv("SUBM3D_FORWARD_KERNEL")
        torch.cuda.synchronize()
        assert S._abi.subm3d_device_status() == 0
        assert torch.equal(knob, gather), cin
        if cin < 48:
            assert torch.equal(auto, gather), cin
        ref = _oracle(wl.coords, wl.grid_dim, 1, xt.float().cpu().numpy(),
                      wt.float().cpu().numpy(), bf16_out=True)
        for what, y in (("auto", auto), ("gather", gather)):
            assert_close(y.float().cpu().numpy(), ref, RTOL_BF16, f"{what} cin={cin}")
