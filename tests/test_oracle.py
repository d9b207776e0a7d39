"""Pins for the CPU oracle: every check compares it with something other than
itself (a brute-force scan, torch's dense Conv3d, closed forms, invariants,
hand-worked fixtures), so a dropped term, a wrong sign or index, or a
transposed operand in either oracle fails here.  CPU only."""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import workloads as WL
from oracle import cpp as C
from oracle import subm3d_oracle as P

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
ORACLES = [pytest.param(P, id="py"), pytest.param(C, id="cpp")]


def _rand_coords(rng, n, grid, batch=1):
    """n distinct random voxels of a batch x grid^3 volume, random row order."""
    cells = rng.choice(batch * grid ** 3, size=n, replace=False)
    b, rem = np.divmod(cells, grid ** 3)
    z, rem = np.divmod(rem, grid * grid)
    y, x = np.divmod(rem, grid)
    return np.stack([b, z, y, x], 1).astype(np.int32)


# ---------------------------------------------------------------- the map ---

@pytest.mark.parametrize("orc", ORACLES)
def test_map_matches_all_pairs_brute_force(orc):
    c = WL.tiny_coords()
    assert c.shape[0] == 1223
    nbr = orc.build_map(c, 16)
    assert np.array_equal(nbr, P.brute_force_map(c))
    # 9.6k non-empty entries on the tiny set, the centre always included
    assert int((nbr >= 0).sum()) == 9637


@pytest.mark.parametrize("orc", ORACLES)
def test_map_brute_force_random_batched(orc):
    rng = np.random.default_rng(7)
    c = _rand_coords(rng, 1500, 12, batch=3)
    nbr = orc.build_map(c, 12, batch=3)
    assert np.array_equal(nbr, P.brute_force_map(c))


def test_map_invariants_and_symmetry():
    c = WL.shell_coords()
    nbr = C.build_map(c, 64)
    n = c.shape[0]
    assert np.array_equal(nbr[:, 13], np.arange(n))
    # j is the k-neighbour of i  <=>  i is the (26-k)-neighbour of j
    i, k = np.nonzero(nbr >= 0)
    j = nbr[i, k]
    assert np.array_equal(nbr[j, 26 - k], i)
    # every recorded neighbour really sits at offset d_k and shares b
    d = c[j].astype(np.int64) - c[i]
    off = np.array(P.OFFSETS)[k]
    assert np.array_equal(d[:, 1:], off) and np.all(d[:, 0] == 0)


def test_map_dense_count_closed_form():
    # In a fully occupied g^3 grid the number of ordered neighbour pairs (self
    # included) is (3g-2)^3: per axis, sum over positions of the in-range
    # offsets is g + 2(g-1).
    for g in (3, 5, 9):
        nbr = C.build_map(WL.dense_coords(g), g)
        assert int((nbr >= 0).sum()) == (3 * g - 2) ** 3


def test_map_row_permutation_equivariance():
    c = WL.shell_coords()
    nbr = C.build_map(c, 64)
    perm = WL.permute_rows(c.shape[0], 3)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size)
    nbr_p = C.build_map(c[perm], 64)
    expect = np.where(nbr[perm] >= 0, inv[np.maximum(nbr[perm], 0)], -1)
    assert np.array_equal(nbr_p, expect)


def test_map_translation_invariance():
    c = WL.tiny_coords()
    nbr = C.build_map(c, 16)
    t = np.array([0, 5, 2, 7], np.int32)
    assert np.array_equal(C.build_map(c + t, 32), nbr)


def test_map_never_crosses_batch():
    c0 = WL.tiny_coords()
    c = np.concatenate([c0, c0 + np.array([1, 0, 0, 0], np.int32)])
    nbr = C.build_map(c, 16, batch=2)
    n0 = c0.shape[0]
    assert np.all(nbr[:n0][nbr[:n0] >= 0] < n0)
    assert np.all(nbr[n0:][nbr[n0:] >= 0] >= n0)
    assert np.array_equal(nbr[n0:], np.where(nbr[:n0] >= 0, nbr[:n0] + n0, -1))


@pytest.mark.parametrize("orc", ORACLES)
@pytest.mark.parametrize("bad", [[0, 0, 0, 16], [0, -1, 0, 0], [0, 0, 16, 0], [1, 0, 0, 0],
                                 [-1, 0, 0, 0]])
def test_map_rejects_out_of_range(orc, bad):
    c = np.array([[0, 1, 1, 1], bad], np.int32)
    with pytest.raises(ValueError):
        orc.build_map(c, 16, batch=1)


@pytest.mark.parametrize("orc", ORACLES)
def test_map_rejects_duplicates(orc):
    c = np.array([[0, 1, 1, 1], [0, 2, 2, 2], [0, 1, 1, 1]], np.int32)
    with pytest.raises(ValueError):
        orc.build_map(c, 16)


def test_map_empty_and_single():
    for orc in (P, C):
        assert orc.build_map(np.zeros((0, 4), np.int32), 8).shape == (0, 27)
        one = orc.build_map(np.array([[0, 0, 0, 0]], np.int32), 1)
        assert one[0, 13] == 0 and (one >= 0).sum() == 1


# ------------------------------------------------------------ the forward ---

def _dense_case(g, batch, cin, cout, seed):
    rng = np.random.default_rng(seed)
    c = WL.dense_coords(g, batch)
    x = rng.standard_normal((c.shape[0], cin))
    w = rng.standard_normal((cout, 3, 3, 3, cin))
    return c, x, w


def _dense_conv(c, x, w, g, batch, flip):
    """torch's dense zero-padded Conv3d on the grid the voxels fill."""
    cin = x.shape[1]
    xd = torch.zeros(batch, cin, g, g, g, dtype=torch.float64)
    ct = torch.from_numpy(c.astype(np.int64))
    xd[ct[:, 0], :, ct[:, 1], ct[:, 2], ct[:, 3]] = torch.from_numpy(x)
    wt = torch.from_numpy(w).permute(0, 4, 1, 2, 3)  # KRSC -> [Cout, Cin, kz, ky, kx]
    if flip:
        wt = wt.flip(2, 3, 4)
    yd = F.conv3d(xd, wt, padding=1)
    return yd[ct[:, 0], :, ct[:, 1], ct[:, 2], ct[:, 3]].numpy()


@pytest.mark.parametrize("orc", ORACLES)
@pytest.mark.parametrize("g,batch,cin,cout", [(4, 1, 3, 5), (7, 2, 4, 2)])
@pytest.mark.parametrize("flip", [False, True])
def test_forward_equals_dense_conv3d_on_full_grid(orc, g, batch, cin, cout, flip):
    c, x, w = _dense_case(g, batch, cin, cout, seed=g)
    nbr = orc.build_map(c, g, batch)
    out = orc.forward(nbr, x, w, flip=flip)
    ref = _dense_conv(c, x, w, g, batch, flip)
    assert np.max(np.abs(out - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_forward_dense_16_cubed_cpp():
    c, x, w = _dense_case(16, 1, 8, 8, seed=16)
    nbr = C.build_map(c, 16)
    ref = _dense_conv(c, x, w, 16, 1, False)
    assert np.max(np.abs(C.forward(nbr, x, w) - ref)) <= 1e-12 * np.max(np.abs(ref))


@pytest.mark.parametrize("orc", ORACLES)
def test_isolated_voxels_see_only_centre_slice(orc):
    # voxels on a stride-2 lattice never touch: out = W[:, 13, :] @ x
    g = 9
    pts = [(0, z, y, x) for z in range(0, g, 2) for y in range(0, g, 2) for x in range(0, g, 2)]
    c = np.array(pts, np.int32)
    rng = np.random.default_rng(1)
    x = rng.standard_normal((c.shape[0], 6))
    w = rng.standard_normal((5, 3, 3, 3, 6))
    out = orc.forward(orc.build_map(c, g), x, w)
    assert np.allclose(out, x @ w[:, 1, 1, 1, :].T, rtol=0, atol=1e-13)
    assert np.allclose(orc.forward(orc.build_map(c, g), x, w, flip=True), out, rtol=0, atol=1e-13)


@pytest.mark.parametrize("orc", ORACLES)
def test_one_hot_probe_pins_orientation(orc):
    # Only voxel v carries a feature, e_c.  Every other voxel j then sees it
    # exactly when p_v - p_j = d_k for some k, and out[j] = W[:, k, c]
    # (correlation) or W[:, 26-k, c] (flip).  d_k comes from the coordinates
    # directly, not from any map.
    rng = np.random.default_rng(11)
    c = _rand_coords(rng, 150, 6)
    cin, cout = 3, 4
    w = rng.standard_normal((cout, 3, 3, 3, cin))
    nbr = orc.build_map(c, 6)
    for v in (0, 17, 123):
        for ch in range(cin):
            x = np.zeros((c.shape[0], cin))
            x[v, ch] = 1.0
            for flip in (False, True):
                out = orc.forward(nbr, x, w, flip=flip)
                for j in range(c.shape[0]):
                    d = c[v] - c[j]
                    if d[0] == 0 and np.all(np.abs(d[1:]) <= 1):
                        dz, dy, dx = d[1:]
                        kz, ky, kx = (1 - dz, 1 - dy, 1 - dx) if flip else (1 + dz, 1 + dy, 1 + dx)
                        assert np.array_equal(out[j], w[:, kz, ky, kx, ch])
                    else:
                        assert not out[j].any()


@pytest.mark.parametrize("orc", ORACLES)
def test_translation_invariance_of_outputs(orc):
    c = WL.tiny_coords()
    x = WL.make_features(c.shape[0], 8, 1).astype(np.float64)
    w = WL.make_weight(8, 8, 2).astype(np.float64)
    out = orc.forward(orc.build_map(c, 16), x, w)
    t = np.array([0, 3, 9, 1], np.int32)
    assert np.array_equal(orc.forward(orc.build_map(c + t, 32), x, w), out)


@pytest.mark.parametrize("orc", ORACLES)
def test_flip_equals_reversed_kernel_and_is_involution(orc):
    c = WL.tiny_coords()
    nbr = orc.build_map(c, 16)
    rng = np.random.default_rng(5)
    x = rng.standard_normal((c.shape[0], 8))
    w = rng.standard_normal((8, 3, 3, 3, 8))
    w_mirror = np.ascontiguousarray(w[:, ::-1, ::-1, ::-1, :])
    a = orc.forward(nbr, x, w, flip=True)
    assert np.array_equal(a, orc.forward(nbr, x, w_mirror, flip=False))
    # flipping twice (mirror the weight, then flip) gives back the original
    assert np.array_equal(orc.forward(nbr, x, w_mirror, flip=True), orc.forward(nbr, x, w))


def test_linearity():
    c = WL.shell_coords()
    nbr = C.build_map(c, 64)
    rng = np.random.default_rng(9)
    x1, x2 = rng.standard_normal((2, c.shape[0], 16))
    w = rng.standard_normal((12, 3, 3, 3, 16))
    lhs = C.forward(nbr, 2.5 * x1 - 0.75 * x2, w)
    rhs = 2.5 * C.forward(nbr, x1, w) - 0.75 * C.forward(nbr, x2, w)
    assert np.max(np.abs(lhs - rhs)) <= 1e-12 * np.max(np.abs(rhs))


def test_batch_independence():
    c0 = WL.tiny_coords()
    c = np.concatenate([c0, c0 + np.array([1, 0, 0, 0], np.int32)])
    rng = np.random.default_rng(2)
    x0 = rng.standard_normal((c0.shape[0], 8))
    w = rng.standard_normal((8, 3, 3, 3, 8))
    out = C.forward(C.build_map(c, 16, 2), np.concatenate([x0, x0]), w)
    n0 = c0.shape[0]
    assert np.array_equal(out[:n0], out[n0:])
    assert np.array_equal(out[:n0], C.forward(C.build_map(c0, 16), x0, w))


def test_row_subset_and_permutation():
    c = WL.shell_coords()
    x = WL.make_features(c.shape[0], 16, 4).astype(np.float64)
    w = WL.make_weight(8, 16, 5).astype(np.float64)
    full = C.forward(C.build_map(c, 64), x, w)
    rows = np.array([0, 5, 14533, 77, 77])
    assert np.array_equal(C.forward(C.build_map(c, 64), x, w, rows=rows), full[rows])
    perm = WL.permute_rows(c.shape[0], 8)
    assert np.array_equal(C.forward(C.build_map(c[perm], 64), x[perm], w), full[perm])


def test_python_and_cpp_oracles_agree():
    wl = WL.make_workload("tiny")
    nbr_p = P.build_map(wl.coords, 16)
    nbr_c = C.build_map(wl.coords, 16)
    assert np.array_equal(nbr_p, nbr_c)
    x = wl.features().astype(np.float64)
    w = wl.weights()[0].astype(np.float64)
    for flip in (False, True):
        a = P.forward(nbr_p, x, w, flip=flip, act="gelu", round_to_bf16=True)
        b = C.forward(nbr_c, x, w, flip=flip, act="gelu", round_to_bf16=True)
        assert np.max(np.abs(a - b)) <= 1e-12 * np.max(np.abs(a))
        a = P.forward(nbr_p, x, w, flip=flip)
        b = C.forward(nbr_c, x, w, flip=flip)
        assert np.max(np.abs(a - b)) <= 1e-12 * np.max(np.abs(a))


# --------------------------------------------------------- golden fixtures ---

def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


@pytest.mark.parametrize("orc", ORACLES)
def test_golden_two_voxels(orc):
    g = _load("hand_two_voxels.json")
    c = np.array(g["coords"], np.int32)
    x = np.array(g["feats"], np.float64)
    cout, cin = 3, 2
    w = np.full((cout, 27, cin), float(g["W_other"]))
    for k, s in g["W_slices"].items():
        w[:, int(k), :] = np.array(s, np.float64)
    nbr = orc.build_map(c, g["grid_dim"], g["batch"])
    assert np.array_equal(nbr, np.array(g["nbr"], np.int32))
    assert np.array_equal(orc.forward(nbr, x, w.reshape(cout, 3, 3, 3, cin)), np.array(g["out"], float))
    assert np.array_equal(orc.forward(nbr, x, w.reshape(cout, 3, 3, 3, cin), flip=True),
                          np.array(g["out_flip"], float))


@pytest.mark.parametrize("orc", ORACLES)
def test_golden_four_voxels(orc):
    g = _load("hand_four_voxels.json")
    c = np.array(g["coords"], np.int32)
    x = np.array(g["feats"], np.float64)
    w = np.array(g["W_by_k"], np.float64).reshape(1, 3, 3, 3, 1)
    nbr = orc.build_map(c, g["grid_dim"], g["batch"])
    expect = np.full((4, 27), -1, np.int32)
    for i, row in g["nbr_nonempty"].items():
        for k, j in row.items():
            expect[int(i), int(k)] = j
    assert np.array_equal(nbr, expect)
    assert np.array_equal(orc.forward(nbr, x, w)[:, 0], np.array(g["out"], float))
    assert np.array_equal(orc.forward(nbr, x, w, flip=True)[:, 0], np.array(g["out_flip"], float))


# ------------------------------------------------- activation and rounding ---

@pytest.mark.parametrize("orc", ORACLES)
def test_gelu_closed_forms_and_torch(orc):
    v = np.linspace(-8, 8, 1601)
    got = orc.gelu(v)
    ref = F.gelu(torch.from_numpy(v)).numpy()   # torch's default is the exact erf form
    assert np.max(np.abs(got - ref)) <= 1e-15
    assert orc.gelu(np.array([0.0]))[0] == 0.0
    # Phi(1) = 0.5 * (1 + erf(1/sqrt 2)) = 0.841344746068542948...
    assert abs(orc.gelu(np.array([1.0]))[0] - 0.8413447460685429) < 1e-15
    # gelu(v) - gelu(-v) = v
    assert np.max(np.abs(orc.gelu(v) - orc.gelu(-v) - v)) <= 1e-14
    # tanh form differs by ~1e-3 somewhere: the test would catch a swap
    tanh_form = 0.5 * v * (1 + np.tanh(math.sqrt(2 / math.pi) * (v + 0.044715 * v ** 3)))
    assert np.max(np.abs(got - tanh_form)) > 1e-5


@pytest.mark.parametrize("orc", ORACLES)
def test_round_bf16_ties_and_torch(orc):
    one = 1.0
    ulp = 2.0 ** -7
    cases = {
        one + ulp / 2: one,                        # halfway, ties to even (down)
        one + 3 * ulp / 2: one + 2 * ulp,          # halfway, ties to even (up)
        one + ulp / 2 + 2.0 ** -30: one + ulp,     # just above halfway
        -(one + ulp / 2): -one,
        2.0 ** -130: 2.0 ** -130,                  # subnormal, representable
        2.0 ** -134: 0.0,                          # half the smallest subnormal: tie to 0
        3 * 2.0 ** -134: 2 * 2.0 ** -133,          # 1.5 subnormal ulps: tie to even (2)
        math.ldexp(255.0, 120): math.ldexp(255.0, 120),
        math.ldexp(255.5, 120): math.inf,          # halfway to 2^128 rounds to even: overflow
    }
    got = orc.round_bf16(np.array(list(cases.keys())))
    assert np.array_equal(got, np.array(list(cases.values())))
    # on float32 inputs a single RNE rounding is what torch's cast does
    rng = np.random.default_rng(0)
    f = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        (rng.standard_normal(1000) * 1e-39).astype(np.float32),
                        (rng.standard_normal(1000) * 1e37).astype(np.float32)])
    ref = torch.from_numpy(f).to(torch.bfloat16).double().numpy()
    assert np.array_equal(orc.round_bf16(f.astype(np.float64)), ref)


# ------------------------------------------------------------- generators ---

def test_workload_sizes():
    assert WL.tiny_coords().shape[0] == 1223
    assert WL.shell_coords().shape[0] == 14534
    assert WL.headline_coords().shape[0] == 329839
    b = WL.batched_coords()
    assert [int((b[:, 0] == i).sum()) for i in range(4)] == [281567, 292182, 288644, 272914]
    for c in (WL.tiny_coords(), WL.shell_coords()):
        keys = [tuple(r) for r in c.tolist()]
        assert keys == sorted(keys) and len(set(keys)) == len(keys)


# -------------------------------------------- fused residual-block epilogue ---

def _dense_block(c, x, w, bias, residual, g, batch, flip, act):
    """torch's dense Conv3d with its own bias argument, torch's activation, then
    the residual: the epilogue act(conv + bias) + residual on a full grid."""
    cin = x.shape[1]
    xd = torch.zeros(batch, cin, g, g, g, dtype=torch.float64)
    ct = torch.from_numpy(c.astype(np.int64))
    xd[ct[:, 0], :, ct[:, 1], ct[:, 2], ct[:, 3]] = torch.from_numpy(x)
    wt = torch.from_numpy(w).permute(0, 4, 1, 2, 3)
    if flip:
        wt = wt.flip(2, 3, 4)
    yd = F.conv3d(xd, wt, bias=torch.from_numpy(bias), padding=1)
    y = yd[ct[:, 0], :, ct[:, 1], ct[:, 2], ct[:, 3]]
    y = {"gelu": F.gelu, "silu": F.silu, None: lambda t: t}[act](y)
    return (y + torch.from_numpy(residual)).numpy()


@pytest.mark.parametrize("orc", ORACLES)
@pytest.mark.parametrize("act", [None, "gelu", "silu"])
@pytest.mark.parametrize("flip", [False, True])
def test_block_epilogue_equals_dense_conv3d_bias_act_residual(orc, act, flip):
    g, batch, cin, cout = 5, 2, 3, 4
    c, x, w = _dense_case(g, batch, cin, cout, seed=11)
    rng = np.random.default_rng(12)
    bias = rng.standard_normal(cout)
    residual = rng.standard_normal((c.shape[0], cout))
    nbr = orc.build_map(c, g, batch)
    out = orc.forward(nbr, x, w, flip=flip, act=act, bias=bias, residual=residual)
    ref = _dense_block(c, x, w, bias, residual, g, batch, flip, act)
    assert np.max(np.abs(out - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))
    # the residual enters after the activation and the bias before it
    if act is not None:
        no_res = orc.forward(nbr, x, w, flip=flip, act=act, bias=bias)
        assert np.max(np.abs(out - no_res - residual)) <= 1e-12


def test_block_epilogue_rows_and_bf16_rounding_once():
    wl = WL.make_workload("tiny")
    nbr = C.build_map(wl.coords, wl.grid_dim)
    x = wl.features().astype(np.float64)
    w = wl.weights()[0].astype(np.float64)
    rng = np.random.default_rng(3)
    bias = rng.standard_normal(w.shape[0])
    res = rng.standard_normal((wl.n, w.shape[0]))
    full = C.forward(nbr, x, w, act="silu", bias=bias, residual=res)
    rows = np.array([0, 5, 77, wl.n - 1])
    part = C.forward(nbr, x, w, act="silu", bias=bias, residual=res, rows=rows)
    assert np.array_equal(part, full[rows])
    # the Python oracle agrees, and bf16 rounding is applied once, at the end
    py = P.forward(nbr, x, w, act="silu", bias=bias, residual=res, rows=rows, round_to_bf16=True)
    assert np.array_equal(py, P.round_bf16(full[rows]))


@pytest.mark.parametrize("orc", [P, C])
def test_silu_closed_forms_and_torch(orc):
    v = np.linspace(-30.0, 30.0, 4001)
    got = orc.silu(v)
    ref = F.silu(torch.from_numpy(v)).numpy()
    assert np.max(np.abs(got - ref)) <= 1e-14 * np.max(np.abs(ref))
    assert orc.silu(np.array([0.0]))[0] == 0.0
    # silu(v) - silu(-v) = v (sigmoid(v) + sigmoid(-v) = 1), and silu(1) = 1/(1+e^-1)
    assert np.max(np.abs(orc.silu(v) - orc.silu(-v) - v)) <= 1e-13
    assert abs(orc.silu(np.array([1.0]))[0] - 1.0 / (1.0 + math.exp(-1.0))) < 1e-15


# ------------------------------------------------------------- the backward ---

def _dense_grads(c, x, w, dy, g, batch, flip):
    """torch autograd through the dense zero-padded conv3d on a full grid."""
    cin = x.shape[1]
    xd = torch.zeros(batch, cin, g, g, g, dtype=torch.float64)
    ct = torch.from_numpy(c.astype(np.int64))
    xd[ct[:, 0], :, ct[:, 1], ct[:, 2], ct[:, 3]] = torch.from_numpy(x)
    xd.requires_grad_(True)
    wk = torch.from_numpy(w).clone().requires_grad_(True)        # KRSC
    wt = wk.permute(0, 4, 1, 2, 3)
    if flip:
        wt = wt.flip(2, 3, 4)
    yd = F.conv3d(xd, wt, padding=1)
    y = yd[ct[:, 0], :, ct[:, 1], ct[:, 2], ct[:, 3]]
    (y * torch.from_numpy(dy)).sum().backward()
    dx = xd.grad[ct[:, 0], :, ct[:, 1], ct[:, 2], ct[:, 3]].numpy()
    return dx, wk.grad.numpy()


@pytest.mark.parametrize("orc", ORACLES)
@pytest.mark.parametrize("flip", [False, True])
def test_backward_equals_torch_autograd_on_full_grid(orc, flip):
    g, batch, cin, cout = 5, 2, 3, 4
    c, x, w = _dense_case(g, batch, cin, cout, seed=21)
    dy = np.random.default_rng(22).standard_normal((c.shape[0], cout))
    nbr = orc.build_map(c, g, batch)
    dx_ref, dw_ref = _dense_grads(c, x, w, dy, g, batch, flip)
    dx = orc.backward_data(nbr, dy, w, flip=flip)
    dw = orc.backward_weight(nbr, x, dy, flip=flip)
    assert np.max(np.abs(dx - dx_ref)) <= 1e-12 * max(1.0, np.max(np.abs(dx_ref)))
    assert np.max(np.abs(dw - dw_ref)) <= 1e-12 * max(1.0, np.max(np.abs(dw_ref)))


@pytest.mark.parametrize("orc", ORACLES)
def test_backward_adjoint_identities_on_sparse_sets(orc):
    """<forward(x), dy> = <x, backward_data(dy)> = <W, backward_weight(x, dy)>
    for both orientations on a random sparse set (the forward is bilinear)."""
    rng = np.random.default_rng(23)
    c = _rand_coords(rng, 300, 9, batch=2)
    x = rng.standard_normal((300, 5))
    w = rng.standard_normal((6, 3, 3, 3, 5))
    dy = rng.standard_normal((300, 6))
    nbr = orc.build_map(c, 9, 2)
    for flip in (False, True):
        lhs = float(np.sum(orc.forward(nbr, x, w, flip=flip) * dy))
        via_x = float(np.sum(x * orc.backward_data(nbr, dy, w, flip=flip)))
        via_w = float(np.sum(w * orc.backward_weight(nbr, x, dy, flip=flip)))
        assert abs(lhs - via_x) <= 1e-10 * abs(lhs) and abs(lhs - via_w) <= 1e-10 * abs(lhs)


def test_backward_python_and_cpp_agree():
    wl = WL.make_workload("tiny")
    nbr = C.build_map(wl.coords, wl.grid_dim)
    x = wl.features().astype(np.float64)
    w = wl.weights()[0].astype(np.float64)
    dy = np.random.default_rng(24).standard_normal((wl.n, w.shape[0]))
    for flip in (False, True):
        assert np.max(np.abs(P.backward_data(nbr, dy, w, flip) - C.backward_data(nbr, dy, w, flip))) <= 1e-12
        assert np.max(np.abs(P.backward_weight(nbr, x, dy, flip) - C.backward_weight(nbr, x, dy, flip))) <= 1e-10
