"""Backward on the GPU (through the C ABI) vs the CPU oracle's scatter-form
gradients, element by element.

Bars: the input gradient is a forward (bf16 out 2e-2, fp32 1e-5 of
|ref| + rms(ref)).  The weight gradient is fp32 for both dtypes and sums up to
N voxel terms per element in fp32 with atomics across voxel slices: a
random-walk rounding error of ~sqrt(N) * 2^-24 of the term scale (~1e-5 at
N = 14.5k); the bar is 1e-4 of |ref| + rms(ref).
"""
import numpy as np
import pytest
import torch

import workloads as WL
from oracle import cpp as C
from tests.helpers import RTOL_BF16, RTOL_F32, assert_close

pytestmark = pytest.mark.gpu
RTOL_WGRAD = 1e-4

# (name, dtype, cin, cout).  The input gradient is a forward Cout -> Cin, so
# xrun runs the x-run kernel there (Cout >= 48), gather the per-offset one.
PATHS = [("xrun", "bf16", 64, 128), ("gather", "bf16", 48, 32), ("f32", "f32", 24, 40)]


@pytest.fixture(scope="module")
def S():
    import sparse_voxel_conv_b200 as S
    return S


@pytest.fixture(scope="module")
def shell():
    wl = WL.make_workload("shell")
    return wl, C.build_map(wl.coords, wl.grid_dim, wl.batch)


def _vals(a, dtype):
    return WL.to_bf16_values(a) if dtype == "bf16" else a.astype(np.float32)


def _tensors(S, wl, dtype, cin, cout, seed):
    x = _vals(WL.make_features(wl.n, cin, seed), dtype)
    w = _vals(WL.make_weight(cout, cin, seed + 1), dtype)
    dy = _vals(WL.make_features(wl.n, cout, seed + 2), dtype)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    h = S.build_map(torch.from_numpy(wl.coords).cuda(), wl.grid_dim, wl.batch)
    t = lambda a: torch.from_numpy(a).cuda().to(tdt)
    return h, x, w, dy, t(x), t(w), t(dy)


@pytest.mark.parametrize("path", PATHS, ids=[p[0] for p in PATHS])
@pytest.mark.parametrize("flip", [False, True])
def test_backward_data_matches_oracle(S, shell, path, flip):
    name, dtype, cin, cout = path
    wl, nbr = shell
    h, x, w, dy, xt, wt, dyt = _tensors(S, wl, dtype, cin, cout, 31)
    dx = S.backward_data(h, dyt, wt, flip=flip)
    torch.cuda.synchronize()
    assert S._abi.subm3d_device_status() == 0
    ref = C.backward_data(nbr, dy.astype(np.float64), w.astype(np.float64), flip=flip)
    if dtype == "bf16":
        ref = C.round_bf16(ref)
    assert_close(dx.float().cpu().numpy(), ref, RTOL_BF16 if dtype == "bf16" else RTOL_F32,
                 f"dgrad {name} flip={flip}")


@pytest.mark.parametrize("path", PATHS, ids=[p[0] for p in PATHS])
@pytest.mark.parametrize("flip", [False, True])
def test_backward_weight_matches_oracle(S, shell, path, flip):
    name, dtype, cin, cout = path
    wl, nbr = shell
    h, x, w, dy, xt, wt, dyt = _tensors(S, wl, dtype, cin, cout, 41)
    dw = S.backward_weight(h, xt, dyt, flip=flip)
    torch.cuda.synchronize()
    ref = C.backward_weight(nbr, x.astype(np.float64), dy.astype(np.float64), flip=flip)
    assert dw.dtype == torch.float32 and tuple(dw.shape) == (cout, 3, 3, 3, cin)
    assert_close(dw.cpu().numpy(), ref, RTOL_WGRAD, f"wgrad {name} flip={flip}")


def test_backward_weight_ragged_and_empty(S):
    # the tiny set (1,223 voxels, not a multiple of the 16-voxel slices) and an empty one
    wl = WL.make_workload("tiny")
    nbr = C.build_map(wl.coords, wl.grid_dim)
    x, w = wl.features(), wl.weights()[0]
    dy = WL.make_features(wl.n, w.shape[0], 9)
    h = S.build_map(torch.from_numpy(wl.coords).cuda(), wl.grid_dim, 1)
    dw = S.backward_weight(h, torch.from_numpy(x).cuda(), torch.from_numpy(dy).cuda())
    ref = C.backward_weight(nbr, x.astype(np.float64), dy.astype(np.float64))
    assert_close(dw.cpu().numpy(), ref, RTOL_WGRAD, "wgrad tiny")
    dx = S.backward_data(h, torch.from_numpy(dy).cuda(), torch.from_numpy(w).cuda())
    assert_close(dx.cpu().numpy(), C.backward_data(nbr, dy.astype(np.float64), w.astype(np.float64)),
                 RTOL_F32, "dgrad tiny")
    h0 = S.build_map(torch.zeros((0, 4), dtype=torch.int32, device="cuda"), 8, 1)
    dw0 = torch.full((4, 3, 3, 3, 8), 7.0, device="cuda")
    S.backward_weight(h0, torch.zeros((0, 8), device="cuda"), torch.zeros((0, 4), device="cuda"),
                      out=dw0)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dw0).item() == 0     # the gradient of an empty sum is zero


@pytest.mark.parametrize("cin,cout", [(3, 5), (70, 130), (128, 128)])
def test_backward_weight_f32_shapes(S, shell, cin, cout):
    """The CUDA-core weight gradient (fp32): element-wise row pieces where Cin or
    Cout is not a multiple of 4, two output-channel blocks (130), whole tiles."""
    wl, nbr = shell
    h, x, w, dy, xt, wt, dyt = _tensors(S, wl, "f32", cin, cout, 71)
    dw = S.backward_weight(h, xt, dyt)
    torch.cuda.synchronize()
    ref = C.backward_weight(nbr, x.astype(np.float64), dy.astype(np.float64))
    assert_close(dw.cpu().numpy(), ref, RTOL_WGRAD, f"f32 wgrad {cin}->{cout}")


def test_backward_weight_f32_headline_slices(S):
    """fp32 128 -> 128 on the headline set (329,839 voxels, many voxel slices):
    dW[o][k][c] depends on dy[:, o] and x[:, c] only, so rows and columns of the
    full gradient are checked against the oracle on those columns."""
    wl = WL.make_workload("headline")
    x = WL.make_features(wl.n, 128, 81)
    dy = WL.make_features(wl.n, 128, 82)
    h = S.build_map(torch.from_numpy(wl.coords).cuda(), wl.grid_dim, 1)
    dw = S.backward_weight(h, torch.from_numpy(x).cuda(), torch.from_numpy(dy).cuda()).cpu().numpy()
    osel, csel = np.r_[0:8, 60:68, 120:128], np.r_[0:8, 64:72, 124:128]
    nbr = C.build_map(wl.coords, wl.grid_dim, 1)
    ref = C.backward_weight(nbr, x[:, csel].astype(np.float64), dy[:, osel].astype(np.float64))
    assert_close(dw[osel][:, :, :, :, csel], ref, RTOL_WGRAD, "f32 wgrad headline")


def test_autograd_through_subm_conv(S):
    """SubMConv3d with a trainable weight: loss = sum(y * g); torch autograd
    calls the library's backward kernels."""
    wl = WL.make_workload("shell")
    nbr = C.build_map(wl.coords, wl.grid_dim, wl.batch)
    cin = cout = 64
    x = WL.to_bf16_values(WL.make_features(wl.n, cin, 51))
    g = WL.to_bf16_values(WL.make_features(wl.n, cout, 52))
    conv = S.SubMConv3d(cin, cout, "ag", device="cuda")
    conv.weight.requires_grad_(True)
    xt = torch.from_numpy(x).cuda().to(torch.bfloat16).requires_grad_(True)
    st = S.SparseTensor(torch.from_numpy(wl.coords).cuda(), xt, wl.grid_dim, wl.batch)
    y = conv(st).feats
    (y.float() * torch.from_numpy(g).cuda()).sum().backward()
    torch.cuda.synchronize()
    w = conv.weight.detach().float().cpu().numpy().astype(np.float64)
    dx_ref = C.round_bf16(C.backward_data(nbr, g.astype(np.float64), w))
    dw_ref = C.backward_weight(nbr, x.astype(np.float64), g.astype(np.float64))
    assert_close(xt.grad.float().cpu().numpy(), dx_ref, RTOL_BF16, "autograd dx")
    # the weight gradient is returned in the weight's dtype (bf16): one rounding
    assert_close(conv.weight.grad.float().cpu().numpy(), C.round_bf16(dw_ref), RTOL_BF16,
                 "autograd dW")


@pytest.mark.parametrize("cin,cout", [(128, 128), (192, 64), (64, 144), (80, 64), (48, 48)])
@pytest.mark.parametrize("flip", [False, True])
def test_backward_weight_tensor_core_blocks(S, shell, cin, cout, flip):
    """The tcgen05 weight gradient over channel blocks of 128: full blocks, a
    partial input-channel block (192 = 128 + 64), output channels below and
    above one block (64, 144 = 128 + 16), and input channels that end inside a
    64-channel chunk (80 = 64 + 16, 48)."""
    wl, nbr = shell
    h, x, w, dy, xt, wt, dyt = _tensors(S, wl, "bf16", cin, cout, 61)
    dw = S.backward_weight(h, xt, dyt, flip=flip)
    torch.cuda.synchronize()
    assert S._abi.subm3d_device_status() == 0
    ref = C.backward_weight(nbr, x.astype(np.float64), dy.astype(np.float64), flip=flip)
    assert_close(dw.cpu().numpy(), ref, RTOL_WGRAD, f"wgrad {cin}->{cout} flip={flip}")


def test_backward_weight_headline_set(S):
    """The full headline set (329,839 voxels, 1,567 position tiles split over the
    CTAs' tile ranges) with 64 -> 64 channels, against the oracle."""
    wl = WL.make_workload("headline")
    nbr = C.build_map(wl.coords, wl.grid_dim, wl.batch)
    x = WL.to_bf16_values(WL.make_features(wl.n, 64, 71))
    dy = WL.to_bf16_values(WL.make_features(wl.n, 64, 72))
    h = S.build_map(torch.from_numpy(wl.coords).cuda(), wl.grid_dim, wl.batch)
    t = lambda a: torch.from_numpy(a).cuda().to(torch.bfloat16)
    dw = S.backward_weight(h, t(x), t(dy))
    torch.cuda.synchronize()
    assert S._abi.subm3d_device_status() == 0
    ref = C.backward_weight(nbr, x.astype(np.float64), dy.astype(np.float64))
    # up to 330k voxel terms per element: random-walk fp32 error ~sqrt(N) 2^-24 ~ 3e-5
    assert_close(dw.cpu().numpy(), ref, 2e-4, "wgrad headline")
