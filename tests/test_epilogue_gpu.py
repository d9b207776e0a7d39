"""Residual-block epilogue on the GPU vs the CPU oracle:
out = act(conv + bias) + residual, one rounding of a bf16 output, on every
forward kernel (x-run bf16, per-offset gather bf16, fp32), with the residual
separate or in place (residual is out), and the two-convolution block that
chains them on one map.  Bars as the plain forward: 2e-2 (bf16), 1e-5 (fp32)
of |ref| + rms(ref)."""
import zlib

import numpy as np
import pytest
import torch

import workloads as WL
from oracle import cpp as C
from tests.helpers import RTOL_BF16, RTOL_F32, assert_close

pytestmark = pytest.mark.gpu

# (name, dtype, cin, cout): the x-run kernel takes bf16 with Cin >= 48 (48: a
# partial 64-channel chunk), the gather kernel narrower bf16, fp32 the
# CUDA-core kernel
PATHS = [("xrun64", "bf16", 64, 64), ("xrun128", "bf16", 128, 128),
         ("xrun48", "bf16", 48, 32), ("gather32", "bf16", 32, 48), ("f32", "f32", 24, 40)]


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


@pytest.mark.parametrize("path", PATHS, ids=[p[0] for p in PATHS])
@pytest.mark.parametrize("act", [None, "gelu", "silu"])
@pytest.mark.parametrize("with_bias", [False, True])
@pytest.mark.parametrize("res_mode", [None, "separate", "inplace"])
def test_fused_epilogue_matches_oracle(S, shell, path, act, with_bias, res_mode):
    name, dtype, cin, cout = path
    wl, nbr = shell
    n = wl.n
    rng = np.random.default_rng(zlib.crc32(f"{name}/{act}/{with_bias}/{res_mode}".encode()))
    x = _vals(WL.make_features(n, cin, 5), dtype)
    w = _vals(WL.make_weight(cout, cin, 6), dtype)
    bias = _vals(rng.standard_normal(cout).astype(np.float32) * 0.5, dtype) if with_bias else None
    res = _vals(rng.standard_normal((n, cout)).astype(np.float32), dtype) if res_mode else None
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    h = S.build_map(torch.from_numpy(wl.coords).cuda(), wl.grid_dim, wl.batch)
    xt = torch.from_numpy(x).cuda().to(tdt)
    wt = torch.from_numpy(w).cuda().to(tdt)
    bt = torch.from_numpy(bias).cuda().to(tdt) if bias is not None else None
    rt = torch.from_numpy(res).cuda().to(tdt) if res is not None else None
    out = rt if res_mode == "inplace" else None
    y = S.forward(h, xt, wt, act=act, bias=bt, residual=rt, out=out)
    torch.cuda.synchronize()
    assert S._abi.subm3d_device_status() == 0
    if res_mode == "inplace":
        assert y.data_ptr() == rt.data_ptr()
    ref = C.forward(nbr, x.astype(np.float64), w.astype(np.float64), act=act,
                    bias=None if bias is None else bias.astype(np.float64),
                    residual=None if res is None else res.astype(np.float64),
                    round_to_bf16=(dtype == "bf16"))
    assert_close(y.float().cpu().numpy(), ref, RTOL_BF16 if dtype == "bf16" else RTOL_F32,
                 f"{name} act={act} bias={with_bias} residual={res_mode}")


@pytest.mark.parametrize("act", ["silu", "gelu"])
def test_res_block_two_convs_one_map(S, act):
    """SubMResBlock3d: h = bf16(act(conv1(x) + b1)); out = bf16(conv2(h) + b2 + x),
    both convolutions on one cached map, against the oracle chain."""
    wl = WL.make_workload("shell_bf16")
    c = wl.channels[0]
    torch.manual_seed(0)
    blk = S.SubMResBlock3d(c, indice_key="blk", act=act, device="cuda")
    x = WL.to_bf16_values(wl.features())
    st = S.SparseTensor(torch.from_numpy(wl.coords).cuda(), torch.from_numpy(x).cuda().to(torch.bfloat16),
                        wl.grid_dim, wl.batch)
    y = blk(st)
    torch.cuda.synchronize()
    assert list(st.cache) == ["blk"] and y.cache is st.cache   # one map for both convolutions
    f64 = lambda t: t.detach().float().cpu().numpy().astype(np.float64)
    nbr = C.build_map(wl.coords, wl.grid_dim, wl.batch)
    h_ref = C.forward(nbr, x.astype(np.float64), f64(blk.conv1.weight), act=act,
                      bias=f64(blk.conv1.bias), round_to_bf16=True)
    ref = C.forward(nbr, h_ref, f64(blk.conv2.weight), bias=f64(blk.conv2.bias),
                    residual=x.astype(np.float64), round_to_bf16=True)
    assert_close(y.feats.float().cpu().numpy(), ref, RTOL_BF16, f"res block {act}")


def test_fused_argument_errors(S):
    wl = WL.make_workload("shell")
    h = S.build_map(torch.from_numpy(wl.coords).cuda(), wl.grid_dim, wl.batch)
    n, c = wl.n, 64
    x = torch.zeros(n, c, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(c, 27, c, dtype=torch.bfloat16, device="cuda")
    buf = torch.zeros(n * c + 64, dtype=torch.bfloat16, device="cuda")
    out = buf[:n * c].view(n, c)
    lib, A = S._abi.lib, S._abi
    # residual partly overlapping out: E_INVALID; identical: allowed (in place)
    part = buf[8:8 + n * c]
    assert lib.subm3d_forward_fused(h.ptr, x.data_ptr(), w.data_ptr(), None, part.data_ptr(),
                                    out.data_ptr(), c, c, A.SUBM3D_BF16, 0, 0, None) \
        == A.SUBM3D_E_INVALID
    assert lib.subm3d_forward_fused(h.ptr, x.data_ptr(), w.data_ptr(), None, out.data_ptr(),
                                    out.data_ptr(), c, c, A.SUBM3D_BF16, 0, 0, None) == A.SUBM3D_OK
    # a bf16 residual not 16-byte aligned: E_UNSUPPORTED; an unknown activation: E_INVALID
    other = torch.zeros(n * c + 64, dtype=torch.bfloat16, device="cuda")
    assert lib.subm3d_forward_fused(h.ptr, x.data_ptr(), w.data_ptr(), None,
                                    other.data_ptr() + 2, out.data_ptr(), c, c, A.SUBM3D_BF16, 0,
                                    0, None) == A.SUBM3D_E_UNSUPPORTED
    assert lib.subm3d_forward_fused(h.ptr, x.data_ptr(), w.data_ptr(), None, None,
                                    out.data_ptr(), c, c, A.SUBM3D_BF16, 0, 3, None) \
        == A.SUBM3D_E_INVALID
    torch.cuda.synchronize()
    with pytest.raises(ValueError):
        S.forward(h, x, w, bias=torch.zeros(c + 1, dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ValueError):
        S.forward(h, x, w, residual=torch.zeros(n, c + 16, dtype=torch.bfloat16, device="cuda"))
