"""Calls on explicit, non-default streams.

Every entry point takes a stream (the Python binding: `stream=`, else torch's
current stream).  A map is built on one side stream behind a sleeping kernel,
the forward, input gradient and weight gradient run on a second stream that
waits for the first, and the resolution changes run inside a
`torch.cuda.stream` context.  Outputs start as NaN and must equal, bit for bit
(the fp32 weight gradient: at the fp32 bar), the same calls on the default
stream; a call enqueued on the wrong stream would run before the build it
depends on and leave NaN or stale rows.
"""
import numpy as np
import pytest
import torch

import workloads as WL
from tests.helpers import RTOL_F32, assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    import sparse_voxel_conv_b200 as S
    return S


@pytest.fixture(scope="module")
def shell():
    wl = WL.make_workload("shell")
    x = WL.to_bf16_values(WL.make_features(wl.n, 64, 21))
    w = WL.to_bf16_values(WL.make_weight(64, 64, 22))
    return wl, x, w


def _nan_like(t):
    o = torch.empty_like(t)
    o.view(torch.int16).fill_(-1)
    return o


def test_conv_calls_on_side_streams(S, shell):
    wl, x, w = shell
    c = torch.from_numpy(wl.coords).cuda()
    xt = torch.from_numpy(x).cuda().to(torch.bfloat16)
    wt = torch.from_numpy(w).cuda().to(torch.bfloat16)
    h0 = S.build_map(c, wl.grid_dim, wl.batch)
    y0 = S.forward(h0, xt, wt, act="gelu")
    dx0 = S.backward_data(h0, y0, wt)
    dw0 = S.backward_weight(h0, xt, y0)
    torch.cuda.synchronize()

    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    y, dx = _nan_like(y0), _nan_like(dx0)
    dw = torch.full_like(dw0, float("nan"))
    torch.cuda.synchronize()
    with torch.cuda.stream(s1):
        torch.cuda._sleep(4_000_000)  # the build waits behind this on s1
    h = S.build_map(c, wl.grid_dim, wl.batch, check=False, stream=s1)
    s2.wait_stream(s1)
    S.forward(h, xt, wt, act="gelu", out=y, stream=s2)
    S.backward_data(h, y, wt, out=dx, stream=s2)
    S.backward_weight(h, xt, y, out=dw, stream=s2)
    torch.cuda.synchronize()
    assert S._abi.subm3d_device_status() == 0
    assert S.map_status(h) == 0
    assert torch.equal(h.nbr, h0.nbr)
    assert torch.equal(y, y0)
    assert torch.equal(dx, dx0)
    assert_close(dw.cpu().numpy(), dw0.cpu().numpy(), RTOL_F32, "weight gradient on a side stream")


def test_resolution_changes_in_a_stream_context(S, shell):
    wl, x, _ = shell
    c = torch.from_numpy(wl.coords).cuda()
    xt = torch.from_numpy(x).cuda().to(torch.bfloat16)
    st0 = S.SparseTensor(c, xt, grid_dim=wl.grid_dim, batch=wl.batch)
    fine0 = S.subdivide(st0)
    back0 = S.downsample(fine0, "mean")
    torch.cuda.synchronize()

    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        torch.cuda._sleep(4_000_000)
        st = S.SparseTensor(c, xt, grid_dim=wl.grid_dim, batch=wl.batch)
        fine = S.subdivide(st)
        back = S.downsample(fine, "mean")
    torch.cuda.synchronize()
    assert S._abi.subm3d_device_status() == 0
    assert torch.equal(fine.coords, fine0.coords) and torch.equal(fine.feats, fine0.feats)
    assert torch.equal(back.coords, back0.coords) and torch.equal(back.feats, back0.feats)
