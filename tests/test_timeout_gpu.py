"""Bounded device waits that run out, and the calls after them.

Every pipeline wait of the tensor-core kernels (an mbarrier wait for a copy,
an MMA group or an accumulator) gives up after a time limit: 2 s by default,
or the testing knob SUBM3D_WAIT_LIMIT_NS.  Here the limit is cut to one
microsecond, far below what a 256-position tile of a 128 -> 128 layer takes
(~20 us), so the epilogue's wait for the first accumulator runs out without
any input or protocol being broken.  The kernel must then leave its loops,
wait for the copies and MMAs it has in flight, free its tensor memory and
report SUBM3D_E_TIMEOUT through subm3d_device_status(); the next call, with
the default limit, must give the same result as before the timeout."""
import numpy as np
import pytest
import torch

import workloads as WL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def headline():
    import sparse_voxel_conv_b200 as S
    wl = WL.make_workload("headline")
    c = torch.from_numpy(wl.coords).cuda()
    h = S.build_map(c, wl.grid_dim, wl.batch)
    x = torch.from_numpy(WL.to_bf16_values(WL.make_features(wl.n, 128, 1))).cuda().to(
        torch.bfloat16)
    w = torch.from_numpy(WL.to_bf16_values(WL.make_weight(128, 128, 2))).cuda().to(torch.bfloat16)
    return S, h, x, w


def _timed_out_then_clean(A, monkeypatch, run):
    """run() once with a 1 us wait limit (must report a timeout), then with the
    default limit (must be clean); returns the clean result."""
    assert A.subm3d_device_status() == A.SUBM3D_OK
    monkeypatch.setenv("SUBM3D_WAIT_LIMIT_NS", "1000")
    run()
    assert A.subm3d_device_status() == A.SUBM3D_E_TIMEOUT
    monkeypatch.delenv("SUBM3D_WAIT_LIMIT_NS")
    y = run()
    assert A.subm3d_device_status() == A.SUBM3D_OK
    return y


@pytest.mark.parametrize("kernel", ["auto", "gather"])
def test_forward_wait_runs_out_then_next_call_is_clean(headline, monkeypatch, kernel):
    S, h, x, w = headline
    A = S._abi
    ref = S.forward(h, x, w, kernel=kernel)
    torch.cuda.synchronize()
    junk = torch.full_like(ref, 3.0)
    _timed_out_then_clean(A, monkeypatch, lambda: S.forward(h, x, w, kernel=kernel, out=junk))
    # the same kernel is deterministic: every output is one CTA's fixed-order sum
    assert torch.equal(junk, ref)
    # and the library keeps working on other shapes (tensor memory was released)
    y = S.forward(h, x[:, :64].contiguous(), w[..., :64].contiguous(), kernel=kernel)
    torch.cuda.synchronize()
    assert A.subm3d_device_status() == A.SUBM3D_OK
    assert torch.isfinite(y.float()).all()


def test_weight_gradient_wait_runs_out_then_next_call_is_clean(headline, monkeypatch):
    S, h, x, w = headline
    A = S._abi
    dy = torch.from_numpy(WL.to_bf16_values(WL.make_features(h.n, 128, 3))).cuda().to(
        torch.bfloat16)
    ref = S.backward_weight(h, x, dy)
    torch.cuda.synchronize()
    dw = torch.full_like(ref, 7.0)
    _timed_out_then_clean(A, monkeypatch, lambda: S.backward_weight(h, x, dy, out=dw))
    # fp32 atomics: the summation order varies, the sums agree to rounding
    err = (dw - ref).abs().max().item()
    assert err <= 1e-4 * ref.abs().max().item(), err
    assert np.isfinite(dw.cpu().numpy()).all()
