"""Map builds, forwards and weight gradients queued on one stream with no
synchronisation between them.

The library launches its kernels with programmatic dependent launch: a kernel
may start while the previous one on the stream is still running, and reads that
kernel's output only after griddepcontrol.wait.  Here the host queues every call
behind a sleeping kernel, so the GPU runs them back to back.  Two coordinate sets
(raster row order, and the same voxels with the rows permuted: a different x-run
layout) alternate on one nbr buffer and one workspace, and one set is rebuilt
again and again.  Every queued forward must equal, bit for bit, the forward of
a build that was waited for, in each table kind; outputs start as NaN, so a
skipped tile cannot pass.  A forward whose header read went through the
non-coherent load path failed this on most calls (whole tiles never written).
"""
import numpy as np
import pytest
import torch

import workloads as WL
from oracle import cpp as C
from tests.helpers import RTOL_BF16, RTOL_F32, assert_close, sample_rows

pytestmark = pytest.mark.gpu

SLEEP_CYCLES = 4_000_000  # ~2 ms: the host queues the whole sequence meanwhile


@pytest.fixture(scope="module")
def S():
    import sparse_voxel_conv_b200 as S
    return S


@pytest.fixture(scope="module")
def sets():
    wl = WL.make_workload("headline")
    perm = np.random.default_rng(3).permutation(wl.n)
    x = WL.to_bf16_values(WL.make_features(wl.n, 128, 11))
    w = WL.to_bf16_values(WL.make_weight(128, 128, 12))
    return wl, perm, x, w


@pytest.fixture(params=["auto", "brick", "hash"])
def kind(request, monkeypatch):
    """auto: the direct table the headline takes; brick / hash: forced
    (testing knob SUBM3D_MAP_KIND)."""
    if request.param == "auto":
        monkeypatch.delenv("SUBM3D_MAP_KIND", raising=False)
    else:
        monkeypatch.setenv("SUBM3D_MAP_KIND", request.param)
    return request.param


def _dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t if dtype is None else t.to(dtype)


def _sets_on_device(sets):
    wl, perm, x, w = sets
    cA = _dev(wl.coords)
    cB = _dev(wl.coords[perm])
    xA = _dev(x.astype(np.float32), torch.bfloat16)
    xB = _dev(x[perm].astype(np.float32), torch.bfloat16)
    wt = _dev(w.astype(np.float32), torch.bfloat16)
    return {"A": (cA, xA), "B": (cB, xB)}, wt


def test_queued_forwards_match_waited_builds(S, sets, kind):
    wl, perm, x, w = sets
    dev_sets, wt = _sets_on_device(sets)
    n = wl.n
    ref = {}
    for name, (c, xx) in dev_sets.items():
        h = S.build_map(c, wl.grid_dim, wl.batch)  # waits for the build
        ref[name] = S.forward(h, xx, wt, act="gelu")
        torch.cuda.synchronize()
    assert torch.equal(ref["B"], ref["A"][_dev(perm)])  # same voxels, permuted rows
    # the queued outputs of set A against the oracle on sampled rows
    rows = sample_rows(n, 3000, seed=5)
    want = C.forward(C.build_map(wl.coords, wl.grid_dim, wl.batch), np.asarray(x, np.float64),
                     np.asarray(w, np.float64), act="gelu", round_to_bf16=True, rows=rows)
    assert_close(ref["A"].float().cpu().numpy()[rows], want, RTOL_BF16, "waited build, set A")

    nbr = torch.empty((n, 27), dtype=torch.int32, device="cuda")
    work = torch.empty(S._abi.subm3d_map_workspace_bytes(n, wl.grid_dim, wl.batch),
                       dtype=torch.uint8, device="cuda")
    order = "ABABAABBBA"
    outs = [torch.empty((n, 128), dtype=torch.bfloat16, device="cuda") for _ in order]
    for o in outs:
        o.view(torch.int16).fill_(-1)  # NaN
    torch.cuda.synchronize()
    torch.cuda._sleep(SLEEP_CYCLES)
    for name, o in zip(order, outs):
        c, xx = dev_sets[name]
        h = S.build_map(c, wl.grid_dim, wl.batch, check=False, nbr=nbr, workspace=work)
        S.forward(h, xx, wt, act="gelu", out=o)
    torch.cuda.synchronize()
    assert S._abi.subm3d_device_status() == 0
    assert S.map_status(h) == 0
    for k, (name, o) in enumerate(zip(order, outs)):
        unwritten = int(torch.isnan(o.float()).any(dim=1).sum())
        differ = int((o.view(torch.int16) != ref[name].view(torch.int16)).any(dim=1).sum())
        assert unwritten == 0 and differ == 0, (kind, k, name, unwritten, differ)


def test_queued_layers_match_waited_build(S, sets):
    """A build, then two layers on its map, queued three times over: the first
    layer starts right behind the map build, the second right behind the first."""
    wl, perm, x, w = sets
    dev_sets, wt = _sets_on_device(sets)
    c, xx = dev_sets["A"]
    h = S.build_map(c, wl.grid_dim, wl.batch)
    y1 = S.forward(h, xx, wt, act="gelu")
    y2 = S.forward(h, y1, wt)
    torch.cuda.synchronize()
    nbr = torch.empty_like(h.nbr)
    work = torch.empty_like(h.workspace)
    outs = [(torch.empty_like(y1), torch.empty_like(y2)) for _ in range(3)]
    torch.cuda._sleep(SLEEP_CYCLES)
    for o1, o2 in outs:
        hq = S.build_map(c, wl.grid_dim, wl.batch, check=False, nbr=nbr, workspace=work)
        S.forward(hq, xx, wt, act="gelu", out=o1)
        S.forward(hq, o1, wt, out=o2)
    torch.cuda.synchronize()
    assert S._abi.subm3d_device_status() == 0
    for k, (o1, o2) in enumerate(outs):
        assert torch.equal(o1, y1) and torch.equal(o2, y2), k


def test_queued_weight_gradients_match_waited_build(S, sets):
    """The tensor-core weight gradient reads the x-run layout too; queued right
    behind alternating builds it must sum every tile (fp32 atomics: compared at
    the fp32 bar, not bit for bit)."""
    wl, perm, x, w = sets
    dev_sets, wt = _sets_on_device(sets)
    n = wl.n
    g = torch.Generator(device="cuda").manual_seed(9)
    dy = {"A": (torch.randn((n, 128), generator=g, device="cuda") * 0.1).to(torch.bfloat16)}
    dy["B"] = dy["A"][_dev(perm)].contiguous()
    ref = {}
    for name, (c, xx) in dev_sets.items():
        h = S.build_map(c, wl.grid_dim, wl.batch)
        ref[name] = S.backward_weight(h, xx, dy[name])
        torch.cuda.synchronize()
    nbr = torch.empty((n, 27), dtype=torch.int32, device="cuda")
    work = torch.empty(S._abi.subm3d_map_workspace_bytes(n, wl.grid_dim, wl.batch),
                       dtype=torch.uint8, device="cuda")
    order = "ABBA"
    outs = []
    torch.cuda._sleep(SLEEP_CYCLES)
    for name in order:
        c, xx = dev_sets[name]
        h = S.build_map(c, wl.grid_dim, wl.batch, check=False, nbr=nbr, workspace=work)
        outs.append(S.backward_weight(h, xx, dy[name]))
    torch.cuda.synchronize()
    assert S._abi.subm3d_device_status() == 0
    for name, o in zip(order, outs):
        assert_close(o.cpu().numpy(), ref[name].cpu().numpy(), RTOL_F32, f"queued wgrad {name}")
