"""A set past 2^24 voxels: every cell of 2 x 256^3 (33,554,432 voxels, a
134 MB direct table, 131,072 x-runs of 256, ~1.2 GB of E index table).  On a
full grid the neighbour map has a closed form -- the row of (b, z, y, x) in
raster order is ((b * 256 + z) * 256 + y) * 256 + x -- so sampled rows of the
map are checked bit for bit against it and sampled rows of the bf16 forward
against an fp64 sum over those rows.  (Collected after the other GPU tests,
before the no-allocation test that closes the run.)"""
import numpy as np
import pytest
import torch

import workloads as WL
from tests.helpers import RTOL_BF16, assert_close

pytestmark = pytest.mark.gpu
G, B, C = 256, 2, 64


def _row(b, z, y, x):
    return ((b * G + z) * G + y) * G + x


def test_full_two_by_256_cubed():
    import sparse_voxel_conv_b200 as S
    n = B * G ** 3
    idx = torch.arange(n, device="cuda", dtype=torch.int64)
    coords = torch.stack([idx // G ** 3, (idx // G ** 2) % G, (idx // G) % G, idx % G],
                         1).to(torch.int32).contiguous()
    del idx
    h = S.build_map(coords, G, B)
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([rng.choice(n, 4000, replace=False),
                                     [0, 255, 256 * 255, G ** 3 - 1, G ** 3, n - 1]]))
    nbr = h.nbr[torch.from_numpy(rows).cuda()].cpu().numpy()
    b, rem = np.divmod(rows, G ** 3)
    z, rem = np.divmod(rem, G * G)
    y, x = np.divmod(rem, G)
    expect = np.full((rows.size, 27), -1, np.int64)
    for k in range(27):
        dz, dy, dx = k // 9 - 1, (k // 3) % 3 - 1, k % 3 - 1
        zz, yy, xx = z + dz, y + dy, x + dx
        ok = (zz >= 0) & (zz < G) & (yy >= 0) & (yy < G) & (xx >= 0) & (xx < G)
        expect[ok, k] = _row(b[ok], zz[ok], yy[ok], xx[ok])
    assert np.array_equal(nbr, expect)
    pos, et, hdr = S.run_layout_tensors(h)
    assert hdr.tolist()[:3] == [B * G * G, (n + 2 * B * G * G + 255) // 256, n + 2 * B * G * G]
    # bf16 forward on the x-run kernel; sampled rows against an fp64 sum
    gen = torch.Generator(device="cuda").manual_seed(3)
    feats = torch.randn(n, C, device="cuda", generator=gen).to(torch.bfloat16)
    w = (torch.randn(C, 27, C, device="cuda", generator=gen) / np.sqrt(27 * C)).to(torch.bfloat16)
    y_out = S.forward(h, feats, w)
    torch.cuda.synchronize()
    assert S._abi.subm3d_device_status() == 0
    sel = torch.from_numpy(expect.clip(min=0)).cuda()
    xg = feats[sel.reshape(-1)].reshape(rows.size, 27, C).double().cpu().numpy()
    xg[expect < 0] = 0.0
    ref = np.einsum("okc,rkc->ro", w.double().cpu().numpy(), xg)
    got = y_out[torch.from_numpy(rows).cuda()].float().cpu().numpy()
    assert_close(got, WL.to_bf16_values(ref.astype(np.float32)), RTOL_BF16, "2 x 256^3 forward")
