"""The epilogue activations element by element, through the fp32 forward.

On a set of isolated voxels (coordinates two apart on every axis, so no voxel
has a neighbour) with the centre weight slice the identity and every other
slice zero, the fp32 convolution sum is exactly the input, so the output is
act(x) element-wise.  GELU (erf form; erfc by the Abramowitz & Stegun 7.1.26
approximation, absolute error <= 1.5e-7, plus fp32 rounding and the fast
exponential and divide) and SiLU (fast exponential and divide) are checked
against fp64 over [-12, 12] and a few special values, with a bar of
2e-6 * max(1, |x|)."""
import math

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu
C = 16


def _isolated_set(m=16):
    i = np.arange(m)
    z, y, x = np.meshgrid(i, i, i, indexing="ij")
    c = np.stack([np.zeros(m ** 3, np.int64), 2 * z.ravel(), 2 * y.ravel(), 2 * x.ravel()], 1)
    return c.astype(np.int32), 2 * m


def _ref(act, x):
    x = x.astype(np.float64)
    if act == "gelu":
        return np.array([0.5 * v * (1.0 + math.erf(v / math.sqrt(2.0))) for v in x.ravel()]
                        ).reshape(x.shape)
    return x / (1.0 + np.exp(-x))


@pytest.mark.parametrize("act", ["gelu", "silu"])
def test_activation_elementwise_fp32(act):
    import sparse_voxel_conv_b200 as S
    coords, grid = _isolated_set()
    n = coords.shape[0]
    vals = np.linspace(-12.0, 12.0, n * C - 8, dtype=np.float32)
    vals = np.concatenate([vals, np.array([0.0, -0.0, 1e-30, -1e-30, 1e-4, -1e-4, 30.0, -30.0],
                                          np.float32)])
    x = vals.reshape(n, C)
    w = np.zeros((C, 27, C), np.float32)
    w[:, 13, :] = np.eye(C, dtype=np.float32)
    h = S.build_map(torch.from_numpy(coords).cuda(), grid, 1)
    assert int((h.nbr >= 0).sum().item()) == n  # the centre only
    y = S.forward(h, torch.from_numpy(x).cuda(), torch.from_numpy(w).cuda(), act=act)
    torch.cuda.synchronize()
    assert S._abi.subm3d_device_status() == 0
    y = y.cpu().numpy().astype(np.float64)
    ref = _ref(act, x)
    err = np.abs(y - ref)
    bound = 2e-6 * np.maximum(1.0, np.abs(x.astype(np.float64)))
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), (act, x[worst], y[worst], ref[worst])
