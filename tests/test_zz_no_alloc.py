"""The allocation-free map build, subm3d_build_map_noalloc, against the
regular workspace build, subm3d_build_map.

Callers that cannot allocate device memory while they run (a plugin whose
host framework owns every device allocation, or a serving loop that must not
call cudaMalloc/cudaFree) use the no-alloc entry point, which keeps its
scratch in a fixed device array inside the library.  Its maps must be the
same as the regular build's, bit for bit, on consecutive calls that share that
array.  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import workloads as WL

pytestmark = pytest.mark.gpu


def _noalloc(A, coords_np, grid, batch):
    c = torch.from_numpy(np.ascontiguousarray(coords_np)).cuda()
    n = c.shape[0]
    nbr = torch.full((n, 27), -7, dtype=torch.int32, device="cuda")
    mask = torch.full(((n + 127) // 128,), -7, dtype=torch.int32, device="cuda")
    st = A.subm3d_build_map_noalloc(c, n, grid, batch, nbr, mask)
    return st, c, nbr, mask


def test_noalloc_matches_workspace_build_on_consecutive_calls():
    import sparse_voxel_conv_b200 as S
    from sparse_voxel_conv_b200 import _abi as A

    cases = [(WL.headline_coords(), 128, 1),
             (WL.shell_coords()[WL.permute_rows(14534, 9)], 64, 1),
             (WL.tiny_coords(), 16, 1)]
    for coords, grid, batch in cases:  # three calls in a row share the scratch array
        st, c, nbr, mask = _noalloc(A, coords, grid, batch)
        assert st == A.SUBM3D_OK, A.subm3d_status_string(st)
        ref = S.build_map(c, grid, batch)
        assert torch.equal(nbr, ref.nbr)
        assert torch.equal(mask, S.tile_mask_tensor(ref))

    # the forward over the no-alloc map equals the forward over the regular map
    coords, grid, batch = cases[0]
    st, c, nbr, mask = _noalloc(A, coords, grid, batch)
    assert st == A.SUBM3D_OK
    ref = S.build_map(c, grid, batch)
    x = torch.from_numpy(WL.make_features(c.shape[0], 128, 1)).cuda().to(torch.bfloat16)
    w = torch.from_numpy(WL.make_weight(128, 128, 2)).cuda().to(torch.bfloat16)
    y_ref = S.forward(ref, x, w)
    y = torch.empty_like(y_ref)
    A.subm3d_forward(nbr, mask, c.shape[0], x, w, y, 128, 128, A.SUBM3D_BF16, False,
                     A.SUBM3D_ACT_NONE)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)


def test_noalloc_wide_keys_match_oracle():
    """batch > 4 or grid_dim > 1024 takes the 64-bit key form, whose hash table
    keeps its rows in a separate region of the fixed scratch array.  Its maps
    are checked against the oracle directly, on two calls in a row."""
    from oracle import cpp as C
    from sparse_voxel_conv_b200 import _abi as A
    from tests.helpers import masks_from_nbr

    parts = []
    for b in range(5):                                    # batch 5: wide keys
        c = WL.tiny_coords(seed=30 + b)
        c[:, 0] = b
        parts.append(c)
    five = np.concatenate(parts)[WL.permute_rows(sum(len(p) for p in parts), 31)]
    far = WL.tiny_coords(seed=32)
    far[:, 1:] += 1500                                    # grid 2048: wide keys
    for coords, grid, batch in ((five, 16, 5), (far, 2048, 1)):
        st, c, nbr, mask = _noalloc(A, coords, grid, batch)
        assert st == A.SUBM3D_OK, A.subm3d_status_string(st)
        ref = C.build_map(coords, grid, batch)
        assert np.array_equal(nbr.cpu().numpy(), ref)
        words = mask.cpu().numpy().view(np.uint32).astype(np.int64)
        assert np.array_equal(words, masks_from_nbr(ref))


def test_noalloc_reports_data_errors_and_rejects_oversize():
    from sparse_voxel_conv_b200 import _abi as A

    dup = np.concatenate([WL.tiny_coords(), WL.tiny_coords()[5:6]])
    assert _noalloc(A, dup, 16, 1)[0] == A.SUBM3D_E_DUPLICATE
    bad = np.concatenate([WL.tiny_coords(), np.array([[0, 0, 0, 16]], np.int32)])
    assert _noalloc(A, bad, 16, 1)[0] == A.SUBM3D_E_RANGE
    # the next call after a failed one is clean again
    st, c, nbr, mask = _noalloc(A, WL.tiny_coords(), 16, 1)
    assert st == A.SUBM3D_OK
    big = A.SUBM3D_NOALLOC_MAX_VOXELS + 1
    st = A.subm3d_build_map_noalloc(c.data_ptr(), big, 16, 1, nbr.data_ptr(), mask.data_ptr())
    assert st == A.SUBM3D_E_UNSUPPORTED
