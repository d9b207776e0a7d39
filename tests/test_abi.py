"""The C ABI library loads, exports every symbol include/*.h declares, and
rejects bad arguments on the host before touching the device.  CPU only:
no call here reaches a CUDA kernel."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def abi():
    from sparse_voxel_conv_b200 import build
    build.build()
    from sparse_voxel_conv_b200 import _abi
    return _abi


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        txt = open(h).read()
        txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
        names |= set(re.findall(r"SUBM3D_API\s+[\w\s\*]*?\b(subm3d_\w+)\s*\(", txt))
    return names


def test_exports_every_declared_symbol(abi):
    names = _declared()
    assert len(names) >= 11
    lib = ctypes.CDLL(abi.LIB_PATH)
    for name in sorted(names):
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"


def test_version_and_strings(abi):
    assert abi.subm3d_abi_version() == 1
    for st in range(8):
        assert abi.subm3d_status_string(st) not in ("", "unknown status")
    assert abi.subm3d_status_string(99) == "unknown status"


def _expected_ws(n, table_bytes):
    """Workspace layout: 256-B status block, tile masks, lookup table, run-start
    counts (one int32 per 128-row tile, one per 128 tiles), 256-B header,
    position table (3N rounded to 256, + 256), E index table (9 lines of
    pos_max + 4 int32); 256-B aligned parts."""
    up = lambda v: (v + 255) // 256 * 256
    head = up(256 + 4 * ((n + 127) // 128))
    tiles = (n + 127) // 128
    pos_max = up(3 * n) + 256
    after_table = up(head + table_bytes)
    pos_off = up(up(after_table + 4 * tiles) + 4 * ((tiles + 127) // 128)) + 256
    et_off = up(pos_off + 4 * pos_max)
    return up(et_off + 9 * (pos_max + 4) * 4)


def _brick_bytes(n, grid, batch):
    """Brick table: an int32 directory over the bordered grids in bricks of
    8 (x) x 4 (y) x 2 (z) cells, then min(N, bricks) blocks of 64 int32 cells."""
    up = lambda v: (v + 255) // 256 * 256
    g2 = grid + 2
    dirn = batch * ((g2 + 1) // 2) * ((g2 + 3) // 4) * ((g2 + 7) // 8)
    return up(4 * dirn) + 256 * max(1, min(n, dirn))


def test_workspace_bytes(abi, monkeypatch):
    monkeypatch.delenv("SUBM3D_MAP_KIND", raising=False)
    monkeypatch.delenv("SUBM3D_TABLE_CAPACITY", raising=False)
    f = abi.subm3d_map_workspace_bytes
    assert f(-1, 16, 1) == 0 and f(10, 0, 1) == 0 and f(10, 16, 0) == 0
    assert f(10, 70000, 1) == 0 and f(10, 16, 70000) == 0
    n = 329839
    # direct table: one int32 per cell of each bordered grid, (grid + 2)^3 cells,
    # while that fits max(64 MB, 256 B x N) and is at most 64 MB or 16 cells per voxel
    up = lambda v: (v + 255) // 256 * 256
    assert f(n, 128, 1) == _expected_ws(n, up(4 * 130 ** 3))
    small = 1000                                     # budget 64 MB
    assert f(small, 254, 1) == _expected_ws(small, up(4 * 256 ** 3))   # exactly 64 MB
    assert f(small, 255, 1) == _expected_ws(small, _brick_bytes(small, 255, 1))  # just over
    dense = 2_097_152                                # 130^3 cells, 1.05 per voxel
    assert f(dense, 128, 1) == _expected_ws(dense, up(4 * 130 ** 3))
    # sparser volumes: the brick table while its directory fits the budget
    big = 1_135_307                                  # 4 x 258^3 cells = 60 per voxel
    assert f(big, 256, 4) == _expected_ws(big, _brick_bytes(big, 256, 4))
    assert f(n, 256, 4) == _expected_ws(n, _brick_bytes(n, 256, 4))
    assert f(n, 512, 1) == _expected_ws(n, _brick_bytes(n, 512, 1))
    # beyond: hash table, 8-byte slots, capacity max(1024, pow2 >= 2N); wide keys
    # (batch > 4 or grid > 1024) add a 4-byte row array
    assert f(n, 2048, 1) == _expected_ws(n, 12 * (1 << 20))
    assert f(1000, 4000, 1) == _expected_ws(1000, 12 * 2048)
    monkeypatch.setenv("SUBM3D_MAP_KIND", "direct")  # where it fits
    assert f(big, 256, 4) == _expected_ws(big, up(4 * 4 * 258 ** 3))
    assert f(n, 512, 1) == _expected_ws(n, _brick_bytes(n, 512, 1))
    monkeypatch.setenv("SUBM3D_MAP_KIND", "brick")
    assert f(n, 128, 1) == _expected_ws(n, _brick_bytes(n, 128, 1))
    monkeypatch.setenv("SUBM3D_MAP_KIND", "hash")
    assert f(n, 128, 1) == _expected_ws(n, 8 * (1 << 20))
    assert f(n, 128, 5) == _expected_ws(n, 12 * (1 << 20))
    assert f(0, 16, 1) > 0


def test_build_map_argument_errors(abi):
    lib = abi.lib
    out = ctypes.c_void_p()
    ws = abi.subm3d_map_workspace_bytes(100, 16, 1)
    A = 1 << 20  # a 256-byte aligned fake address; never dereferenced on these paths
    E_INVALID, E_UNSUP = abi.SUBM3D_E_INVALID, abi.SUBM3D_E_UNSUPPORTED
    assert lib.subm3d_build_map(A, 100, 16, 1, A, A, ws, None, None) == E_INVALID
    assert lib.subm3d_build_map(None, 100, 16, 1, A, A, ws, None, ctypes.byref(out)) == E_INVALID
    assert lib.subm3d_build_map(A, -1, 16, 1, A, A, ws, None, ctypes.byref(out)) == E_INVALID
    assert lib.subm3d_build_map(A, 100, 16, 1, A, A, ws - 1, None, ctypes.byref(out)) == E_INVALID
    assert lib.subm3d_build_map(A + 4, 100, 16, 1, A, A, ws, None, ctypes.byref(out)) == E_INVALID
    assert lib.subm3d_build_map(A, 100, 16, 1, A, A + 16, ws, None, ctypes.byref(out)) == E_INVALID
    assert lib.subm3d_build_map(A, 100, 0, 1, A, A, ws, None, ctypes.byref(out)) == E_INVALID
    assert lib.subm3d_build_map(A, 100, 70000, 1, A, A, ws, None, ctypes.byref(out)) == E_UNSUP
    assert out.value is None


def test_forward_argument_errors(abi):
    lib = abi.lib
    A, B, W = 1 << 20, 1 << 24, 1 << 28   # disjoint fake addresses
    E_INVALID, E_UNSUP, OK = abi.SUBM3D_E_INVALID, abi.SUBM3D_E_UNSUPPORTED, abi.SUBM3D_OK
    f = lib.subm3d_forward
    # n = 0 is a no-op
    assert f(None, None, 0, None, None, None, 16, 16, 1, 0, 0, None) == OK
    assert f(A, None, -1, A, W, B, 16, 16, 1, 0, 0, None) == E_INVALID
    assert f(A, None, 10, A, W, B, 0, 16, 1, 0, 0, None) == E_INVALID
    assert f(A, None, 10, None, W, B, 16, 16, 1, 0, 0, None) == E_INVALID
    assert f(A, None, 10, A, W, B, 16, 16, 7, 0, 0, None) == E_INVALID     # bad dtype
    assert f(A, None, 10, A, W, B, 16, 16, 1, 0, 9, None) == E_INVALID     # bad act
    assert f(A, None, 10, A, W, A + 64, 16, 16, 1, 0, 0, None) == E_INVALID  # out overlaps feats
    assert f(A, None, 10, A, W, B, 8, 16, 1, 0, 0, None) == E_UNSUP        # bf16 Cin % 16
    assert f(A, None, 10, A, W, B, 16, 24, 1, 0, 0, None) == E_UNSUP       # bf16 Cout % 16
    assert f(A, None, 10, A + 8, W, B, 16, 16, 1, 0, 0, None) == E_UNSUP   # bf16 alignment
    assert f(A, None, 10, A + 2, W, B, 3, 5, 0, 0, 0, None) == E_INVALID   # f32 alignment


def test_resample_and_backward_argument_errors(abi):
    """Host-side checks of the newer entry points: no CUDA call is reached."""
    lib = abi.lib
    cnt = ctypes.c_int64(5)
    E_INVALID = abi.SUBM3D_E_INVALID
    A = 1 << 20
    assert abi.subm3d_expand_workspace_bytes(-1) == 0
    assert abi.subm3d_expand_workspace_bytes(1000) > 8 * 1000 * 8
    assert abi.subm3d_pool_workspace_bytes(10, 0, 1) == 0
    assert abi.subm3d_pool_workspace_bytes(10, 64, 1) >= 32 ** 3
    # expand: no count pointer, bad mode, subdivide with a mask, upsample without one
    assert lib.subm3d_expand(A, A, None, 10, 8, abi.SUBM3D_F32, 0, A, A, A, 1 << 20, None,
                             None) == E_INVALID
    assert lib.subm3d_expand(A, A, None, 10, 8, abi.SUBM3D_F32, 7, A, A, A, 1 << 20,
                             ctypes.byref(cnt), None) == E_INVALID and cnt.value == 0
    assert lib.subm3d_expand(A, A, A, 10, 8, abi.SUBM3D_F32, abi.SUBM3D_EXPAND_SUBDIVIDE, A, A,
                             A, 1 << 20, ctypes.byref(cnt), None) == E_INVALID
    assert lib.subm3d_expand(A, A, None, 10, 8, abi.SUBM3D_F32, abi.SUBM3D_EXPAND_UPSAMPLE, A, A,
                             A, 1 << 20, ctypes.byref(cnt), None) == E_INVALID
    # expand: workspace too small, misaligned coordinates
    assert lib.subm3d_expand(A, A, None, 10, 8, abi.SUBM3D_F32, 0, A, A, A, 16,
                             ctypes.byref(cnt), None) == E_INVALID
    assert lib.subm3d_expand(A + 4, A, None, 10, 8, abi.SUBM3D_F32, 0, A, A, A, 1 << 20,
                             ctypes.byref(cnt), None) == E_INVALID
    # empty expansion: nothing to do, count 0
    assert lib.subm3d_expand(None, None, None, 0, 8, abi.SUBM3D_F32, 0, None, None, None, 0,
                             ctypes.byref(cnt), None) == abi.SUBM3D_OK and cnt.value == 0
    # pool / backward need a map handle
    assert lib.subm3d_pool(None, A, A, 8, abi.SUBM3D_F32, 0, A, A, A, 1 << 20, ctypes.byref(cnt),
                           None) == E_INVALID
    assert lib.subm3d_backward_data(None, A, A, A, A, 8, 8, abi.SUBM3D_F32, 0, None) == E_INVALID
    assert lib.subm3d_backward_weight(None, A, A, A, 8, 8, abi.SUBM3D_F32, 0, None) == E_INVALID
    assert lib.subm3d_forward_fused(None, A, A, None, None, A, 8, 8, abi.SUBM3D_F32, 0, 0,
                                    None) == E_INVALID
