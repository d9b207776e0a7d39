"""ctypes binding of libsubm3d.so (include/subm3d.h): argument marshalling only.

Each function has the C name and passes torch tensors' device pointers and
the current CUDA stream straight through.  Nothing here computes any part of
the convolution; if the shared library is missing the import fails loudly,
there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsubm3d.so")

SUBM3D_OK = 0
SUBM3D_E_INVALID = 1
SUBM3D_E_RANGE = 2
SUBM3D_E_DUPLICATE = 3
SUBM3D_E_TABLE_FULL = 4
SUBM3D_E_UNSUPPORTED = 5
SUBM3D_E_CUDA = 6
SUBM3D_E_TIMEOUT = 7

SUBM3D_F32 = 0
SUBM3D_BF16 = 1
SUBM3D_ACT_NONE = 0
SUBM3D_ACT_GELU = 1
SUBM3D_ACT_SILU = 2
SUBM3D_KVOL = 27
SUBM3D_EXPAND_SUBDIVIDE = 0
SUBM3D_EXPAND_UPSAMPLE = 1
SUBM3D_EXPAND_CHANNEL2SPATIAL = 2
SUBM3D_POOL_MAX = 0
SUBM3D_POOL_MEAN = 1
SUBM3D_POOL_SPATIAL2CHANNEL = 2
SUBM3D_TILE_ROWS = 128


class Subm3dError(RuntimeError):
    """A non-OK subm3d_status returned by the library."""

    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {subm3d_status_string(status)} (status {status})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m sparse_voxel_conv_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "subm3d_abi_version": (i32, []),
        "subm3d_status_string": (ctypes.c_char_p, [i32]),
        "subm3d_map_workspace_bytes": (sz, [i64, i32, i32]),
        "subm3d_build_map": (ctypes.c_int, [vp, i64, i32, i32, vp, vp, sz, vp,
                                            ctypes.POINTER(vp)]),
        "subm3d_map_status": (ctypes.c_int, [vp]),
        "subm3d_map_nbr": (vp, [vp]),
        "subm3d_map_tile_mask": (vp, [vp]),
        "subm3d_map_size": (i64, [vp]),
        "subm3d_map_table": (ctypes.c_int32, [vp]),
        "subm3d_map_destroy": (None, [vp]),
        "subm3d_forward": (ctypes.c_int, [vp, vp, i64, vp, vp, vp, i32, i32, ctypes.c_int, i32,
                                          ctypes.c_int, vp]),
        "subm3d_device_status": (ctypes.c_int, [vp]),
        "subm3d_build_map_noalloc": (ctypes.c_int, [vp, i64, i32, i32, vp, vp, vp]),
        "subm3d_forward_map": (ctypes.c_int, [vp, vp, vp, vp, i32, i32, ctypes.c_int, i32,
                                              ctypes.c_int, vp]),
        "subm3d_map_run_layout": (ctypes.c_int, [vp, ctypes.POINTER(vp), ctypes.POINTER(vp),
                                                 ctypes.POINTER(vp)]),
        "subm3d_forward_fused": (ctypes.c_int, [vp, vp, vp, vp, vp, vp, i32, i32, ctypes.c_int,
                                                i32, ctypes.c_int, vp]),
        "subm3d_backward_data": (ctypes.c_int, [vp, vp, vp, vp, vp, i32, i32, ctypes.c_int, i32,
                                                vp]),
        "subm3d_expand_workspace_bytes": (sz, [i64]),
        "subm3d_expand": (ctypes.c_int, [vp, vp, vp, i64, i32, ctypes.c_int, ctypes.c_int, vp, vp,
                                         vp, sz, ctypes.POINTER(i64), vp]),
        "subm3d_pool_workspace_bytes": (sz, [i64, i32, i32]),
        "subm3d_pool": (ctypes.c_int, [vp, vp, vp, i32, ctypes.c_int, ctypes.c_int, vp, vp, vp, sz,
                                       ctypes.POINTER(i64), vp]),
        "subm3d_backward_weight": (ctypes.c_int, [vp, vp, vp, vp, i32, i32, ctypes.c_int, i32,
                                                  vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _check(status: int, where: str) -> None:
    if status != SUBM3D_OK:
        raise Subm3dError(status, where)


def subm3d_abi_version() -> int:
    return int(lib.subm3d_abi_version())


def subm3d_status_string(status: int) -> str:
    return lib.subm3d_status_string(int(status)).decode()


def subm3d_map_workspace_bytes(n: int, grid_dim: int, batch: int) -> int:
    return int(lib.subm3d_map_workspace_bytes(int(n), int(grid_dim), int(batch)))


class MapHandle:
    """Owns a subm3d_map* and keeps the tensors it points into alive."""

    def __init__(self, ptr: int, n: int, grid_dim: int, batch: int, nbr, workspace):
        self._ptr = ptr
        self.n = int(n)
        self.grid_dim = int(grid_dim)
        self.batch = int(batch)
        self.nbr = nbr
        self.workspace = workspace

    @property
    def ptr(self) -> int:
        return self._ptr

    def close(self) -> None:
        if self._ptr:
            lib.subm3d_map_destroy(self._ptr)
            self._ptr = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def subm3d_build_map(coords, n: int, grid_dim: int, batch: int, nbr, workspace,
                     workspace_bytes: int | None = None, stream=None) -> MapHandle:
    """Enqueue the map build; raises Subm3dError on an argument error."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    out = ctypes.c_void_p()
    st = lib.subm3d_build_map(_ptr(coords), int(n), int(grid_dim), int(batch), _ptr(nbr),
                              _ptr(workspace), int(workspace_bytes), _stream(stream),
                              ctypes.byref(out))
    _check(st, "subm3d_build_map")
    return MapHandle(out.value, n, grid_dim, batch, nbr, workspace)


def subm3d_map_status(handle: MapHandle) -> int:
    """Blocking: the device-detected status of the build (an int status code)."""
    return int(lib.subm3d_map_status(handle.ptr))


def subm3d_map_nbr(handle: MapHandle) -> int:
    return int(lib.subm3d_map_nbr(handle.ptr) or 0)


def subm3d_map_tile_mask(handle: MapHandle) -> int:
    return int(lib.subm3d_map_tile_mask(handle.ptr) or 0)


def subm3d_map_size(handle: MapHandle) -> int:
    return int(lib.subm3d_map_size(handle.ptr))


SUBM3D_TABLE_DIRECT, SUBM3D_TABLE_HASH, SUBM3D_TABLE_BRICK = 0, 1, 2


def subm3d_map_table(handle: MapHandle) -> int:
    """The lookup table the build chose: SUBM3D_TABLE_DIRECT, _HASH or _BRICK."""
    return int(lib.subm3d_map_table(handle.ptr))


def subm3d_forward(nbr, tile_mask, n: int, feats, weight, out, cin: int, cout: int,
                   dtype: int, flip: bool, act: int, stream=None) -> None:
    """Enqueue one layer's forward; raises Subm3dError on an argument error."""
    st = lib.subm3d_forward(_ptr(nbr), _ptr(tile_mask), int(n), _ptr(feats), _ptr(weight),
                            _ptr(out), int(cin), int(cout), int(dtype), 1 if flip else 0,
                            int(act), _stream(stream))
    _check(st, "subm3d_forward")


def subm3d_forward_map(handle: MapHandle, feats, weight, out, cin: int, cout: int, dtype: int,
                       flip: bool, act: int, stream=None) -> None:
    """Enqueue one layer's forward over a built map (x-run kernel for bf16 with
    Cin >= 48); raises Subm3dError on an argument error."""
    st = lib.subm3d_forward_map(handle.ptr, _ptr(feats), _ptr(weight), _ptr(out), int(cin),
                                int(cout), int(dtype), 1 if flip else 0, int(act),
                                _stream(stream))
    _check(st, "subm3d_forward_map")


def subm3d_forward_fused(handle: MapHandle, feats, weight, bias, residual, out, cin: int,
                         cout: int, dtype: int, flip: bool, act: int, stream=None) -> None:
    """Enqueue one layer with the residual-block epilogue act(conv + bias) +
    residual (bias / residual may be None); raises Subm3dError on an argument
    error."""
    st = lib.subm3d_forward_fused(handle.ptr, _ptr(feats), _ptr(weight), _ptr(bias),
                                  _ptr(residual), _ptr(out), int(cin), int(cout), int(dtype),
                                  1 if flip else 0, int(act), _stream(stream))
    _check(st, "subm3d_forward_fused")


def subm3d_backward_data(handle: MapHandle, dy, weight, weight_t, dx, cin: int, cout: int,
                         dtype: int, flip: bool, stream=None) -> None:
    """Enqueue dx = the input gradient (W^T into weight_t, then the forward)."""
    st = lib.subm3d_backward_data(handle.ptr, _ptr(dy), _ptr(weight), _ptr(weight_t), _ptr(dx),
                                  int(cin), int(cout), int(dtype), 1 if flip else 0,
                                  _stream(stream))
    _check(st, "subm3d_backward_data")


def subm3d_backward_weight(handle: MapHandle, feats, dy, dweight, cin: int, cout: int,
                           dtype: int, flip: bool, stream=None) -> None:
    """Enqueue dweight (fp32 KRSC) = the weight gradient."""
    st = lib.subm3d_backward_weight(handle.ptr, _ptr(feats), _ptr(dy), _ptr(dweight), int(cin),
                                    int(cout), int(dtype), 1 if flip else 0, _stream(stream))
    _check(st, "subm3d_backward_weight")


def subm3d_expand_workspace_bytes(n: int) -> int:
    return int(lib.subm3d_expand_workspace_bytes(int(n)))


def subm3d_expand(coords, feats, mask, n: int, channels_out: int, dtype: int, mode: int,
                  out_coords, out_feats, workspace, workspace_bytes: int, stream=None) -> int:
    """Enqueue an expansion; returns the number of child rows (blocking with a mask)."""
    count = ctypes.c_int64(0)
    st = lib.subm3d_expand(_ptr(coords), _ptr(feats), _ptr(mask), int(n), int(channels_out),
                           int(dtype), int(mode), _ptr(out_coords), _ptr(out_feats),
                           _ptr(workspace), int(workspace_bytes), ctypes.byref(count),
                           _stream(stream))
    _check(st, "subm3d_expand")
    return int(count.value)


def subm3d_pool_workspace_bytes(n: int, grid_dim: int, batch: int) -> int:
    return int(lib.subm3d_pool_workspace_bytes(int(n), int(grid_dim), int(batch)))


def subm3d_pool(handle: MapHandle, coords, feats, channels: int, dtype: int, mode: int,
                out_coords, out_feats, workspace, workspace_bytes: int, stream=None) -> int:
    """Pool to parents coord // 2 (blocking); returns the number of parents."""
    count = ctypes.c_int64(0)
    st = lib.subm3d_pool(handle.ptr, _ptr(coords), _ptr(feats), int(channels), int(dtype),
                         int(mode), _ptr(out_coords), _ptr(out_feats), _ptr(workspace),
                         int(workspace_bytes), ctypes.byref(count), _stream(stream))
    _check(st, "subm3d_pool")
    return int(count.value)


def subm3d_map_run_layout(handle: MapHandle):
    """Device pointers (position table, E index table, header) of the map."""
    pos, et, hdr = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_void_p()
    _check(lib.subm3d_map_run_layout(handle.ptr, ctypes.byref(pos), ctypes.byref(et),
                                     ctypes.byref(hdr)), "subm3d_map_run_layout")
    return int(pos.value), int(et.value), int(hdr.value)


def subm3d_device_status(stream=None) -> int:
    """Blocking: SUBM3D_E_TIMEOUT if a forward kernel gave up a bounded wait."""
    return int(lib.subm3d_device_status(_stream(stream)))


SUBM3D_NOALLOC_MAX_VOXELS = 524288


def subm3d_build_map_noalloc(coords, n: int, grid_dim: int, batch: int, nbr, tile_mask,
                             stream=None) -> int:
    """Allocation-free map build into caller-given nbr [N, 27] and tile_mask
    [ceil(N/128)] buffers, using the library's fixed scratch array.  Blocking;
    returns the status code (no exception), as the C function does."""
    return int(lib.subm3d_build_map_noalloc(_ptr(coords), int(n), int(grid_dim), int(batch),
                                            _ptr(nbr), _ptr(tile_mask), _stream(stream)))
