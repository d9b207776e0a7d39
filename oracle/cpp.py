"""ctypes wrapper around the C++ oracle (subm3d_oracle.cpp).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).  build() compiles the
shared library next to the source with g++ and OpenMP; load() builds it on
first use when it is missing or older than its source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_DIR = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_DIR, "subm3d_oracle.cpp")
_LIB = os.path.join(_DIR, "liboracle.so")
_lib = None


class OracleError(ValueError):
    """A coordinate set the op does not accept (out of range or duplicated)."""


def build(force: bool = False) -> str:
    """Compile liboracle.so (g++ -O2 -fopenmp) if missing or stale; return its path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fopenmp", "-shared", "-fPIC",
                               _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


def load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64p = ctypes.POINTER(ctypes.c_int64)
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_build_map.restype = ctypes.c_int
        lib.oracle_build_map.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                                         ctypes.c_int32, ctypes.c_void_p]
        lib.oracle_forward.restype = None
        lib.oracle_forward.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                       ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
        lib.oracle_backward_data.restype = None
        lib.oracle_backward_data.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                             ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32,
                                             ctypes.c_int32, ctypes.c_void_p]
        lib.oracle_backward_weight.restype = None
        lib.oracle_backward_weight.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                               ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32,
                                               ctypes.c_int32, ctypes.c_void_p]
        lib.oracle_gelu.argtypes = [ctypes.c_void_p, ctypes.c_int64]
        lib.oracle_silu.argtypes = [ctypes.c_void_p, ctypes.c_int64]
        lib.oracle_round_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64]
        del i64p
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(load().oracle_num_threads())


def build_map(coords, grid_dim: int, batch: int = 1) -> np.ndarray:
    """nbr int32 [N, 27] (see subm3d_oracle.cpp, oracle_build_map)."""
    c = np.ascontiguousarray(coords, np.int32)
    n = c.shape[0]
    nbr = np.empty((n, 27), np.int32)
    rc = load().oracle_build_map(c.ctypes.data, n, int(grid_dim), int(batch), nbr.ctypes.data)
    if rc == 2:
        raise OracleError("coordinate out of range")
    if rc == 3:
        raise OracleError("duplicate coordinate")
    if rc != 0:
        raise OracleError(f"oracle_build_map returned {rc}")
    return nbr


def forward(nbr, x, w, flip: bool = False, act: str | None = None,
            round_to_bf16: bool = False, rows=None, bias=None, residual=None) -> np.ndarray:
    """fp64 forward over all rows or a subset (see oracle_forward), then the
    epilogue act(sum + bias) + residual and an optional bf16 rounding."""
    nbr = np.ascontiguousarray(nbr, np.int32)
    x = np.ascontiguousarray(x, np.float64)
    w = np.ascontiguousarray(w, np.float64)
    cout = w.shape[0]
    cin = x.shape[1]
    assert w.size == cout * 27 * cin
    if rows is None:
        rows_arr, n_rows, rows_ptr = None, nbr.shape[0], None
    else:
        rows_arr = np.ascontiguousarray(rows, np.int64)
        n_rows, rows_ptr = rows_arr.shape[0], rows_arr.ctypes.data
    out = np.empty((n_rows, cout), np.float64)
    load().oracle_forward(nbr.ctypes.data, x.ctypes.data, w.ctypes.data, cin, cout,
                          1 if flip else 0, rows_ptr, n_rows, out.ctypes.data)
    if bias is not None:
        out += np.asarray(bias, np.float64)[None, :]
    if act == "gelu":
        load().oracle_gelu(out.ctypes.data, out.size)
    elif act == "silu":
        load().oracle_silu(out.ctypes.data, out.size)
    elif act is not None:
        raise ValueError(f"unknown activation {act!r}")
    if residual is not None:
        res = np.asarray(residual, np.float64)
        out += res if rows_arr is None else res[rows_arr]
    if round_to_bf16:
        load().oracle_round_bf16(out.ctypes.data, out.size)
    return out


def backward_data(nbr, dy, w, flip: bool = False) -> np.ndarray:
    """fp64 gradient with respect to the input features (see oracle_backward_data)."""
    nbr = np.ascontiguousarray(nbr, np.int32)
    dy = np.ascontiguousarray(dy, np.float64)
    w = np.ascontiguousarray(w, np.float64)
    cout = w.shape[0]
    cin = w.size // (27 * cout)
    dx = np.empty((nbr.shape[0], cin), np.float64)
    load().oracle_backward_data(nbr.ctypes.data, nbr.shape[0], dy.ctypes.data, w.ctypes.data,
                                cin, cout, 1 if flip else 0, dx.ctypes.data)
    return dx


def backward_weight(nbr, x, dy, flip: bool = False) -> np.ndarray:
    """fp64 gradient with respect to the KRSC weight, [Cout, 3, 3, 3, Cin]."""
    nbr = np.ascontiguousarray(nbr, np.int32)
    x = np.ascontiguousarray(x, np.float64)
    dy = np.ascontiguousarray(dy, np.float64)
    cin, cout = x.shape[1], dy.shape[1]
    dw = np.empty((cout, 27, cin), np.float64)
    load().oracle_backward_weight(nbr.ctypes.data, nbr.shape[0], x.ctypes.data, dy.ctypes.data,
                                  cin, cout, 1 if flip else 0, dw.ctypes.data)
    return dw.reshape(cout, 3, 3, 3, cin)


def gelu(v) -> np.ndarray:
    v = np.array(v, np.float64, copy=True, order="C")
    load().oracle_gelu(v.ctypes.data, v.size)
    return v


def silu(v) -> np.ndarray:
    v = np.array(v, np.float64, copy=True, order="C")
    load().oracle_silu(v.ctypes.data, v.size)
    return v


def round_bf16(v) -> np.ndarray:
    v = np.array(v, np.float64, copy=True, order="C")
    load().oracle_round_bf16(v.ctypes.data, v.size)
    return v
