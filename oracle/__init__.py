"""CPU oracle for the per-group 128x4 blocked layout of MXFP8 E8M0 scales.

TEST INFRASTRUCTURE ONLY.  The product package never imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg do.  The arithmetic lives in ``mx_oracle.c`` (plain single-threaded C,
built with gcc); this file builds it and marshals numpy arrays.  Every
function is pinned by ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "mx_oracle.c")
LIB = os.path.join(HERE, "libmxoracle.so")

DIM_M = 0
DIM_K = 1

_lib = None


def build(force: bool = False, src: str = SRC, out: str = LIB) -> str:
    """Compile the oracle with gcc (-O2, no vectorisation pragmas, one thread)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        cmd = ["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-I", HERE, src, "-o", out + ".tmp"]
        subprocess.run(cmd, check=True)
        os.replace(out + ".tmp", out)
    return out


_I64 = ctypes.c_int64
_I32 = ctypes.c_int32
_P = ctypes.c_void_p


def _bind(lib):
    lib.oracle_rearranged_size.restype = _I64
    lib.oracle_rearranged_size.argtypes = [ctypes.c_int, _I64, _I64, _I32]
    lib.oracle_clamp_ends.restype = None
    lib.oracle_clamp_ends.argtypes = [_P, _I32, _I64, _P]
    lib.oracle_padded_group_starts.restype = ctypes.c_int
    lib.oracle_padded_group_starts.argtypes = [ctypes.c_int, _I64, _I64, _P, _I32, _P]
    for name in ("oracle_read_bytes", "oracle_written_bytes"):
        f = getattr(lib, name)
        f.restype = _I64
        f.argtypes = [ctypes.c_int, _I64, _I64, _P, _I32]
    lib.oracle_rearrange.restype = ctypes.c_int
    lib.oracle_rearrange.argtypes = [ctypes.c_int, _P, _I64, _I64, _I64, _P, _I32, _P, _I64]
    lib.oracle_dest_index.restype = ctypes.c_int
    lib.oracle_dest_index.argtypes = [ctypes.c_int, _I64, _I64, _P, _I32, _P]
    lib.oracle_decode_at.restype = ctypes.c_int
    lib.oracle_decode_at.argtypes = [ctypes.c_int, _I64, _I64, _P, _I32, _P, _I64, _P, _P]
    lib.oracle_gather_at.restype = ctypes.c_int
    lib.oracle_gather_at.argtypes = [ctypes.c_int, _P, _I64, _I64, _I64, _P, _I32, _P, _I64, _P]
    lib.oracle_inverse.restype = ctypes.c_int
    lib.oracle_inverse.argtypes = [ctypes.c_int, _P, _I64, _I64, _I64, _P, _I32, _P]
    return lib


def load(path: str | None = None):
    """Load the oracle library (building it first if needed).  ``path`` loads
    another build of the same source, e.g. a planted-mistake copy in a test."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        build()
        _lib = _bind(ctypes.CDLL(LIB))
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _ends(ends) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(ends, dtype=np.int32))


def rearranged_size(dim: int, rows: int, cols: int, num_groups: int, lib=None) -> int:
    lib = lib or load()
    return int(lib.oracle_rearranged_size(dim, rows, cols, num_groups))


def clamp_ends(ends, limit: int, lib=None) -> np.ndarray:
    lib = lib or load()
    e = _ends(ends)
    out = np.zeros(len(e), dtype=np.int64)
    lib.oracle_clamp_ends(_ptr(e), len(e), limit, _ptr(out))
    return out


def padded_group_starts(dim: int, rows: int, cols: int, ends, lib=None) -> np.ndarray:
    lib = lib or load()
    e = _ends(ends)
    out = np.zeros(len(e) + 1, dtype=np.int64)
    if lib.oracle_padded_group_starts(dim, rows, cols, _ptr(e), len(e), _ptr(out)) != 0:
        raise ValueError("invalid arguments")
    return out


def read_bytes(dim: int, rows: int, cols: int, ends, lib=None) -> int:
    lib = lib or load()
    e = _ends(ends)
    return int(lib.oracle_read_bytes(dim, rows, cols, _ptr(e), len(e)))


def written_bytes(dim: int, rows: int, cols: int, ends, lib=None) -> int:
    lib = lib or load()
    e = _ends(ends)
    return int(lib.oracle_written_bytes(dim, rows, cols, _ptr(e), len(e)))


def _strided(scales: np.ndarray):
    """(buffer, rows, cols, row_stride) of a uint8 2-D array whose last dim is dense."""
    assert scales.dtype == np.uint8 and scales.ndim == 2
    rows, cols = scales.shape
    if rows == 0 or cols == 0:
        return scales, rows, cols, cols
    assert scales.strides[1] == 1 and scales.strides[0] >= cols
    return scales, rows, cols, scales.strides[0]


def rearrange(dim: int, scales: np.ndarray, ends, out_size: int | None = None, lib=None) -> np.ndarray:
    """Scatter form over a (rows, cols) uint8 array (rows may be strided)."""
    lib = lib or load()
    buf, rows, cols, stride = _strided(scales)
    e = _ends(ends)
    size = rearranged_size(dim, rows, cols, len(e), lib) if out_size is None else out_size
    out = np.empty(max(size, 0), dtype=np.uint8)
    base = ctypes.c_void_p(buf.__array_interface__["data"][0])
    if lib.oracle_rearrange(dim, base, rows, cols, stride, _ptr(e), len(e), _ptr(out), size) != 0:
        raise ValueError("invalid arguments")
    return out


def dest_index(dim: int, rows: int, cols: int, ends, lib=None) -> np.ndarray:
    lib = lib or load()
    e = _ends(ends)
    dest = np.empty(rows * cols, dtype=np.int64)
    if lib.oracle_dest_index(dim, rows, cols, _ptr(e), len(e), _ptr(dest)) != 0:
        raise ValueError("invalid arguments")
    return dest.reshape(rows, cols)


def decode_at(dim: int, rows: int, cols: int, ends, pos, lib=None):
    lib = lib or load()
    e = _ends(ends)
    p = np.ascontiguousarray(np.asarray(pos, dtype=np.int64))
    r = np.empty(len(p), dtype=np.int64)
    c = np.empty(len(p), dtype=np.int64)
    if lib.oracle_decode_at(dim, rows, cols, _ptr(e), len(e), _ptr(p), len(p), _ptr(r), _ptr(c)) != 0:
        raise ValueError("invalid arguments")
    return r, c


def gather_at(dim: int, scales: np.ndarray, ends, pos, lib=None) -> np.ndarray:
    lib = lib or load()
    buf, rows, cols, stride = _strided(scales)
    e = _ends(ends)
    p = np.ascontiguousarray(np.asarray(pos, dtype=np.int64))
    vals = np.empty(len(p), dtype=np.uint8)
    base = ctypes.c_void_p(buf.__array_interface__["data"][0])
    if lib.oracle_gather_at(dim, base, rows, cols, stride, _ptr(e), len(e), _ptr(p), len(p), _ptr(vals)) != 0:
        raise ValueError("invalid arguments")
    return vals


def gather(dim: int, scales: np.ndarray, ends, lib=None) -> np.ndarray:
    """Gather form over the whole allocation."""
    rows, cols = scales.shape
    size = rearranged_size(dim, rows, cols, len(_ends(ends)), lib)
    return gather_at(dim, scales, ends, np.arange(size, dtype=np.int64), lib)


def inverse(dim: int, out: np.ndarray, rows: int, cols: int, ends, lib=None) -> np.ndarray:
    lib = lib or load()
    e = _ends(ends)
    o = np.ascontiguousarray(out, dtype=np.uint8)
    s = np.empty((rows, cols), dtype=np.uint8)
    if lib.oracle_inverse(dim, _ptr(o), len(o), rows, cols, _ptr(e), len(e), _ptr(s)) != 0:
        raise ValueError("invalid arguments")
    return s
