"""ctypes binding of libmxscale's C ABI (include/mxscale.h).

Argument marshalling only: every step of the rearrange runs in the library's
CUDA kernels.  The library is loaded from this package directory; if it is
missing the first call raises, there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmxscale.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "mxscale.h")

MX_OK, MX_ERR_INVALID_ARG, MX_ERR_MISALIGNED, MX_ERR_UNSUPPORTED, MX_ERR_CUDA = range(5)
MX_GROUPS_M, MX_GROUPS_K = 0, 1
MX_PATH_AUTO, MX_PATH_TMA, MX_PATH_WORD, MX_PATH_BYTE, MX_PATH_FLAT = range(5)
MX_MAX_GROUPS = 64
PATHS = {"auto": MX_PATH_AUTO, "tma": MX_PATH_TMA, "word": MX_PATH_WORD, "byte": MX_PATH_BYTE,
         "flat": MX_PATH_FLAT}
PATH_NAMES = {v: k for k, v in PATHS.items()}

_lock = threading.Lock()
_lib = None

_I64, _I32, _P, _U32P = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.POINTER(ctypes.c_uint32)

_SIGNATURES = {
    "mx_rearranged_size": (ctypes.c_size_t, [ctypes.c_int, _I64, _I64, _I32]),
    "mx_rearrange_m_groups": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _I32, _P, _P]),
    "mx_rearrange_k_groups": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _I32, _P, _P]),
    "mx_rearrange_ex": (ctypes.c_int, [ctypes.c_int, _P, _I64, _I64, _I64, _P, _I32, _P, ctypes.c_int, _P]),
    "mx_select_path": (ctypes.c_int, [ctypes.c_int, _P, _I64, _I64, _I64]),
    "mx_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "mx_device_flags": (ctypes.c_int, [_U32P, ctypes.c_int]),
    "mx_selftest_bounded_wait": (ctypes.c_int, [_I64, _P]),
    "mx_unrearrange_m_groups": (ctypes.c_int, [_P, _I64, _I64, _P, _I32, _P, _I64, _P]),
    "mx_unrearrange_k_groups": (ctypes.c_int, [_P, _I64, _I64, _P, _I32, _P, _I64, _P]),
    "mx_padded_group_starts": (ctypes.c_int, [ctypes.c_int, _I64, _I64, _P, _I32, _P, _P]),
    "mx_last_cuda_error": (ctypes.c_int, []),
    "mx_version": (ctypes.c_int, []),
}


class MxError(RuntimeError):
    def __init__(self, where: str, status: int):
        extra = f", CUDA error {mx_last_cuda_error()}" if status == MX_ERR_CUDA else ""
        super().__init__(f"{where}: {status_string(status)} (status {status}{extra})")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(
                        f"libmxscale.so is missing at {LIB_PATH}; build it with "
                        "`python -m scale_factor_layout_b200._build` (nvcc, sm_100a)")
                handle = ctypes.CDLL(LIB_PATH)
                for name, (res, args) in _SIGNATURES.items():
                    f = getattr(handle, name)
                    f.restype, f.argtypes = res, args
                _lib = handle
    return _lib


def declared_symbols(header: str = HEADER):
    """Function names declared in include/mxscale.h."""
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mx_[a-z_0-9]+)\s*\(", text)))


def status_string(status: int) -> str:
    return lib().mx_status_string(status).decode()


def mx_rearranged_size(dim: int, rows: int, cols: int, num_groups: int) -> int:
    return int(lib().mx_rearranged_size(dim, rows, cols, num_groups))


def mx_rearrange_m_groups(scales: int, rows: int, cols: int, row_stride: int, group_end_offsets: int,
                          num_groups: int, out: int, stream: int) -> int:
    return lib().mx_rearrange_m_groups(scales, rows, cols, row_stride, group_end_offsets, num_groups, out, stream)


def mx_rearrange_k_groups(scales: int, rows: int, cols: int, row_stride: int, group_end_offsets: int,
                          num_groups: int, out: int, stream: int) -> int:
    return lib().mx_rearrange_k_groups(scales, rows, cols, row_stride, group_end_offsets, num_groups, out, stream)


def mx_rearrange_ex(dim: int, scales: int, rows: int, cols: int, row_stride: int, group_end_offsets: int,
                    num_groups: int, out: int, path: int, stream: int) -> int:
    return lib().mx_rearrange_ex(dim, scales, rows, cols, row_stride, group_end_offsets, num_groups, out,
                                 path, stream)


def mx_unrearrange_m_groups(blocked: int, rows: int, cols: int, group_end_offsets: int, num_groups: int,
                            scales: int, row_stride: int, stream: int) -> int:
    return lib().mx_unrearrange_m_groups(blocked, rows, cols, group_end_offsets, num_groups, scales, row_stride,
                                         stream)


def mx_unrearrange_k_groups(blocked: int, rows: int, cols: int, group_end_offsets: int, num_groups: int,
                            scales: int, row_stride: int, stream: int) -> int:
    return lib().mx_unrearrange_k_groups(blocked, rows, cols, group_end_offsets, num_groups, scales, row_stride,
                                         stream)


def mx_padded_group_starts(dim: int, rows: int, cols: int, group_end_offsets: int, num_groups: int, starts: int,
                           stream: int) -> int:
    return lib().mx_padded_group_starts(dim, rows, cols, group_end_offsets, num_groups, starts, stream)


def mx_select_path(dim: int, scales: int, rows: int, cols: int, row_stride: int) -> int:
    return int(lib().mx_select_path(dim, scales, rows, cols, row_stride))


def mx_device_flags(clear: bool = False) -> int:
    v = ctypes.c_uint32(0)
    st = lib().mx_device_flags(ctypes.byref(v), 1 if clear else 0)
    if st != MX_OK:
        raise MxError("mx_device_flags", st)
    return int(v.value)


def mx_selftest_bounded_wait(limit_cycles: int, stream: int = 0) -> int:
    return lib().mx_selftest_bounded_wait(limit_cycles, stream)


def mx_last_cuda_error() -> int:
    return int(lib().mx_last_cuda_error())


def mx_version() -> int:
    return int(lib().mx_version())
