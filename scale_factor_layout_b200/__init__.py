"""scale_factor_layout_b200 -- MXFP8 E8M0 scale factors -> per-group 128x4
blocked layout, on NVIDIA B200 (sm_100a).

The work runs in libmxscale.so (C ABI in include/mxscale.h); this package is
its binding.  ``_binding`` mirrors the C entry points one for one (raw
pointers and sizes); the functions below take torch tensors for convenience,
allocate the output with torch (the library itself never allocates), and pass
torch's current CUDA stream.
"""
from __future__ import annotations

from ._binding import (  # noqa: F401
    MX_GROUPS_K, MX_GROUPS_M, MX_MAX_GROUPS, MX_OK, MX_PATH_AUTO, MX_PATH_BYTE, MX_PATH_FLAT, MX_PATH_TMA,
    MX_PATH_WORD, PATHS, MxError, declared_symbols, lib, mx_device_flags, mx_rearrange_ex,
    mx_rearrange_k_groups, mx_rearrange_m_groups, mx_rearranged_size, mx_select_path,
    mx_padded_group_starts, mx_selftest_bounded_wait, mx_unrearrange_k_groups, mx_unrearrange_m_groups,
    mx_version, status_string,
)

__all__ = [
    "rearrange_m_groups", "rearrange_k_groups", "rearrange", "rearranged_size",
    "mx_rearrange_m_groups", "mx_rearrange_k_groups", "mx_rearrange_ex", "mx_rearranged_size",
    "mx_select_path", "mx_device_flags", "mx_version", "MxError", "unrearrange", "padded_group_starts",
    "mx_unrearrange_m_groups", "mx_unrearrange_k_groups", "mx_padded_group_starts",
]


def rearranged_size(dim: int, rows: int, cols: int, num_groups: int) -> int:
    return mx_rearranged_size(dim, rows, cols, num_groups)


def _check_inputs(scales, group_end_offsets):
    import torch

    if scales.dtype != torch.uint8 or scales.dim() != 2:
        raise ValueError("scales must be a 2-D uint8 tensor")
    if scales.shape[0] > 1 and scales.shape[1] > 1 and scales.stride(1) != 1:
        raise ValueError("scales must be dense along columns (stride(1) == 1)")
    if group_end_offsets.dtype != torch.int32 or group_end_offsets.dim() != 1:
        raise ValueError("group_end_offsets must be a 1-D int32 tensor")
    if not group_end_offsets.is_contiguous():
        raise ValueError("group_end_offsets must be contiguous")
    if not (scales.is_cuda and group_end_offsets.is_cuda):
        raise ValueError("scales and group_end_offsets must be CUDA tensors")


def rearrange(dim: int, scales, group_end_offsets, out=None, path: str = "auto", stream=None):
    """Rearrange ``scales`` (rows, cols) uint8 for groups along M (dim 0) or K
    (dim 1); returns the flat uint8 output of ``rearranged_size`` bytes."""
    import torch

    _check_inputs(scales, group_end_offsets)
    rows, cols = scales.shape
    G = group_end_offsets.numel()
    size = mx_rearranged_size(dim, rows, cols, G)
    if out is None:
        out = torch.empty(size, dtype=torch.uint8, device=scales.device)
    elif out.numel() < size or out.dtype != torch.uint8 or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous uint8 tensor of at least {size} bytes")
    stride = scales.stride(0) if rows > 1 else cols
    if stream is None:
        stream = torch.cuda.current_stream(scales.device).cuda_stream
    st = mx_rearrange_ex(dim, scales.data_ptr(), rows, cols, stride, group_end_offsets.data_ptr(), G,
                         out.data_ptr(), PATHS[path], stream)
    if st != MX_OK:
        raise MxError("mx_rearrange_ex", st)
    return out


def rearrange_m_groups(scales, group_end_offsets, out=None, path: str = "auto"):
    return rearrange(MX_GROUPS_M, scales, group_end_offsets, out, path)


def rearrange_k_groups(scales, group_end_offsets, out=None, path: str = "auto"):
    return rearrange(MX_GROUPS_K, scales, group_end_offsets, out, path)


def unrearrange(dim: int, blocked, rows: int, cols: int, group_end_offsets, out=None, stream=None):
    """Inverse of ``rearrange``: the blocked flat uint8 buffer back to a
    (rows, cols) uint8 tensor; elements no group covers come back as 0."""
    import torch

    if blocked.dtype != torch.uint8 or not blocked.is_contiguous() or not blocked.is_cuda:
        raise ValueError("blocked must be a contiguous CUDA uint8 tensor")
    if group_end_offsets.dtype != torch.int32 or not group_end_offsets.is_cuda or not group_end_offsets.is_contiguous():
        raise ValueError("group_end_offsets must be a contiguous CUDA int32 tensor")
    G = group_end_offsets.numel()
    if blocked.numel() < mx_rearranged_size(dim, rows, cols, G):
        raise ValueError("blocked is smaller than the layout's allocation")
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.uint8, device=blocked.device)
    elif (out.dtype != torch.uint8 or out.dim() != 2 or tuple(out.shape) != (rows, cols) or not out.is_cuda
          or (rows > 1 and cols > 1 and out.stride(1) != 1)):
        raise ValueError(f"out must be a CUDA uint8 tensor of shape ({rows}, {cols}), dense along columns")
    stride = out.stride(0) if rows > 1 else cols
    if stream is None:
        stream = torch.cuda.current_stream(blocked.device).cuda_stream
    fn = mx_unrearrange_m_groups if dim == MX_GROUPS_M else mx_unrearrange_k_groups
    st = fn(blocked.data_ptr(), rows, cols, group_end_offsets.data_ptr(), G, out.data_ptr(), stride, stream)
    if st != MX_OK:
        raise MxError("mx_unrearrange", st)
    return out


def padded_group_starts(dim: int, rows: int, cols: int, group_end_offsets, stream=None):
    """int32[G + 1] padded group starts (rows for M, columns for K), computed on the GPU."""
    import torch

    if group_end_offsets.dtype != torch.int32 or group_end_offsets.dim() != 1 or not group_end_offsets.is_cuda:
        raise ValueError("group_end_offsets must be a 1-D CUDA int32 tensor")
    if not group_end_offsets.is_contiguous():
        raise ValueError("group_end_offsets must be contiguous")
    G = group_end_offsets.numel()
    starts = torch.empty(G + 1, dtype=torch.int32, device=group_end_offsets.device)
    if stream is None:
        stream = torch.cuda.current_stream(group_end_offsets.device).cuda_stream
    st = mx_padded_group_starts(dim, rows, cols, group_end_offsets.data_ptr(), G, starts.data_ptr(), stream)
    if st != MX_OK:
        raise MxError("mx_padded_group_starts", st)
    return starts
