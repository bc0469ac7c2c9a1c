"""Helpers for GPU tests: place a synthetic case on the device exactly as laid
out on the host (row stride, gap bytes, a chosen misalignment), call the C ABI
through the binding, and read back the output between canary bytes."""
from __future__ import annotations

import numpy as np
import torch

import scale_factor_layout_b200 as mxs
from scale_factor_layout_b200 import _binding as B

CANARY = 0xA5
GUARD = 256


def base_bytes(scales: np.ndarray) -> np.ndarray:
    """The (rows, row_stride) bytes a strided (rows, cols) view sits in, flattened."""
    rows, cols = scales.shape
    if rows == 0 or cols == 0:
        return np.zeros(0, np.uint8)
    stride = scales.strides[0]
    full = np.lib.stride_tricks.as_strided(scales, shape=(rows, stride), strides=(stride, 1))
    # the last row may end at cols; only copy what the view spans
    flat = np.empty((rows - 1) * stride + cols, np.uint8)
    flat[: (rows - 1) * stride] = full[:-1].reshape(-1)
    flat[(rows - 1) * stride:] = scales[-1]
    return flat


class DeviceCase:
    def __init__(self, case, misalign: int = 0, device: str = "cuda"):
        self.case = case
        raw = base_bytes(case.scales)
        self.buf = torch.empty(len(raw) + misalign + 64, dtype=torch.uint8, device=device)
        self.buf.fill_(0xFF)
        if len(raw):
            self.buf[misalign: misalign + len(raw)].copy_(torch.from_numpy(raw))
        self.ptr = self.buf.data_ptr() + misalign
        self.ends = torch.from_numpy(np.ascontiguousarray(case.ends, dtype=np.int32)).to(device)
        self.size = mxs.mx_rearranged_size(case.dim, case.rows, case.cols, case.num_groups)
        self.outbuf = torch.full((self.size + 2 * GUARD,), CANARY, dtype=torch.uint8, device=device)
        self.out_ptr = self.outbuf.data_ptr() + GUARD

    def run(self, path: str = "auto", stream=None, ends=None) -> int:
        c = self.case
        s = torch.cuda.current_stream().cuda_stream if stream is None else stream
        e = self.ends if ends is None else ends
        return B.mx_rearrange_ex(c.dim, self.ptr, c.rows, c.cols, max(c.row_stride, c.cols) if c.rows > 1 else c.cols,
                                 e.data_ptr(), e.numel(), self.out_ptr, B.PATHS[path], s)

    def output(self) -> np.ndarray:
        host = self.outbuf.cpu().numpy()
        assert (host[:GUARD] == CANARY).all(), "bytes before the output were written"
        assert (host[GUARD + self.size:] == CANARY).all(), "bytes after the output were written"
        return host[GUARD: GUARD + self.size]
