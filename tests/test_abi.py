"""C ABI checks that need no GPU: the library loads, exports every symbol the
header declares, sizes outputs like the oracle, picks paths by the stated
alignment rules, and rejects bad arguments before touching the device."""
import ctypes

import numpy as np
import pytest

from scale_factor_layout_b200 import _binding as B

M, K = B.MX_GROUPS_M, B.MX_GROUPS_K


def test_exports_every_declared_symbol(mxlib):
    declared = B.declared_symbols()
    assert {"mx_rearrange_m_groups", "mx_rearrange_k_groups", "mx_rearranged_size"} <= set(declared)
    for name in declared:
        assert hasattr(mxlib, name), f"{name} declared in include/mxscale.h but not exported"
    assert B.mx_version() >= 100


def test_sizes_match_oracle(mxlib, orc):
    rng = np.random.default_rng(0)
    for _ in range(500):
        dim = int(rng.integers(0, 2))
        rows, cols, G = int(rng.integers(0, 300000)), int(rng.integers(0, 20000)), int(rng.integers(1, 65))
        assert B.mx_rearranged_size(dim, rows, cols, G) == orc.rearranged_size(dim, rows, cols, G)
    for bad in ((M, 10, 10, 0), (M, 10, 10, 65), (K, -1, 10, 1), (K, 10, -1, 1), (2, 10, 10, 1)):
        assert B.mx_rearranged_size(*bad) == 0


def test_path_selection(mxlib):
    assert B.mx_select_path(M, 0x1000, 100, 224, 224) == B.MX_PATH_TMA
    assert B.mx_select_path(M, 0x1000, 100, 44, 44) == B.MX_PATH_FLAT      # narrow rows, stride % 16 != 0
    assert B.mx_select_path(M, 0x1000, 100, 44, 300) == B.MX_PATH_WORD     # stride above the flat limit
    assert B.mx_select_path(M, 0x1000, 100, 43, 44) == B.MX_PATH_WORD      # cols not a multiple of 4
    assert B.mx_select_path(K, 0x1000, 100, 44, 44) == B.MX_PATH_WORD      # flat is M-groups only
    assert B.mx_select_path(M, 0x1004, 100, 48, 48) == B.MX_PATH_WORD      # base not 16-aligned
    assert B.mx_select_path(K, 0x1000, 100, 45, 45) == B.MX_PATH_BYTE      # odd stride
    assert B.mx_select_path(K, 0x1001, 100, 48, 48) == B.MX_PATH_BYTE      # odd base
    assert B.mx_select_path(K, 0x1000, 7168, 4096, 4096) == B.MX_PATH_TMA
    assert B.mx_select_path(K, 0x1000, 0, 4096, 4096) == B.MX_PATH_WORD    # nothing to load


def _call(dim=M, scales=0x1000, rows=256, cols=64, stride=64, ends=0x2000, G=2, out=0x3000, path=0):
    return B.mx_rearrange_ex(dim, scales, rows, cols, stride, ends, G, out, path, 0)


@pytest.mark.parametrize("kwargs,status", [
    (dict(G=0), B.MX_ERR_INVALID_ARG),
    (dict(G=65), B.MX_ERR_INVALID_ARG),
    (dict(rows=-1), B.MX_ERR_INVALID_ARG),
    (dict(cols=-5), B.MX_ERR_INVALID_ARG),
    (dict(rows=1 << 31), B.MX_ERR_INVALID_ARG),
    (dict(stride=63), B.MX_ERR_INVALID_ARG),
    (dict(ends=0), B.MX_ERR_INVALID_ARG),
    (dict(out=0), B.MX_ERR_INVALID_ARG),
    (dict(scales=0), B.MX_ERR_INVALID_ARG),
    (dict(dim=3), B.MX_ERR_INVALID_ARG),
    (dict(path=7), B.MX_ERR_INVALID_ARG),
    (dict(out=0x3008), B.MX_ERR_MISALIGNED),
    (dict(stride=72, path=B.MX_PATH_TMA), B.MX_ERR_MISALIGNED),
    (dict(scales=0x1008, path=B.MX_PATH_TMA), B.MX_ERR_MISALIGNED),
    (dict(stride=66, path=B.MX_PATH_WORD), B.MX_ERR_MISALIGNED),
    (dict(scales=0x1002, path=B.MX_PATH_WORD), B.MX_ERR_MISALIGNED),
    (dict(dim=K, rows=0), B.MX_OK),          # empty allocation: nothing to do, no launch
    (dict(dim=K, cols=44, stride=44, path=B.MX_PATH_FLAT), B.MX_ERR_UNSUPPORTED),
    (dict(cols=44, stride=300, path=B.MX_PATH_FLAT), B.MX_ERR_UNSUPPORTED),
    (dict(cols=44, stride=44, scales=0x1004, path=B.MX_PATH_FLAT), B.MX_ERR_MISALIGNED),
    (dict(cols=43, stride=44, path=B.MX_PATH_FLAT), B.MX_ERR_MISALIGNED),
    (dict(path=5), B.MX_ERR_INVALID_ARG),
])
def test_host_validation(mxlib, kwargs, status):
    assert _call(**kwargs) == status


def test_status_strings(mxlib):
    for st in range(5):
        assert B.status_string(st)
    assert "misaligned" in B.status_string(B.MX_ERR_MISALIGNED)


@pytest.mark.parametrize("kwargs,status", [
    (dict(G=0), B.MX_ERR_INVALID_ARG),
    (dict(G=65), B.MX_ERR_INVALID_ARG),
    (dict(rows=-1), B.MX_ERR_INVALID_ARG),
    (dict(stride=10), B.MX_ERR_INVALID_ARG),
    (dict(ends=0), B.MX_ERR_INVALID_ARG),
    (dict(blocked=0), B.MX_ERR_INVALID_ARG),
    (dict(scales=0), B.MX_ERR_INVALID_ARG),
    (dict(blocked=0x4004), B.MX_ERR_MISALIGNED),
    (dict(rows=0), B.MX_OK),          # nothing to write, no launch
])
def test_inverse_host_validation(mxlib, kwargs, status):
    a = dict(blocked=0x4000, rows=256, cols=64, ends=0x2000, G=2, scales=0x5000, stride=64)
    a.update(kwargs)
    for fn in (B.mx_unrearrange_m_groups, B.mx_unrearrange_k_groups):
        assert fn(a["blocked"], a["rows"], a["cols"], a["ends"], a["G"], a["scales"], a["stride"], 0) == status


def test_padded_starts_host_validation(mxlib):
    assert B.mx_padded_group_starts(B.MX_GROUPS_M, 10, 10, 0, 2, 0x1000, 0) == B.MX_ERR_INVALID_ARG
    assert B.mx_padded_group_starts(B.MX_GROUPS_M, 10, 10, 0x1000, 0, 0x2000, 0) == B.MX_ERR_INVALID_ARG
    assert B.mx_padded_group_starts(7, 10, 10, 0x1000, 2, 0x2000, 0) == B.MX_ERR_INVALID_ARG


def test_torch_wrappers_reject_bad_tensors():
    """The torch-level wrappers check their tensors before any library call."""
    import torch

    import scale_factor_layout_b200 as mxs

    ends = torch.tensor([10, 20], dtype=torch.int32)
    with pytest.raises(ValueError):   # not on a CUDA device
        mxs.rearrange(mxs.MX_GROUPS_M, torch.zeros((20, 8), dtype=torch.uint8), ends)
    with pytest.raises(ValueError):   # wrong dtype
        mxs.rearrange(mxs.MX_GROUPS_M, torch.zeros((20, 8), dtype=torch.int32), ends)
    with pytest.raises(ValueError):   # blocked buffer not on a CUDA device
        mxs.unrearrange(mxs.MX_GROUPS_M, torch.zeros(4096, dtype=torch.uint8), 20, 8, ends)
    with pytest.raises(ValueError):   # offsets of the wrong dtype
        mxs.padded_group_starts(mxs.MX_GROUPS_M, 20, 8, torch.tensor([10, 20], dtype=torch.int64))


def test_header_is_plain_c_and_links(mxlib, tmp_path):
    """include/mxscale.h compiles as C (not C++), every declared entry point
    links against libmxscale.so, and the host-only calls run from C."""
    import os
    import shutil
    import subprocess

    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    names = B.declared_symbols()
    refs = "\n".join(f"    (entry_fn)&{n}," for n in names)
    src = tmp_path / "use_mxscale.c"
    src.write_text(f'''#include <stdio.h>
#include "mxscale.h"
typedef void (*entry_fn)(void);
static const entry_fn entry_points[] = {{
{refs}
}};
int main(void) {{
    size_t n = sizeof entry_points / sizeof entry_points[0];
    for (size_t i = 0; i < n; ++i)
        if (entry_points[i] == 0) return 2;
    printf("%zu %d %zu %zu %s\\n", n, mx_version(),
           mx_rearranged_size(MX_GROUPS_M, 1000, 44, 4), mx_rearranged_size(MX_GROUPS_K, 7168, 4096, 8),
           mx_status_string(MX_ERR_MISALIGNED));
    return 0;
}}
''')
    exe = tmp_path / "use_mxscale"
    lib_dir = os.path.dirname(B.LIB_PATH)
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-pedantic", "-I", os.path.dirname(B.HEADER),
                    "-I", cuda_inc, str(src), "-o", str(exe), "-L", lib_dir, "-lmxscale",
                    f"-Wl,-rpath,{lib_dir}"], check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split(maxsplit=4)
    assert int(out[0]) == len(names)
    assert int(out[1]) == B.mx_version()
    assert int(out[2]) == B.mx_rearranged_size(M, 1000, 44, 4)
    assert int(out[3]) == B.mx_rearranged_size(K, 7168, 4096, 8)
    assert out[4].strip() == B.status_string(B.MX_ERR_MISALIGNED)
