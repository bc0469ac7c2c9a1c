"""Plant plausible mistakes in copies of the CPU oracle and check that the pins
catch every one.  Each mutant is compiled from a textual copy of
``oracle/mx_oracle.c`` in a temporary directory (the real oracle is never
touched) and run against the pin suite in a subprocess, so a mutant that
crashes counts as caught without taking the test run down."""
import os
import shutil
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
sys.path.insert(0, ROOT)
import oracle  # noqa: E402

# (name, original text, planted text, expected replacement count or None for >= 1)
MUTANTS = [
    ("tile_rows_swapped", "(r % 32) * 16 + (r / 32) * 4 + c", "(r / 32) * 16 + (r % 32) * 4 + c", 1),
    ("tile_col_dropped", "(r % 32) * 16 + (r / 32) * 4 + c", "(r % 32) * 16 + (r / 32) * 4", 1),
    ("tile_stride_8", "(r % 32) * 16 + (r / 32) * 4 + c", "(r % 32) * 16 + (r / 32) * 8 + c", 1),
    ("m_tiles_col_major", "(l / 128) * 128 * PC + (j / 4) * 512", "(l / 128) * 512 + (j / 4) * 128 * PC", 1),
    ("m_group_start_dropped", "return P_g * PC + ", "return ", 1),
    ("k_group_start_dropped", "return R * Q_g + ", "return ", 1),
    ("k_row_block_stride_R", "(i / 128) * 128 * W_g", "(i / 128) * 128 * R", 1),
    ("m_rows_not_padded", "int64_t edge = (dim == DIM_M) ? 128 : 4;", "int64_t edge = (dim == DIM_M) ? 1 : 4;", 1),
    ("k_cols_not_padded", "int64_t edge = (dim == DIM_M) ? 128 : 4;", "int64_t edge = (dim == DIM_M) ? 128 : 1;", 1),
    ("k_width_unpadded", "W_g = round_up(e[g] - begin, 4);", "W_g = e[g] - begin;", None),
    ("clamp_not_monotone", "if (e < prev) e = prev;", "", 1),
    ("clamp_not_bounded", "if (e > limit) e = limit;", "", 1),
    ("m_alloc_127", "(rows + 128 * (int64_t)num_groups)", "(rows + 127 * (int64_t)num_groups)", 1),
    ("k_alloc_3g", "(cols + 4 * (int64_t)num_groups)", "(cols + 3 * (int64_t)num_groups)", 1),
    ("k_rows_not_padded", "return round_up(rows, 128) * (cols", "return rows * (cols", 1),
    ("decode_row_order", "int64_t r = rb * 128 + a * 32 + line;", "int64_t r = rb * 128 + line * 4 + a;", 1),
    ("padding_not_zeroed", "memset(out, 0, (size_t)out_size);", "", 1),
]


@pytest.mark.parametrize("name,orig,planted,count", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(tmp_path, name, orig, planted, count):
    src = open(oracle.SRC).read()
    n = src.count(orig)
    assert n >= 1 and (count is None or n == count), f"mutation site for {name} not found ({n})"
    shutil.copy(os.path.join(os.path.dirname(oracle.SRC), "mx_oracle.h"), tmp_path / "mx_oracle.h")
    mutant_src = tmp_path / "mx_oracle.c"
    mutant_src.write_text(src.replace(orig, planted))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-I", str(tmp_path), str(mutant_src),
                    "-o", str(lib)], check=True)
    proc = subprocess.run([sys.executable, os.path.join(HERE, "oracle_pins.py"), str(lib)],
                          capture_output=True, text=True, timeout=300)
    assert proc.returncode != 0, f"planted mistake {name} survived every pin:\n{proc.stdout}{proc.stderr}"


def test_unmutated_copy_passes(tmp_path):
    """The harness itself: an unmodified copy passes every pin."""
    shutil.copy(oracle.SRC, tmp_path / "mx_oracle.c")
    shutil.copy(os.path.join(os.path.dirname(oracle.SRC), "mx_oracle.h"), tmp_path / "mx_oracle.h")
    lib = tmp_path / "libcopy.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-I", str(tmp_path),
                    str(tmp_path / "mx_oracle.c"), "-o", str(lib)], check=True)
    proc = subprocess.run([sys.executable, os.path.join(HERE, "oracle_pins.py"), str(lib)],
                          capture_output=True, text=True, timeout=300)
    assert proc.returncode == 0, proc.stdout + proc.stderr
