"""Host check of the decode kernel's shared-memory layouts (no GPU needed).

The decode kernel addresses its code tables by byte permutes and keeps the
staged key / value rows of the 3-bit-key / 4-bit-value shape inside the value
table's unused halves (a second, mapped address space).  tests/native/
decode_layout_check.cu evaluates the kernel's own constexpr layout functions
on the host and checks, for every shape that uses these layouts: each staged
byte and merge float maps one-to-one into its region without touching a table
entry, the kernel's read formulas equal the mapped addresses, a warp's reads
fall on 32 distinct banks, and the shared memory fits the CTAs per SM the
register budget assumes.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "native", "decode_layout_check.cu")


def _nvcc():
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    return exe if os.path.exists(exe) else None


@pytest.mark.skipif(_nvcc() is None, reason="nvcc not available")
def test_decode_layouts(tmp_path):
    exe = tmp_path / "decode_layout_check"
    cmd = [_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "--expt-relaxed-constexpr",
           "-I", os.path.join(ROOT, "turboquant_kv_cache_rht_b200", "csrc"), "-I", os.path.join(ROOT, "include"),
           SRC, "-o", str(exe)]
    build = subprocess.run(cmd, capture_output=True, text=True)
    assert build.returncode == 0, build.stderr[-4000:]
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout[-4000:]
    assert "total bad 0" in run.stdout
