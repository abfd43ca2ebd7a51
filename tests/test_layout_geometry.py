"""The layout's launch geometry over the ABI's whole range (CPU only).

tests/layout_geometry_check.cu is built with nvcc together with the
library's layout.cu and run on the host (it makes no CUDA call): for ~23,000
shapes spanning T*k < 2^31, k <= 32, E <= 4096, every R dividing E, packed
and padded, the geometry the library would launch must have whole-warp
blocks within 1,024 threads, shared memory within the 227 KB a block may
opt into, count matrices within their bound (the no-allocation scratch) and
tiles that cover the batch exactly; and the dispatch's work units must tile
every row for hidden sizes up to the ABI's 2^24.  Shapes this large cannot
all be run on a GPU; their launch shapes can all be checked here.
"""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_layout_geometry_is_valid_for_every_shape(tmp_path):
    from combine_ep_layout_10_b200 import build as B
    try:
        nvcc = B.nvcc()
    except RuntimeError:
        pytest.skip("nvcc not available")
    exe = tmp_path / "check"
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17",
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(ROOT, "combine_ep_layout_10_b200", "csrc"),
           os.path.join(ROOT, "tests", "layout_geometry_check.cu"),
           os.path.join(ROOT, "combine_ep_layout_10_b200", "csrc", "layout.cu"), "-o", str(exe)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stdout[-4000:]
    assert "0 violations" in out.stdout
