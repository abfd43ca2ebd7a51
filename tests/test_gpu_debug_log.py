"""EP_DEBUG host logging (GPU): one stderr line per layout / dispatch /
column-major dispatch / combine / no-allocation layout call with the launch
shape the library chose; silent by default."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import sys
sys.path.insert(0, %r)
import torch
from combine_ep_layout_10_b200 import ep, workloads as W
for name, T in (("tiny", 128), ("prefill", 512)):
    w = W.WORKLOADS[name].scaled(T=T)
    x, idx, tw = W.make_routing(w)
    res = ep.ep_layout(idx.cuda(), w.E, w.R)
    recv, sc, _ = ep.ep_dispatch(res.handle, x.cuda(), w.fp8)
    out = ep.ep_combine(res.handle, torch.zeros(res.handle.num_recv_rows, w.H, dtype=torch.bfloat16, device="cuda"), tw.cuda())
    if name == "prefill":
        ep.ep_dispatch_fp8_colmajor(res.handle, x.cuda())
    torch.cuda.synchronize()
    res.handle.free()
w = W.WORKLOADS["prefill"].scaled(T=512)
_, idx, _ = W.make_routing(w)
rows = ep.ep_max_recv_rows(w.T, w.k, w.E)
i32 = lambda *s: torch.empty(*s, dtype=torch.int32, device="cuda")
ep.ep_layout_noalloc(idx.cuda(), w.E, w.R, i32(w.T, w.k), i32(rows), i32(w.E + 1), i32(w.R + 1))
torch.cuda.synchronize()
print("done")
""" % ROOT


def run(debug):
    env = dict(os.environ)
    env.pop("EP_DEBUG", None)
    if debug is not None:
        env["EP_DEBUG"] = debug
    return subprocess.run([sys.executable, "-c", SCRIPT], env=env, capture_output=True, text=True, timeout=300)


def test_debug_log_lines():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    res = run("1")
    assert res.returncode == 0, res.stderr
    lines = [ln for ln in res.stderr.splitlines() if ln.startswith("ep: ")]
    assert sum(ln.startswith("ep: layout ") for ln in lines) == 2
    noalloc = [ln for ln in lines if ln.startswith("ep: layout_noalloc ")]
    assert len(noalloc) == 1
    assert "path=tiled" in noalloc[0] and "scratch_words=" in noalloc[0] and "of 32768" in noalloc[0]
    assert sum(ln.startswith("ep: dispatch ") for ln in lines) == 2
    colmajor = [ln for ln in lines if ln.startswith("ep: dispatch_fp8_colmajor ")]
    assert len(colmajor) == 1 and "T=512" in colmajor[0] and "ld=4096" in colmajor[0]
    assert sum(ln.startswith("ep: combine") for ln in lines) == 2
    layouts = [ln for ln in lines if ln.startswith("ep: layout ")]
    assert "path=one-cta" in layouts[0]                     # tiny: 128 tokens x 4 slots = 512 slots
    assert "path=tiled" in layouts[1] and "threads=512" in layouts[1]   # prefill: 512 x 8 = 4K slots
    assert any("mode=bf16->e4m3" in ln for ln in lines)     # prefill dispatches FP8
    assert res.stdout.strip() == "done"                     # stdout untouched


def test_silent_by_default():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    for value in (None, "0"):
        res = run(value)
        assert res.returncode == 0, res.stderr
        assert not any(ln.startswith("ep: ") for ln in res.stderr.splitlines())
