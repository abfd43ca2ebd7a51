"""The C-ABI library loads and exports every symbol include/ep.h declares;
host-side argument validation works without a GPU (no compute calls here)."""
import ctypes
import os
import re

import pytest
import torch

from combine_ep_layout_10_b200 import build as B
from combine_ep_layout_10_b200 import ep

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    B.build()
    return ep.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "ep.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ep_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    assert sorted(ep.ABI_SYMBOLS) == names


def test_status_strings(L):
    assert ep.status_str(0) == "EP_OK"
    assert ep.status_str(3) == "EP_ERR_CAPACITY"
    assert ep.status_str(99) == "EP_ERR_UNKNOWN"


def test_max_recv_rows(L):
    assert ep.ep_max_recv_rows(8192, 8, 256) == 65536
    assert ep.ep_max_recv_rows(8192, 8, 256, 4) == 65536 + 256 * 3
    assert ep.ep_max_recv_rows(128, 8, 256, 1, 128) == 32768
    assert ep.ep_max_recv_rows(-1, 8, 256) == 0
    assert ep.ep_max_recv_rows(16, 33, 256) == 0


def _layout_status(L, T, k, E, R, A=1, C=0, idx=None):
    h = ctypes.c_void_p()
    return L.ep_layout(idx, T, k, E, R, A, C, None, None, None, ctypes.byref(h), None)


def test_layout_argument_errors_on_host(L):
    fake = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    assert _layout_status(L, 4, 2, 4, 3, idx=fake) == ep.EP_ERR_INVALID_ARG       # E % R
    assert _layout_status(L, 4, 33, 64, 2, idx=fake) == ep.EP_ERR_INVALID_ARG     # k > 32
    assert _layout_status(L, 4, 2, 8192, 2, idx=fake) == ep.EP_ERR_INVALID_ARG    # E > 4096
    assert _layout_status(L, 4, 2, 4, 2, A=0, idx=fake) == ep.EP_ERR_INVALID_ARG  # align
    assert _layout_status(L, 4, 2, 4, 2, A=2, C=3, idx=fake) == ep.EP_ERR_INVALID_ARG
    assert _layout_status(L, 4, 2, 4, 2, idx=None) == ep.EP_ERR_INVALID_ARG       # null ids
    assert _layout_status(L, 4, 2, 4, 2, idx=ctypes.c_void_p(258)) == ep.EP_ERR_INVALID_ARG  # misaligned
    assert L.ep_layout(fake, 4, 2, 4, 2, 1, 0, None, None, None, None, None) == ep.EP_ERR_INVALID_ARG


def test_dispatch_combine_argument_errors_on_host(L):
    assert L.ep_dispatch(None, None, 128, 0, None, None, None, 0, None) == ep.EP_ERR_INVALID_ARG
    assert L.ep_combine(None, None, None, 128, 0, None, None) == ep.EP_ERR_INVALID_ARG
    # hidden sizes outside [8, 2^24] or not a multiple of 8 (the handle is never dereferenced)
    fake = ctypes.c_void_p(256)
    for H in (0, 12, (1 << 24) + 8):
        assert L.ep_dispatch(fake, None, H, 0, None, None, None, 0, None) == ep.EP_ERR_INVALID_ARG
        assert L.ep_combine(fake, None, None, H, 0, None, None) == ep.EP_ERR_INVALID_ARG
        assert L.ep_dispatch_backward(fake, None, H, 0, None, None) == ep.EP_ERR_INVALID_ARG
        assert L.ep_combine_backward(fake, None, None, None, H, 0, None, None, None) == ep.EP_ERR_INVALID_ARG
    # column-major FP8 dispatch: no handle, H not a multiple of 128, leading dimension below the rows
    assert L.ep_dispatch_fp8_colmajor(None, None, 128, None, None, 64, None, None, 64, 0, None) == \
        ep.EP_ERR_INVALID_ARG
    for H, ld, rows, sms in ((136, 64, 64, 0), (0, 64, 64, 0), (128, 63, 64, 0), (128, 64, 64, -1)):
        assert L.ep_dispatch_fp8_colmajor(fake, None, H, None, None, ld, None, None, rows, sms, None) == \
            ep.EP_ERR_INVALID_ARG, (H, ld, rows, sms)
    L.ep_handle_free(None)  # no-op
    info = ep._HandleInfo()
    assert L.ep_handle_get_info(None, ctypes.byref(info)) == ep.EP_ERR_INVALID_ARG
    assert L.ep_handle_check(None, None) == ep.EP_ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU answer")
def test_no_device_is_reported(L):
    assert _layout_status(L, 0, 2, 4, 2) == ep.EP_ERR_NO_DEVICE


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(ep, "_LIB", None)
    monkeypatch.setattr(ep, "LIB_PATH", "/nonexistent/libep_b200.so")
    with pytest.raises(RuntimeError, match="missing"):
        ep.lib()


def test_peer_max_recv_rows(L):
    # every slot of every rank may land on one rank, plus alignment slack per owned expert
    assert ep.ep_peer_max_recv_rows(8 * 8192, 8, 256, 8) == 8 * 8192 * 8
    assert ep.ep_peer_max_recv_rows(1000, 8, 256, 8, 4) == 8000 + 32 * 3
    assert ep.ep_peer_max_recv_rows(1000, 8, 256, 8, 1, 128) == 32 * 128
    assert ep.ep_peer_max_recv_rows(1000, 8, 255, 8) == 0      # E % world
    assert ep.ep_peer_max_recv_rows(-1, 8, 256, 8) == 0
    assert ep.ep_peer_max_recv_rows(1000, 33, 256, 8) == 0     # k above the limit
    assert ep.ep_peer_max_recv_rows(1000, 8, 8192, 8) == 0     # E above the limit


def test_multi_gpu_argument_errors_on_host(L):
    P = ctypes.c_void_p
    out = P()
    fake = P(256)   # never dereferenced: validation fails first
    INV = ep.EP_ERR_INVALID_ARG
    # plan: no handle / no output slot
    assert L.ep_plan_create(None, fake, fake, 0, 2, 1, 0, 64, ctypes.byref(out), None) == INV
    assert L.ep_plan_create(fake, fake, fake, 0, 2, 1, 0, 64, None, None) == INV
    # peers: empty group, missing or misaligned receive buffers
    assert L.ep_peers_create(0, None, None, None, None, 64, ctypes.byref(out)) == INV
    assert L.ep_peers_create(2, None, None, None, None, 64, ctypes.byref(out)) == INV
    two = (P * 2)(256, 256 + 8)                                # second one not 16-byte aligned
    assert L.ep_peers_create(2, two, None, None, None, 64, ctypes.byref(out)) == INV
    nul = (P * 2)(256, None)
    assert L.ep_peers_create(2, nul, None, None, None, 64, ctypes.byref(out)) == INV
    # peer calls with no plan or table
    assert L.ep_dispatch_peer(None, None, fake, None, 128, 0, 1, 1, 1, 0, None) == INV
    assert L.ep_combine_peer(None, None, None, 128, fake, 0, None) == INV
    assert L.ep_combine_backward_peer(None, None, fake, fake, 128, None, None) == INV
    # IPC: null arguments
    h = ctypes.create_string_buffer(ep.EP_IPC_HANDLE_BYTES)
    off = ctypes.c_uint64()
    assert L.ep_ipc_export(None, h, ctypes.byref(off)) == INV
    assert L.ep_ipc_import(None, 0, ctypes.byref(out)) == INV
    assert L.ep_ipc_release(None, 0) == INV
    assert L.ep_plan_check(None, None) == INV
    assert L.ep_dispatch_topk(None, None, None, None, None, 0, None) == INV


def test_handle_info_struct_matches_the_header(tmp_path):
    """The ctypes mirror of ep_handle_info has the C struct's size and field
    offsets (compiled from include/ep.h with the host C compiler)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    fields = [f for f, _ in ep._HandleInfo._fields_]
    src = tmp_path / "info.c"
    src.write_text("#include <stdio.h>\n#include <stddef.h>\n#include \"ep.h\"\nint main(void) {\n"
                   "  printf(\"%zu\\n\", sizeof(ep_handle_info));\n"
                   + "".join("  printf(\"%%zu\\n\", offsetof(ep_handle_info, %s));\n" % f for f in fields)
                   + "  return 0;\n}\n")
    exe = tmp_path / "info"
    inc = os.path.join(ROOT, "include")
    subprocess.run([cc, "-I", inc, str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()]
    want = [ctypes.sizeof(ep._HandleInfo)] + [getattr(ep._HandleInfo, f).offset for f in fields]
    assert got == want
