"""Python binding of the C ABI in include/ep.h (libep_b200.so).

Argument marshalling only: every step of layout, dispatch, combine, their
backward pair and the multi-GPU plan runs in the library's CUDA kernels.
PyTorch supplies device memory and the current stream.  There is no
fallback: if the CUDA library is missing or the device is not an sm_100 part,
the calls raise.

The names follow the C ABI: ep_max_recv_rows, ep_layout, ep_dispatch,
ep_combine, ep_handle_free (plus the handle accessors), the option, backward
and per-row calls (ep_dispatch_ex, ep_dispatch_fp8_colmajor, ep_combine_ex,
ep_dispatch_backward, ep_combine_backward, ep_dispatch_topk, ep_layout_noalloc) and the multi-GPU
calls (ep_plan_create, Peers, ep_dispatch_peer, ep_combine_peer,
ep_combine_backward_peer, ipc_export / ipc_import / ipc_release).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
#: The library this binding loads: the in-tree build, or the file named by
#: the EP_B200_LIB environment variable (another build of the same sources).
LIB_PATH = os.environ.get("EP_B200_LIB") or os.path.join(_HERE, "lib", "libep_b200.so")

EP_OK = 0
EP_ERR_INVALID_ARG = 1
EP_ERR_BAD_EXPERT_ID = 2
EP_ERR_CAPACITY = 3
EP_ERR_CUDA = 4
EP_ERR_OOM = 5
EP_ERR_TIMEOUT = 6
EP_ERR_NO_DEVICE = 7
EP_ERR_SCRATCH_LIMIT = 8

#: Every symbol the ABI exports (include/ep.h).
ABI_SYMBOLS = (
    "ep_status_str", "ep_max_recv_rows", "ep_layout", "ep_dispatch", "ep_combine",
    "ep_handle_free", "ep_handle_get_info", "ep_handle_export", "ep_handle_counts_host",
    "ep_handle_check", "ep_layout_noalloc", "ep_dispatch_backward", "ep_combine_backward",
    "ep_dispatch_ex", "ep_combine_ex", "ep_dispatch_topk", "ep_dispatch_fp8_colmajor",
    "ep_peer_max_recv_rows", "ep_plan_create", "ep_plan_free", "ep_plan_export", "ep_plan_recv_rows_host",
    "ep_plan_check", "ep_peers_create", "ep_peers_free", "ep_dispatch_peer", "ep_combine_peer",
    "ep_combine_backward_peer", "ep_peers_set_topk", "ep_dispatch_topk_peer", "ep_e4m3_encode",
    "ep_ipc_export", "ep_ipc_import", "ep_ipc_release",
)

EP_IPC_HANDLE_BYTES = 64

#: How a layout ran (ep_handle_info.layout_path).
EP_LAYOUT_PATH_EMPTY = 0
EP_LAYOUT_PATH_ONE_CTA = 1
EP_LAYOUT_PATH_TILED = 2

EP_FORMAT_BF16 = 0
EP_FORMAT_E4M3 = 1


class EpError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__("%s: %s" % (what, status_str(status)))
        self.status = status


class _HandleInfo(ctypes.Structure):
    _fields_ = [("num_tokens", ctypes.c_int), ("num_topk", ctypes.c_int),
                ("num_experts", ctypes.c_int), ("num_ranks", ctypes.c_int),
                ("expert_alignment", ctypes.c_int), ("capacity", ctypes.c_int),
                ("num_recv_rows", ctypes.c_size_t), ("layout_kernels", ctypes.c_int),
                ("layout_path", ctypes.c_int)]


_LIB = None


def lib() -> ctypes.CDLL:
    """Load libep_b200.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libep_b200.so is missing (%s); build it with "
                               "`python -m combine_ep_layout_10_b200.build`" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.ep_status_str.argtypes = [I]
        L.ep_status_str.restype = ctypes.c_char_p
        L.ep_max_recv_rows.argtypes = [I, I, I, I, I]
        L.ep_max_recv_rows.restype = S
        L.ep_layout.argtypes = [P, I, I, I, I, I, I, P, P, P, ctypes.POINTER(P), P]
        L.ep_layout.restype = I
        L.ep_dispatch.argtypes = [P, P, I, I, P, P, P, S, P]
        L.ep_dispatch.restype = I
        L.ep_combine.argtypes = [P, P, P, I, S, P, P]
        L.ep_combine.restype = I
        L.ep_handle_free.argtypes = [P]
        L.ep_handle_free.restype = None
        L.ep_handle_get_info.argtypes = [P, ctypes.POINTER(_HandleInfo)]
        L.ep_handle_get_info.restype = I
        L.ep_handle_export.argtypes = [P, P, P, P, P, P]
        L.ep_handle_export.restype = I
        L.ep_handle_counts_host.argtypes = [P, P, P]
        L.ep_handle_counts_host.restype = I
        L.ep_handle_check.argtypes = [P, P]
        L.ep_handle_check.restype = I
        L.ep_layout_noalloc.argtypes = [P, I, I, I, I, I, I, P, P, P, P, P, P, P, P, P]
        L.ep_layout_noalloc.restype = I
        L.ep_dispatch_backward.argtypes = [P, P, I, S, P, P]
        L.ep_dispatch_backward.restype = I
        L.ep_combine_backward.argtypes = [P, P, P, P, I, S, P, P, P]
        L.ep_combine_backward.restype = I
        I64 = ctypes.c_int64
        L.ep_dispatch_ex.argtypes = [P, P, P, I, I, I, P, P, I64, I64, P, S, I, P]
        L.ep_dispatch_ex.restype = I
        L.ep_dispatch_fp8_colmajor.argtypes = [P, P, I, P, P, I64, P, P, S, I, P]
        L.ep_dispatch_fp8_colmajor.restype = I
        L.ep_combine_ex.argtypes = [P, P, P, I, S, P, I, P]
        L.ep_dispatch_topk.argtypes = [P, P, P, P, P, S, P]
        L.ep_dispatch_topk.restype = I
        L.ep_combine_ex.restype = I
        I64, U64 = ctypes.c_int64, ctypes.c_uint64
        L.ep_peer_max_recv_rows.argtypes = [I64, I, I, I, I, I]
        L.ep_peer_max_recv_rows.restype = S
        L.ep_plan_create.argtypes = [P, P, P, I, I, I, I, S, ctypes.POINTER(P), P]
        L.ep_plan_create.restype = I
        L.ep_plan_free.argtypes = [P]
        L.ep_plan_free.restype = None
        L.ep_plan_export.argtypes = [P, P, P, P, P]
        L.ep_plan_export.restype = I
        L.ep_plan_recv_rows_host.argtypes = [P, ctypes.POINTER(I64), P]
        L.ep_plan_recv_rows_host.restype = I
        L.ep_plan_check.argtypes = [P, P]
        L.ep_plan_check.restype = I
        L.ep_peers_create.argtypes = [I, P, P, P, P, S, ctypes.POINTER(P)]
        L.ep_peers_create.restype = I
        L.ep_peers_free.argtypes = [P]
        L.ep_peers_free.restype = None
        L.ep_dispatch_peer.argtypes = [P, P, P, P, I, I, I, I64, I64, I, P]
        L.ep_dispatch_peer.restype = I
        L.ep_combine_peer.argtypes = [P, P, P, I, P, I, P]
        L.ep_combine_peer.restype = I
        L.ep_combine_backward_peer.argtypes = [P, P, P, P, I, P, P]
        L.ep_combine_backward_peer.restype = I
        L.ep_peers_set_topk.argtypes = [P, P, P, P, P]
        L.ep_peers_set_topk.restype = I
        L.ep_dispatch_topk_peer.argtypes = [P, P, P, P, P]
        L.ep_dispatch_topk_peer.restype = I
        L.ep_e4m3_encode.argtypes = [P, P, S, P]
        L.ep_e4m3_encode.restype = I
        L.ep_ipc_export.argtypes = [P, P, ctypes.POINTER(U64)]
        L.ep_ipc_export.restype = I
        L.ep_ipc_import.argtypes = [P, U64, ctypes.POINTER(P)]
        L.ep_ipc_import.restype = I
        L.ep_ipc_release.argtypes = [P, U64]
        L.ep_ipc_release.restype = I
        _LIB = L
    return _LIB


def status_str(status: int) -> str:
    return lib().ep_status_str(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != EP_OK:
        raise EpError(status, what)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dev_ptr(t: Optional[torch.Tensor], dtype, name: str, shape=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if t.device.index != torch.cuda.current_device():
        raise ValueError("%s is on %s, but the current device is cuda:%d" % (name, t.device,
                                                                          torch.cuda.current_device()))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    return ctypes.c_void_p(t.data_ptr())


def _check_rows(t: Optional[torch.Tensor], name: str, min_rows: int, cols: Optional[int] = None):
    """A [rows, cols] buffer that the call indexes by receive row must hold
    at least min_rows rows (the library cannot see a buffer's size)."""
    if t is None:
        return
    if t.dim() != (1 if cols is None else 2) or t.shape[0] < min_rows or (cols is not None and t.shape[1] != cols):
        want = "[>= %d]" % min_rows if cols is None else "[>= %d, %d]" % (min_rows, cols)
        raise ValueError("%s must be %s, got %s" % (name, want, tuple(t.shape)))


def ep_max_recv_rows(num_tokens: int, num_topk: int, num_experts: int,
                     expert_alignment: int = 1, capacity: int = 0) -> int:
    return int(lib().ep_max_recv_rows(num_tokens, num_topk, num_experts, expert_alignment, capacity))


class Handle:
    """Owner of an ep_handle* (the pages' EPHandle).  Reusable across calls
    while the routing is unchanged (the cached-handle decoding path)."""

    def __init__(self, ptr: ctypes.c_void_p, device: torch.device):
        self._ptr = ptr
        self.device = device
        info = _HandleInfo()
        _check(lib().ep_handle_get_info(ptr, ctypes.byref(info)), "ep_handle_get_info")
        self.num_tokens = info.num_tokens
        self.num_topk = info.num_topk
        self.num_experts = info.num_experts
        self.num_ranks = info.num_ranks
        self.expert_alignment = info.expert_alignment
        self.capacity = info.capacity
        self.num_recv_rows = int(info.num_recv_rows)
        self.layout_kernels = int(info.layout_kernels)
        self.layout_path = int(info.layout_path)

    @property
    def ptr(self) -> ctypes.c_void_p:
        if self._ptr is None:
            raise RuntimeError("handle already freed")
        return self._ptr

    def export(self, stream=None) -> dict:
        """Device copies of pos [T,k], src_idx [rows], seg [E+1], rank_off [R+1]."""
        dev = self.device
        pos = torch.empty(self.num_tokens, self.num_topk, dtype=torch.int32, device=dev)
        src = torch.empty(self.num_recv_rows, dtype=torch.int32, device=dev)
        seg = torch.empty(self.num_experts + 1, dtype=torch.int32, device=dev)
        roff = torch.empty(self.num_ranks + 1, dtype=torch.int32, device=dev)
        _check(lib().ep_handle_export(self.ptr, _dev_ptr(pos, None, "pos"), _dev_ptr(src, None, "src"),
                                      _dev_ptr(seg, None, "seg"), _dev_ptr(roff, None, "rank_off"),
                                      _stream(stream)), "ep_handle_export")
        return {"pos": pos, "src_idx": src, "seg": seg, "rank_off": roff}

    def counts_host(self, stream=None) -> list:
        """num_recv_tokens_per_expert_list (synchronises the stream)."""
        buf = (ctypes.c_int32 * self.num_experts)()
        _check(lib().ep_handle_counts_host(self.ptr, buf, _stream(stream)), "ep_handle_counts_host")
        return list(buf)

    def check(self, stream=None) -> int:
        """The device error word as a status (synchronises the stream)."""
        return int(lib().ep_handle_check(self.ptr, _stream(stream)))

    def free(self) -> None:
        if self._ptr is not None:
            lib().ep_handle_free(self._ptr)
            self._ptr = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


@dataclass
class LayoutResult:
    num_tokens_per_expert: torch.Tensor   # int32 [E]
    num_tokens_per_rank: torch.Tensor     # int32 [R]
    is_token_in_rank: torch.Tensor        # uint8 [T, R]
    handle: Handle


def ep_layout(topk_idx: torch.Tensor, num_experts: int, num_ranks: int, expert_alignment: int = 1,
              capacity: int = 0, *, num_tokens_per_expert: Optional[torch.Tensor] = None,
              num_tokens_per_rank: Optional[torch.Tensor] = None,
              is_token_in_rank: Optional[torch.Tensor] = None, stream=None) -> LayoutResult:
    if topk_idx.dim() != 2:
        raise ValueError("topk_idx must be [T, k]")
    T, k = topk_idx.shape
    dev = topk_idx.device
    if num_tokens_per_expert is None:
        num_tokens_per_expert = torch.empty(num_experts, dtype=torch.int32, device=dev)
    if num_tokens_per_rank is None:
        num_tokens_per_rank = torch.empty(num_ranks, dtype=torch.int32, device=dev)
    if is_token_in_rank is None:
        is_token_in_rank = torch.empty(T, num_ranks, dtype=torch.uint8, device=dev)
    h = ctypes.c_void_p()
    st = lib().ep_layout(_dev_ptr(topk_idx, torch.int32, "topk_idx"), T, k, num_experts, num_ranks,
                         expert_alignment, capacity,
                         _dev_ptr(num_tokens_per_expert, torch.int32, "num_tokens_per_expert", (num_experts,)),
                         _dev_ptr(num_tokens_per_rank, torch.int32, "num_tokens_per_rank", (num_ranks,)),
                         _dev_ptr(is_token_in_rank, torch.uint8, "is_token_in_rank", (T, num_ranks)),
                         ctypes.byref(h), _stream(stream))
    _check(st, "ep_layout")
    return LayoutResult(num_tokens_per_expert, num_tokens_per_rank, is_token_in_rank, Handle(h, dev))


def ep_dispatch(handle: Handle, x: torch.Tensor, use_fp8: bool, recv_x: Optional[torch.Tensor] = None,
                recv_scales: Optional[torch.Tensor] = None, recv_src_idx: Optional[torch.Tensor] = None,
                stream=None):
    """Returns (recv_x, recv_scales or None, recv_src_idx or None)."""
    T, H = x.shape
    if T != handle.num_tokens:
        raise ValueError("x has %d tokens, the handle %d" % (T, handle.num_tokens))
    rows = handle.num_recv_rows
    dt = torch.float8_e4m3fn if use_fp8 else torch.bfloat16
    if recv_x is None:
        recv_x = torch.empty(rows, H, dtype=dt, device=x.device)
    if use_fp8 and recv_scales is None:
        recv_scales = torch.empty(rows, H // 128, dtype=torch.float32, device=x.device)
    if recv_x.dim() != 2 or recv_x.shape[1] != H:
        raise ValueError("recv_x must be [rows, %d]" % H)
    if use_fp8:
        _check_rows(recv_scales, "recv_scales", recv_x.shape[0], H // 128)
    _check_rows(recv_src_idx, "recv_src_idx", rows)
    st = lib().ep_dispatch(handle.ptr, _dev_ptr(x, torch.bfloat16, "x"), H, 1 if use_fp8 else 0,
                           _dev_ptr(recv_x, dt, "recv_x"),
                           _dev_ptr(recv_scales, torch.float32, "recv_scales") if use_fp8 else None,
                           _dev_ptr(recv_src_idx, torch.int32, "recv_src_idx"),
                           recv_x.shape[0], _stream(stream))
    _check(st, "ep_dispatch")
    return recv_x, (recv_scales if use_fp8 else None), recv_src_idx


def ep_combine(handle: Handle, y: torch.Tensor, topk_weights: torch.Tensor,
               out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    rows, H = y.shape
    if out is None:
        out = torch.empty(handle.num_tokens, H, dtype=torch.bfloat16, device=y.device)
    st = lib().ep_combine(handle.ptr, _dev_ptr(y, torch.bfloat16, "y"),
                          _dev_ptr(topk_weights, torch.float32, "topk_weights",
                                   (handle.num_tokens, handle.num_topk)),
                          H, rows, _dev_ptr(out, torch.bfloat16, "out", (handle.num_tokens, H)),
                          _stream(stream))
    _check(st, "ep_combine")
    return out


def ep_dispatch_ex(handle: Handle, x: torch.Tensor, out_fp8: bool, x_scales: Optional[torch.Tensor] = None,
                   recv_x: Optional[torch.Tensor] = None, recv_scales: Optional[torch.Tensor] = None,
                   scale_layout: str = "row", scale_ld: Optional[int] = None,
                   recv_src_idx: Optional[torch.Tensor] = None, num_sms: int = 0, stream=None):
    """Dispatch with input format (bf16, or e4m3 codes + x_scales), scale
    layout ("row": [rows, H/128]; "col": [H/128, scale_ld]) and SM budget.
    Returns (recv_x, recv_scales or None, recv_src_idx or None)."""
    T, H = x.shape
    if T != handle.num_tokens:
        raise ValueError("x has %d tokens, the handle %d" % (T, handle.num_tokens))
    in_fp8 = x.dtype == torch.float8_e4m3fn
    if not in_fp8 and x.dtype != torch.bfloat16:
        raise ValueError("x must be bf16 or float8_e4m3fn, got %s" % x.dtype)
    if in_fp8 and not out_fp8:
        raise ValueError("e4m3 input needs e4m3 output")
    rows = handle.num_recv_rows if recv_x is None else recv_x.shape[0]
    dt = torch.float8_e4m3fn if out_fp8 else torch.bfloat16
    if recv_x is None:
        recv_x = torch.empty(rows, H, dtype=dt, device=x.device)
    G = H // 128
    s_row, s_grp = G, 1
    if out_fp8:
        if scale_layout == "col":
            if recv_scales is None:
                ld = scale_ld if scale_ld is not None else (rows + 3) // 4 * 4
                recv_scales = torch.empty(G, ld, dtype=torch.float32, device=x.device)
            # scales of row p, group g at g * ld + p: [G, ld] with ld >= rows
            if recv_scales.dim() != 2 or recv_scales.shape[0] != G or recv_scales.shape[1] < rows or \
                    (scale_ld is not None and scale_ld != recv_scales.shape[1]):
                raise ValueError("recv_scales must be [%d, scale_ld >= %d] (column-major), got %s"
                                 % (G, rows, tuple(recv_scales.shape)))
            s_row, s_grp = 1, recv_scales.shape[1]
        elif scale_layout == "row":
            if recv_scales is None:
                recv_scales = torch.empty(rows, G, dtype=torch.float32, device=x.device)
            _check_rows(recv_scales, "recv_scales", rows, G)
        else:
            raise ValueError("scale_layout must be 'row' or 'col'")
    if recv_x.dim() != 2 or recv_x.shape[1] != H:
        raise ValueError("recv_x must be [rows, %d]" % H)
    _check_rows(recv_src_idx, "recv_src_idx", handle.num_recv_rows)
    st = lib().ep_dispatch_ex(handle.ptr, _dev_ptr(x, None, "x"),
                              _dev_ptr(x_scales, torch.float32, "x_scales", (T, G)) if in_fp8 else None,
                              H, EP_FORMAT_E4M3 if in_fp8 else EP_FORMAT_BF16,
                              EP_FORMAT_E4M3 if out_fp8 else EP_FORMAT_BF16,
                              _dev_ptr(recv_x, dt, "recv_x"),
                              _dev_ptr(recv_scales, torch.float32, "recv_scales") if out_fp8 else None,
                              s_row, s_grp, _dev_ptr(recv_src_idx, torch.int32, "recv_src_idx"),
                              rows, num_sms, _stream(stream))
    _check(st, "ep_dispatch_ex")
    return recv_x, (recv_scales if out_fp8 else None), recv_src_idx


def ep_dispatch_fp8_colmajor(handle: Handle, x: torch.Tensor, recv_x: Optional[torch.Tensor] = None,
                             recv_scales: Optional[torch.Tensor] = None, token_scales: Optional[torch.Tensor] = None,
                             recv_src_idx: Optional[torch.Tensor] = None, num_sms: int = 0, stream=None):
    """FP8 dispatch with column-major scales ([H/128, ld], ld >= rows; the
    grouped-GEMM layout) through a per-token scale table.  Returns (recv_x,
    recv_scales [H/128, ld], token_scales [T, H/128], recv_src_idx or None)."""
    T, H = x.shape
    if T != handle.num_tokens:
        raise ValueError("x has %d tokens, the handle %d" % (T, handle.num_tokens))
    if H % 128 != 0:
        raise ValueError("FP8 dispatch needs H %% 128 == 0, got %d" % H)
    G = H // 128
    rows = handle.num_recv_rows if recv_x is None else recv_x.shape[0]
    if recv_x is None:
        recv_x = torch.empty(rows, H, dtype=torch.float8_e4m3fn, device=x.device)
    if recv_x.dim() != 2 or recv_x.shape[1] != H or rows < handle.num_recv_rows:
        raise ValueError("recv_x must be [>= %d, %d], got %s" % (handle.num_recv_rows, H, tuple(recv_x.shape)))
    if recv_scales is None:
        recv_scales = torch.empty(G, (rows + 3) // 4 * 4, dtype=torch.float32, device=x.device)
    if recv_scales.dim() != 2 or recv_scales.shape[0] != G or recv_scales.shape[1] < rows:
        raise ValueError("recv_scales must be [%d, scale_ld >= %d] (column-major), got %s"
                         % (G, rows, tuple(recv_scales.shape)))
    if token_scales is None:
        token_scales = torch.empty(T, G, dtype=torch.float32, device=x.device)
    _check_rows(recv_src_idx, "recv_src_idx", handle.num_recv_rows)
    st = lib().ep_dispatch_fp8_colmajor(handle.ptr, _dev_ptr(x, torch.bfloat16, "x"), H,
                                        _dev_ptr(recv_x, torch.float8_e4m3fn, "recv_x"),
                                        _dev_ptr(recv_scales, torch.float32, "recv_scales"),
                                        recv_scales.shape[1],
                                        _dev_ptr(token_scales, torch.float32, "token_scales", (T, G)),
                                        _dev_ptr(recv_src_idx, torch.int32, "recv_src_idx"),
                                        rows, num_sms, _stream(stream))
    _check(st, "ep_dispatch_fp8_colmajor")
    return recv_x, recv_scales, token_scales, recv_src_idx


def ep_combine_ex(handle: Handle, y: torch.Tensor, topk_weights: torch.Tensor,
                  out: Optional[torch.Tensor] = None, num_sms: int = 0, stream=None) -> torch.Tensor:
    rows, H = y.shape
    if out is None:
        out = torch.empty(handle.num_tokens, H, dtype=torch.bfloat16, device=y.device)
    st = lib().ep_combine_ex(handle.ptr, _dev_ptr(y, torch.bfloat16, "y"),
                             _dev_ptr(topk_weights, torch.float32, "topk_weights",
                                      (handle.num_tokens, handle.num_topk)),
                             H, rows, _dev_ptr(out, torch.bfloat16, "out", (handle.num_tokens, H)),
                             num_sms, _stream(stream))
    _check(st, "ep_combine_ex")
    return out


def ep_dispatch_topk(handle: Handle, topk_weights: Optional[torch.Tensor] = None, want_idx: bool = True,
                     want_slot: bool = True, stream=None):
    """Per-row routing outputs of dispatch: (recv_topk_idx int32 [rows],
    recv_topk_weights fp32 [rows] or None when topk_weights is None,
    recv_slot int32 [rows] or None); -1 / 0 / -1 on rows no slot fills."""
    rows = handle.num_recv_rows
    dev = handle.device
    ri = torch.empty(rows, dtype=torch.int32, device=dev) if want_idx else None
    rw = torch.empty(rows, dtype=torch.float32, device=dev) if topk_weights is not None else None
    rs = torch.empty(rows, dtype=torch.int32, device=dev) if want_slot else None
    st = lib().ep_dispatch_topk(handle.ptr,
                                _dev_ptr(topk_weights, torch.float32, "topk_weights",
                                         (handle.num_tokens, handle.num_topk)),
                                _dev_ptr(ri, torch.int32, "recv_topk_idx"),
                                _dev_ptr(rw, torch.float32, "recv_topk_weights"),
                                _dev_ptr(rs, torch.int32, "recv_slot"), rows, _stream(stream))
    _check(st, "ep_dispatch_topk")
    return ri, rw, rs


def e4m3_encode(x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """fp32 -> e4m3 codes (uint8, same shape) with the dispatch's rounding."""
    if out is None:
        out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    st = lib().ep_e4m3_encode(_dev_ptr(x, torch.float32, "x"), _dev_ptr(out, torch.uint8, "out", tuple(x.shape)),
                              x.numel(), _stream(stream))
    _check(st, "ep_e4m3_encode")
    return out


def ep_dispatch_backward(handle: Handle, grad_recv: torch.Tensor, grad_x: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    """grad_x [T, H] bf16 = sum of each token's receive-row gradients."""
    rows, H = grad_recv.shape
    if grad_x is None:
        grad_x = torch.empty(handle.num_tokens, H, dtype=torch.bfloat16, device=grad_recv.device)
    st = lib().ep_dispatch_backward(handle.ptr, _dev_ptr(grad_recv, torch.bfloat16, "grad_recv"), H, rows,
                                    _dev_ptr(grad_x, torch.bfloat16, "grad_x", (handle.num_tokens, H)),
                                    _stream(stream))
    _check(st, "ep_dispatch_backward")
    return grad_x


def ep_combine_backward(handle: Handle, grad_out: torch.Tensor, topk_weights: torch.Tensor,
                        y: Optional[torch.Tensor] = None, grad_y: Optional[torch.Tensor] = None,
                        grad_weights: Optional[torch.Tensor] = None, want_grad_weights: bool = True,
                        stream=None):
    """Returns (grad_y [rows, H] bf16, grad_weights [T, k] fp32 or None)."""
    T, H = grad_out.shape
    rows = handle.num_recv_rows if y is None else y.shape[0]
    if want_grad_weights and y is None:
        raise ValueError("grad_weights need y (the expert outputs)")
    _check_rows(y, "y", handle.num_recv_rows, H)
    _check_rows(grad_y, "grad_y", handle.num_recv_rows, H)
    if grad_y is None:
        grad_y = torch.empty(rows, H, dtype=torch.bfloat16, device=grad_out.device)
    if want_grad_weights and grad_weights is None:
        grad_weights = torch.empty(T, handle.num_topk, dtype=torch.float32, device=grad_out.device)
    if not want_grad_weights:
        grad_weights = None
    st = lib().ep_combine_backward(handle.ptr, _dev_ptr(grad_out, torch.bfloat16, "grad_out", (handle.num_tokens, H)),
                                   _dev_ptr(y, torch.bfloat16, "y"),
                                   _dev_ptr(topk_weights, torch.float32, "topk_weights",
                                            (handle.num_tokens, handle.num_topk)),
                                   H, grad_y.shape[0], _dev_ptr(grad_y, torch.bfloat16, "grad_y"),
                                   _dev_ptr(grad_weights, torch.float32, "grad_weights",
                                            (handle.num_tokens, handle.num_topk)), _stream(stream))
    _check(st, "ep_combine_backward")
    return grad_y, grad_weights


def ep_handle_free(handle: Handle) -> None:
    handle.free()


def ep_layout_noalloc(topk_idx: torch.Tensor, num_experts: int, num_ranks: int,
                      pos: torch.Tensor, src_idx: torch.Tensor, seg: torch.Tensor,
                      rank_off: torch.Tensor, expert_alignment: int = 1, capacity: int = 0, *,
                      num_tokens_per_expert: Optional[torch.Tensor] = None,
                      num_tokens_per_rank: Optional[torch.Tensor] = None,
                      is_token_in_rank: Optional[torch.Tensor] = None,
                      error_word: Optional[torch.Tensor] = None, stream=None) -> None:
    """The layout into caller-owned buffers only (see ep_layout_noalloc in
    include/ep.h): for callers that cannot allocate device memory.  This
    wrapper allocates nothing either; every buffer is passed in."""
    T, k = topk_idx.shape
    rows = ep_max_recv_rows(T, k, num_experts, expert_alignment, capacity)
    st = lib().ep_layout_noalloc(
        _dev_ptr(topk_idx, torch.int32, "topk_idx"), T, k, num_experts, num_ranks,
        expert_alignment, capacity,
        _dev_ptr(num_tokens_per_expert, torch.int32, "num_tokens_per_expert", (num_experts,)),
        _dev_ptr(num_tokens_per_rank, torch.int32, "num_tokens_per_rank", (num_ranks,)),
        _dev_ptr(is_token_in_rank, torch.uint8, "is_token_in_rank", (T, num_ranks)),
        _dev_ptr(pos, torch.int32, "pos", (T, k)), _dev_ptr(src_idx, torch.int32, "src_idx", (rows,)),
        _dev_ptr(seg, torch.int32, "seg", (num_experts + 1,)),
        _dev_ptr(rank_off, torch.int32, "rank_off", (num_ranks + 1,)),
        _dev_ptr(error_word, torch.int32, "error_word", (1,)), _stream(stream))
    _check(st, "ep_layout_noalloc")


# ---------------------------------------------------------------------------
# Expert parallelism across GPUs (one process per GPU)
# ---------------------------------------------------------------------------

def ep_peer_max_recv_rows(total_tokens: int, num_topk: int, num_experts: int, world: int,
                          expert_alignment: int = 1, capacity: int = 0) -> int:
    return int(lib().ep_peer_max_recv_rows(total_tokens, num_topk, num_experts, world, expert_alignment,
                                           capacity))


class Plan:
    """Owner of an ep_plan*: the (rank, row) of every local slot on its owner."""

    def __init__(self, ptr: ctypes.c_void_p, device, num_tokens: int, num_topk: int, num_experts: int,
                 rank: int, world: int):
        self._ptr = ptr
        self.device = device
        self.num_tokens, self.num_topk, self.num_experts = num_tokens, num_topk, num_experts
        self.rank, self.world = rank, world
        self.experts_per_rank = num_experts // world

    @property
    def ptr(self) -> ctypes.c_void_p:
        if self._ptr is None:
            raise RuntimeError("plan already freed")
        return self._ptr

    def export(self, stream=None) -> dict:
        """Device copies of dst [T,k,2], recv_seg [E/W+1], recv_counts [E/W]."""
        dev = self.device
        dst = torch.empty(self.num_tokens, self.num_topk, 2, dtype=torch.int32, device=dev)
        seg = torch.empty(self.experts_per_rank + 1, dtype=torch.int32, device=dev)
        cnt = torch.empty(self.experts_per_rank, dtype=torch.int32, device=dev)
        _check(lib().ep_plan_export(self.ptr, _dev_ptr(dst, None, "dst"), _dev_ptr(seg, None, "recv_seg"),
                                    _dev_ptr(cnt, None, "recv_counts"), _stream(stream)), "ep_plan_export")
        return {"dst": dst, "recv_seg": seg, "recv_counts": cnt}

    def recv_rows_host(self, stream=None) -> int:
        n = ctypes.c_int64(0)
        _check(lib().ep_plan_recv_rows_host(self.ptr, ctypes.byref(n), _stream(stream)), "ep_plan_recv_rows_host")
        return int(n.value)

    def check(self, stream=None) -> int:
        return int(lib().ep_plan_check(self.ptr, _stream(stream)))

    def free(self) -> None:
        if self._ptr is not None:
            lib().ep_plan_free(self._ptr)
            self._ptr = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def ep_plan_create(local: Handle, topk_idx: torch.Tensor, all_counts: torch.Tensor, rank: int, world: int,
                   recv_rows: int, expert_alignment: int = 1, capacity: int = 0, stream=None) -> Plan:
    """Plan of this rank from its local layout handle (made with num_ranks =
    world, alignment 1, capacity 0) and the all-gathered counts [world, E]."""
    out = ctypes.c_void_p()
    T, k = local.num_tokens, local.num_topk
    st = lib().ep_plan_create(local.ptr, _dev_ptr(topk_idx, torch.int32, "topk_idx", (T, k)),
                              _dev_ptr(all_counts, torch.int32, "all_counts", (world, local.num_experts)),
                              rank, world, expert_alignment, capacity, recv_rows, ctypes.byref(out),
                              _stream(stream))
    _check(st, "ep_plan_create")
    return Plan(out, topk_idx.device, T, k, local.num_experts, rank, world)


def _ptr_array(ptrs):
    arr = (ctypes.c_void_p * len(ptrs))()
    for i, p in enumerate(ptrs):
        arr[i] = int(p.data_ptr()) if isinstance(p, torch.Tensor) else int(p)
    return arr


class Peers:
    """Owner of an ep_peers*: every rank's buffers as addressed from this process."""

    def __init__(self, world: int, recv_x, recv_scales, y, recv_rows: int, grad_y=None):
        out = ctypes.c_void_p()
        st = lib().ep_peers_create(world, _ptr_array(recv_x),
                                   _ptr_array(recv_scales) if recv_scales is not None else None,
                                   _ptr_array(y) if y is not None else None,
                                   _ptr_array(grad_y) if grad_y is not None else None, recv_rows,
                                   ctypes.byref(out))
        _check(st, "ep_peers_create")
        self._ptr = out
        self.world = world
        self.recv_rows = recv_rows

    @property
    def ptr(self) -> ctypes.c_void_p:
        if self._ptr is None:
            raise RuntimeError("peer table already freed")
        return self._ptr

    def set_topk(self, recv_topk_idx=None, recv_topk_weights=None, recv_src_rank=None, recv_slot=None):
        """Register every rank's per-row output tables (lists of `world`
        tensors or device addresses, each [recv_rows])."""
        arrs = [_ptr_array(t) if t is not None else None
                for t in (recv_topk_idx, recv_topk_weights, recv_src_rank, recv_slot)]
        _check(lib().ep_peers_set_topk(self.ptr, *arrs), "ep_peers_set_topk")

    def free(self) -> None:
        if self._ptr is not None:
            lib().ep_peers_free(self._ptr)
            self._ptr = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def ep_dispatch_peer(plan: Plan, peers: Peers, x: torch.Tensor, use_fp8: bool,
                     x_scales: Optional[torch.Tensor] = None, num_sms: int = 0,
                     scale_layout: str = "row", scale_ld: Optional[int] = None, stream=None) -> None:
    """Stores every local token's rows (BF16, fused FP8, or pre-quantised FP8
    when x is float8_e4m3fn with x_scales) into the owners' receive buffers;
    scales row-major [rows, H/128] or column-major [H/128, scale_ld]
    (scale_ld >= the peer table's recv_rows, default recv_rows)."""
    T, H = x.shape
    in_fp8 = x.dtype == torch.float8_e4m3fn
    if not in_fp8 and x.dtype != torch.bfloat16:
        raise ValueError("x must be bf16 or float8_e4m3fn, got %s" % x.dtype)
    if in_fp8 and not use_fp8:
        raise ValueError("FP8 input needs FP8 output")
    if scale_layout == "row":
        s_row, s_grp = H // 128, 1
    elif scale_layout == "col":
        s_row, s_grp = 1, scale_ld if scale_ld is not None else peers.recv_rows
    else:
        raise ValueError("scale_layout must be 'row' or 'col'")
    st = lib().ep_dispatch_peer(plan.ptr, peers.ptr, _dev_ptr(x, x.dtype, "x", (plan.num_tokens, H)),
                                _dev_ptr(x_scales, torch.float32, "x_scales", (plan.num_tokens, H // 128)), H,
                                EP_FORMAT_E4M3 if in_fp8 else EP_FORMAT_BF16,
                                EP_FORMAT_E4M3 if use_fp8 else EP_FORMAT_BF16, s_row, s_grp, num_sms,
                                _stream(stream))
    _check(st, "ep_dispatch_peer")


def ep_combine_peer(plan: Plan, peers: Peers, topk_weights: Optional[torch.Tensor], hidden: int,
                    out: Optional[torch.Tensor] = None, num_sms: int = 0, stream=None) -> torch.Tensor:
    """[T, H] bf16: each local token's weighted sum of its expert outputs read
    from the owners' y buffers (topk_weights None: unit weights)."""
    if out is None:
        out = torch.empty(plan.num_tokens, hidden, dtype=torch.bfloat16, device=plan.device)
    st = lib().ep_combine_peer(plan.ptr, peers.ptr,
                               _dev_ptr(topk_weights, torch.float32, "topk_weights",
                                        (plan.num_tokens, plan.num_topk)),
                               hidden, _dev_ptr(out, torch.bfloat16, "out", (plan.num_tokens, hidden)),
                               num_sms, _stream(stream))
    _check(st, "ep_combine_peer")
    return out


def ep_combine_backward_peer(plan: Plan, peers: Peers, grad_out: torch.Tensor, topk_weights: torch.Tensor,
                             want_grad_weights: bool = True, grad_weights: Optional[torch.Tensor] = None,
                             stream=None) -> Optional[torch.Tensor]:
    """Stores each local slot's gradient row into its owner's grad_y buffer;
    returns grad_weights [T, k] fp32 (dot products with the owners' y rows) or None."""
    T, H = grad_out.shape
    if want_grad_weights and grad_weights is None:
        grad_weights = torch.empty(T, plan.num_topk, dtype=torch.float32, device=grad_out.device)
    if not want_grad_weights:
        grad_weights = None
    st = lib().ep_combine_backward_peer(plan.ptr, peers.ptr,
                                        _dev_ptr(grad_out, torch.bfloat16, "grad_out", (plan.num_tokens, H)),
                                        _dev_ptr(topk_weights, torch.float32, "topk_weights",
                                                 (plan.num_tokens, plan.num_topk)),
                                        H, _dev_ptr(grad_weights, torch.float32, "grad_weights",
                                                    (plan.num_tokens, plan.num_topk)), _stream(stream))
    _check(st, "ep_combine_backward_peer")
    return grad_weights


def ep_dispatch_topk_peer(plan: Plan, peers: Peers, topk_idx: torch.Tensor,
                          topk_weights: Optional[torch.Tensor] = None, stream=None) -> None:
    """Writes every local slot's expert id, weight, rank and slot index into
    its owner's per-row tables (Peers.set_topk) and fills this rank's own
    padding rows with -1 / 0 / -1 / -1."""
    st = lib().ep_dispatch_topk_peer(plan.ptr, peers.ptr,
                                     _dev_ptr(topk_idx, torch.int32, "topk_idx", (plan.num_tokens, plan.num_topk)),
                                     _dev_ptr(topk_weights, torch.float32, "topk_weights",
                                              (plan.num_tokens, plan.num_topk)), _stream(stream))
    _check(st, "ep_dispatch_topk_peer")


def ipc_export(t: torch.Tensor):
    """(64-byte handle, offset) of the allocation holding t, for another process."""
    h = ctypes.create_string_buffer(EP_IPC_HANDLE_BYTES)
    off = ctypes.c_uint64(0)
    _check(lib().ep_ipc_export(_dev_ptr(t, None, "t"), h, ctypes.byref(off)), "ep_ipc_export")
    return h.raw, int(off.value)


def ipc_import(handle: bytes, offset: int) -> int:
    """Device address, in this process, of another process's exported buffer."""
    if len(handle) != EP_IPC_HANDLE_BYTES:
        raise ValueError("IPC handle must be %d bytes" % EP_IPC_HANDLE_BYTES)
    out = ctypes.c_void_p()
    _check(lib().ep_ipc_import(handle, offset, ctypes.byref(out)), "ep_ipc_import")
    return int(out.value)


def ipc_release(ptr: int, offset: int) -> None:
    _check(lib().ep_ipc_release(ctypes.c_void_p(ptr), offset), "ep_ipc_release")
