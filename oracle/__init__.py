"""CPU oracle for the MoE expert-parallel layout / dispatch / combine path.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg (and its ``--impl reference`` arm) may import
this package.  It shares no code with the CUDA library and the CUDA library
never imports it.

The arithmetic lives in ``ep_oracle.c`` (plain single-threaded C, IEEE binary32
without contraction); this module only marshals numpy arrays through ctypes.
Each C function's header comment cites the passage of the pages it follows.

Status codes returned by the C functions (the oracle's own numbering):
    0 ok, 1 invalid argument, 2 expert id outside [-1, E), 3 capacity overflow.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import numpy as np

from . import build as _build

OR_OK = 0
OR_ERR_INVALID_ARG = 1
OR_ERR_BAD_EXPERT_ID = 2
OR_ERR_CAPACITY = 3

_LIB = None


class OracleError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__("%s failed with oracle status %d" % (what, status))
        self.status = status


def lib():
    """Load (building first if needed) the oracle shared library."""
    global _LIB
    if _LIB is None:
        _LIB = load(_build.build())
    return _LIB


def load(path: str):
    """Load an oracle library from `path` and declare its functions."""
    if True:
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i32, i64 = ctypes.c_int, ctypes.c_int64
        L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_f32.restype = ctypes.c_float
        L.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        L.oracle_f32_to_bf16.restype = ctypes.c_uint16
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_decode.restype = ctypes.c_float
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_encode_n.argtypes = [P, P, i64]
        L.oracle_e4m3_encode_n.restype = None
        L.oracle_f32_to_bf16_n.argtypes = [P, P, i64]
        L.oracle_f32_to_bf16_n.restype = None
        L.oracle_max_recv_rows.argtypes = [i32, i32, i32, i32, i32]
        L.oracle_max_recv_rows.restype = i64
        L.oracle_layout.argtypes = [P, i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, P, i64]
        L.oracle_layout.restype = i32
        L.oracle_dispatch_bf16.argtypes = [P, i32, i32, i32, P, P, i64]
        L.oracle_dispatch_bf16.restype = i32
        L.oracle_dispatch_fp8.argtypes = [P, i32, i32, i32, P, P, P, i64]
        L.oracle_dispatch_fp8.restype = i32
        L.oracle_quantize_group.argtypes = [P, P, P]
        L.oracle_quantize_group.restype = None
        L.oracle_combine.argtypes = [P, i64, i32, P, P, i32, i32, P]
        L.oracle_combine.restype = i32
        L.oracle_combine_backward.argtypes = [P, P, i64, i32, P, P, i32, i32, P, P]
        L.oracle_combine_backward.restype = i32
        L.oracle_dispatch_fp8_prequant.argtypes = [P, P, i32, i32, i32, P, P, P, i64]
        L.oracle_dispatch_fp8_prequant.restype = i32
        L.oracle_dispatch_topk.argtypes = [P, P, i32, i32, P, i64, P, P, P]
        L.oracle_dispatch_topk.restype = i32
    return L


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    """bf16 data as its raw 16-bit patterns (accepts a torch bf16 tensor or uint16 array)."""
    if hasattr(a, "view") and hasattr(a, "dtype") and str(a.dtype) == "torch.bfloat16":
        import torch
        return np.ascontiguousarray(a.contiguous().view(torch.int16).numpy().view(np.uint16))
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


# ---------------------------------------------------------------------------
# Number formats
# ---------------------------------------------------------------------------

def bf16_to_f32(h: int) -> float:
    return float(lib().oracle_bf16_to_f32(int(h)))


def f32_to_bf16(f: float) -> int:
    return int(lib().oracle_f32_to_bf16(float(f)))


def e4m3_decode(code: int) -> float:
    return float(lib().oracle_e4m3_decode(int(code)))


def e4m3_encode(v: float) -> int:
    return int(lib().oracle_e4m3_encode(float(v)))


def e4m3_encode_array(v: np.ndarray) -> np.ndarray:
    """Encode every element of a float32 array with the oracle's e4m3 encoder."""
    v = np.ascontiguousarray(v, dtype=np.float32).ravel()
    out = np.empty(v.shape, dtype=np.uint8)
    lib().oracle_e4m3_encode_n(_ptr(v), _ptr(out), v.size)
    return out


def f32_to_bf16_array(v: np.ndarray) -> np.ndarray:
    """Round every element of a float32 array to bf16 bits with the oracle's rounding."""
    v = np.ascontiguousarray(v, dtype=np.float32).ravel()
    out = np.empty(v.shape, dtype=np.uint16)
    lib().oracle_f32_to_bf16_n(_ptr(v), _ptr(out), v.size)
    return out


# ---------------------------------------------------------------------------
# Layout / dispatch / combine
# ---------------------------------------------------------------------------

def max_recv_rows(T: int, k: int, E: int, align: int = 1, capacity: int = 0) -> int:
    return int(lib().oracle_max_recv_rows(T, k, E, align, capacity))


@dataclass
class Layout:
    """The oracle's routing layout (the content of the pages' handle)."""
    T: int
    k: int
    E: int
    R: int
    align: int
    capacity: int
    n_rows: int
    num_tokens_per_expert: np.ndarray  # int32 [E]
    num_tokens_per_rank: np.ndarray    # int32 [R]
    is_token_in_rank: np.ndarray       # uint8 [T, R]
    seg: np.ndarray                    # int32 [E+1]
    rank_off: np.ndarray               # int32 [R+1]
    pos: np.ndarray                    # int32 [T, k]
    src_idx: np.ndarray                # int32 [n_rows]


def layout(topk_idx: np.ndarray, E: int, R: int, align: int = 1, capacity: int = 0,
           n_rows: int | None = None, check: bool = True):
    """Run the oracle layout; returns (status, Layout)."""
    idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    T, k = idx.shape
    if n_rows is None:
        n_rows = max(max_recv_rows(T, k, E, align, capacity), 0)
    cnt = np.zeros(E, np.int32)
    rank_tok = np.zeros(R, np.int32)
    in_rank = np.zeros((T, R), np.uint8)
    seg = np.zeros(E + 1, np.int32)
    rank_off = np.zeros(R + 1, np.int32)
    pos = np.zeros((T, k), np.int32)
    src = np.zeros(max(n_rows, 1), np.int32)
    st = lib().oracle_layout(_ptr(idx), T, k, E, R, align, capacity, _ptr(cnt), _ptr(rank_tok),
                             _ptr(in_rank), _ptr(seg), _ptr(rank_off), _ptr(pos), _ptr(src), n_rows)
    if check and st != OR_OK:
        raise OracleError(st, "oracle_layout")
    return st, Layout(T, k, E, R, align, capacity, n_rows, cnt, rank_tok, in_rank, seg, rank_off,
                      pos, src[:n_rows])


def dispatch_bf16(x, pos: np.ndarray, n_rows: int) -> np.ndarray:
    """x: bf16 [T, H] (torch tensor or uint16 array).  Returns uint16 [n_rows, H]; rows that
    no slot maps to are left zero."""
    xb = _u16(x)
    T, H = xb.shape
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    k = pos.shape[1]
    recv = np.zeros((n_rows, H), np.uint16)
    st = lib().oracle_dispatch_bf16(_ptr(xb), T, H, k, _ptr(pos), _ptr(recv), n_rows)
    if st != OR_OK:
        raise OracleError(st, "oracle_dispatch_bf16")
    return recv


def dispatch_fp8(x, pos: np.ndarray, n_rows: int):
    """Returns (codes uint8 [n_rows, H], scales float32 [n_rows, H/128]); unmapped rows zero."""
    xb = _u16(x)
    T, H = xb.shape
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    k = pos.shape[1]
    recv = np.zeros((n_rows, H), np.uint8)
    scales = np.zeros((n_rows, H // 128), np.float32)
    st = lib().oracle_dispatch_fp8(_ptr(xb), T, H, k, _ptr(pos), _ptr(recv), _ptr(scales), n_rows)
    if st != OR_OK:
        raise OracleError(st, "oracle_dispatch_fp8")
    return recv, scales


def quantize_rows(x) -> tuple[np.ndarray, np.ndarray]:
    """Per-token FP8 quantisation (the dispatch's per-group step) of a whole
    bf16 [T, H] batch: (codes uint8 [T, H], scales float32 [T, H/128])."""
    xb = _u16(x)
    T, H = xb.shape
    pos = np.arange(T, dtype=np.int32)[:, None]
    return dispatch_fp8(xb, pos, T)


def dispatch_fp8_prequant(xq: np.ndarray, xs: np.ndarray, pos: np.ndarray, n_rows: int):
    """Dispatch of already-quantised input: bit copies of codes and scales."""
    xq = np.ascontiguousarray(xq, dtype=np.uint8)
    xs = np.ascontiguousarray(xs, dtype=np.float32)
    T, H = xq.shape
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    k = pos.shape[1]
    recv = np.zeros((n_rows, H), np.uint8)
    scales = np.zeros((n_rows, H // 128), np.float32)
    st = lib().oracle_dispatch_fp8_prequant(_ptr(xq), _ptr(xs), T, H, k, _ptr(pos), _ptr(recv),
                                            _ptr(scales), n_rows)
    if st != OR_OK:
        raise OracleError(st, "oracle_dispatch_fp8_prequant")
    return recv, scales


def quantize_group(xg) -> tuple[np.ndarray, float]:
    """Quantise one 128-channel bf16 group; returns (codes uint8 [128], scale)."""
    xb = _u16(xg).ravel()
    assert xb.size == 128
    q = np.zeros(128, np.uint8)
    s = np.zeros(1, np.float32)
    lib().oracle_quantize_group(_ptr(xb), _ptr(q), _ptr(s))
    return q, float(s[0])


def dispatch_topk(topk_idx, w, pos: np.ndarray, n_rows: int):
    """Per-row routing outputs of dispatch: (recv_topk_idx int32 [n_rows],
    recv_topk_weights float32 [n_rows], recv_slot int32 [n_rows]); -1 / 0 / -1
    on rows no slot fills."""
    idx = np.ascontiguousarray(np.asarray(topk_idx), dtype=np.int32)
    w = np.ascontiguousarray(np.asarray(w), dtype=np.float32)
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    T, k = pos.shape
    assert idx.shape == (T, k) and w.shape == (T, k)
    ri = np.empty(n_rows, np.int32)
    rw = np.empty(n_rows, np.float32)
    rs = np.empty(n_rows, np.int32)
    st = lib().oracle_dispatch_topk(_ptr(idx), _ptr(w), T, k, _ptr(pos), n_rows, _ptr(ri), _ptr(rw), _ptr(rs))
    if st != OR_OK:
        raise OracleError(st, "oracle_dispatch_topk")
    return ri, rw, rs


def combine(y, w: np.ndarray, pos: np.ndarray) -> np.ndarray:
    """y: bf16 [n_rows, H]; w: float32 [T, k]; pos: int32 [T, k].  Returns uint16 [T, H]."""
    yb = _u16(y)
    n_rows, H = yb.shape
    w = np.ascontiguousarray(w, dtype=np.float32)
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    T, k = pos.shape
    out = np.zeros((T, H), np.uint16)
    st = lib().oracle_combine(_ptr(yb), n_rows, H, _ptr(w), _ptr(pos), T, k, _ptr(out))
    if st != OR_OK:
        raise OracleError(st, "oracle_combine")
    return out


def dispatch_backward(grad_recv, pos: np.ndarray) -> np.ndarray:
    """Gradient of x from the gradients of the receive rows: the combine with
    every weight 1 (uint16 bf16 bits [T, H])."""
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    return combine(grad_recv, np.ones(pos.shape, np.float32), pos)


def combine_backward(grad_out, y, w: np.ndarray, pos: np.ndarray):
    """Returns (grad_y uint16 [n_rows, H], rows never written are 0;
    grad_w float64 [T, k])."""
    gb = _u16(grad_out)
    yb = _u16(y)
    n_rows, H = yb.shape
    w = np.ascontiguousarray(w, dtype=np.float32)
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    T, k = pos.shape
    grad_y = np.zeros((n_rows, H), np.uint16)
    grad_w = np.zeros((T, k), np.float64)
    st = lib().oracle_combine_backward(_ptr(gb), _ptr(yb), n_rows, H, _ptr(w), _ptr(pos), T, k,
                                       _ptr(grad_y), _ptr(grad_w))
    if st != OR_OK:
        raise OracleError(st, "oracle_combine_backward")
    return grad_y, grad_w


def bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 values (exact widening)."""
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)
