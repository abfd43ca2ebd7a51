"""Per-row routing outputs of dispatch (ep_dispatch_topk) against the oracle (GPU).

Bit-exact: expert ids and slot ids are integers and the weights are copies.
Cases cover the one-CTA and the tiled layout paths, padded (capacity) and
aligned segments, unused slots, a token naming one expert twice, and the
full-size metric workload.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from combine_ep_layout_10_b200 import ep
from combine_ep_layout_10_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from combine_ep_layout_10_b200 import build
    build.build()
    ep.lib()
    oracle.lib()


def routing(name, T=None, unused=False, dup=False):
    w = W.WORKLOADS[name]
    w = w.scaled(T=T) if T else w
    _, idx, tw = W.make_routing(w)
    if unused:
        idx[::5, -1] = -1
    if dup:
        idx[1::7, 0] = idx[1::7, 1]
    return w, idx, tw


@pytest.mark.parametrize("name,T,align,cap,unused,dup", [
    ("tiny", None, 1, 0, False, False),
    ("tiny", None, 1, 0, True, True),
    ("tiny", None, 4, 0, True, False),
    ("prefill", 300, 1, 0, True, True),
    ("decode", None, 1, 128, False, False),
    ("decode", None, 1, 160, True, True),
    ("group_limited", 2048, 8, 0, True, False),   # tiled layout path
    ("group_limited", None, 1, 0, False, False),  # metric workload, full size
    ("large_skewed", None, 1, 0, True, False),
])
def test_dispatch_topk_matches_oracle(name, T, align, cap, unused, dup):
    w, idx, tw = routing(name, T, unused, dup)
    res = ep.ep_layout(idx.to(DEV), w.E, w.R, align, cap)
    h = res.handle
    ri, rw, rs = ep.ep_dispatch_topk(h, tw.to(DEV))
    torch.cuda.synchronize()
    _, L = oracle.layout(idx.numpy(), w.E, w.R, align, cap)
    assert h.num_recv_rows == L.n_rows
    oi, ow, os_ = oracle.dispatch_topk(idx.numpy(), tw.numpy(), L.pos, L.n_rows)
    assert (ri.cpu().numpy() == oi).all()
    assert (rw.cpu().numpy().view(np.uint32) == ow.view(np.uint32)).all()
    assert (rs.cpu().numpy() == os_).all()


def test_subsets_of_outputs_and_rows_past_the_handle():
    w, idx, tw = routing("prefill", 257, unused=True)
    res = ep.ep_layout(idx.to(DEV), w.E, w.R)
    h = res.handle
    _, L = oracle.layout(idx.numpy(), w.E, w.R)
    oi, ow, os_ = oracle.dispatch_topk(idx.numpy(), tw.numpy(), L.pos, L.n_rows)
    # weights only
    ri, rw, rs = ep.ep_dispatch_topk(h, tw.to(DEV), want_idx=False, want_slot=False)
    assert ri is None and rs is None
    assert (rw.cpu().numpy().view(np.uint32) == ow.view(np.uint32)).all()
    # ids only, into a longer buffer whose tail must stay untouched
    rows = h.num_recv_rows
    buf = torch.full((rows + 37,), 12345, dtype=torch.int32, device=DEV)
    st = ep.lib().ep_dispatch_topk(h.ptr, None, ctypes.c_void_p(buf.data_ptr()), None, None, rows + 37,
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == ep.EP_OK
    got = buf.cpu().numpy()
    assert (got[:rows] == oi).all() and (got[rows:] == 12345).all()
    # argument errors: buffer shorter than the handle's rows; weights out without weights in
    S = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert ep.lib().ep_dispatch_topk(h.ptr, None, ctypes.c_void_p(buf.data_ptr()), None, None, rows - 1,
                                     S) == ep.EP_ERR_INVALID_ARG
    assert ep.lib().ep_dispatch_topk(h.ptr, None, None, ctypes.c_void_p(buf.data_ptr()), None, rows + 37,
                                     S) == ep.EP_ERR_INVALID_ARG


def test_cached_handle_in_a_graph():
    """The decode pattern: new weights each step through one captured graph."""
    w, idx, tw = routing("decode")
    res = ep.ep_layout(idx.to(DEV), w.E, w.R, 1, w.capacity)
    h = res.handle
    _, L = oracle.layout(idx.numpy(), w.E, w.R, 1, w.capacity)
    twd = tw.to(DEV).clone()
    ri, rw, rs = ep.ep_dispatch_topk(h, twd)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            st = ep.lib().ep_dispatch_topk(h.ptr, ctypes.c_void_p(twd.data_ptr()), None,
                                           ctypes.c_void_p(rw.data_ptr()), None, h.num_recv_rows,
                                           ctypes.c_void_p(s.cuda_stream))
    assert st == ep.EP_OK
    for step in range(3):
        new_w = torch.rand(w.T, w.k, generator=torch.Generator().manual_seed(100 + step))
        twd.copy_(new_w.to(DEV))
        g.replay()
        torch.cuda.synchronize()
        _, ow, _ = oracle.dispatch_topk(idx.numpy(), new_w.numpy(), L.pos, L.n_rows)
        assert (rw.cpu().numpy().view(np.uint32) == ow.view(np.uint32)).all()
    del g


@pytest.mark.parametrize("k", [1, 3, 6, 12, 17, 32])
@pytest.mark.parametrize("w_offset", [0, 1])
def test_topk_widths_and_weight_alignment(k, w_offset):
    """Every k (the scalar path for k % 4 != 0, 16-byte loads otherwise, the
    32-slot variant above 8) and weights that are 4- but not 16-byte aligned."""
    w = W.WORKLOADS["tiny"].scaled(E=64, k=k, T=200)
    _, idx, tw = W.make_routing(w)
    idx[::9, 0] = -1
    res = ep.ep_layout(idx.to(DEV), w.E, w.R)
    h = res.handle
    flat = torch.zeros(tw.numel() + 4, dtype=torch.float32, device=DEV)
    flat[w_offset:w_offset + tw.numel()] = tw.reshape(-1).to(DEV)
    twd = flat[w_offset:w_offset + tw.numel()].view(w.T, k)
    assert (twd.data_ptr() % 16 == 0) == (w_offset == 0)
    ri, rw, rs = ep.ep_dispatch_topk(h, twd)
    torch.cuda.synchronize()
    _, L = oracle.layout(idx.numpy(), w.E, w.R)
    oi, ow, os_ = oracle.dispatch_topk(idx.numpy(), tw.numpy(), L.pos, L.n_rows)
    assert (ri.cpu().numpy() == oi).all()
    assert (rw.cpu().numpy().view(np.uint32) == ow.view(np.uint32)).all()
    assert (rs.cpu().numpy() == os_).all()
