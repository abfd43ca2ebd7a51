"""ep_dispatch_ex / ep_combine_ex options against the oracle (GPU).

* pre-quantised FP8 input (codes + scales) is copied bit-exactly;
* a column-major scale layout holds exactly the row-major scales, transposed;
* an SM budget (num_sms) changes the launch shape, never the result;
* the column-major fill pass is exact on back-to-back calls and graph
  replays, also where it starts before the kernel it follows completes.
"""
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


def u8(t):
    return t.contiguous().view(torch.uint8).cpu().numpy()


def u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def setup(name, T=None):
    w = W.WORKLOADS[name]
    w = w.scaled(T=T) if T else w
    x, idx, tw = W.make_routing(w)
    res = ep.ep_layout(idx.to(DEV), w.E, w.R, w.align, w.capacity)
    _, L = oracle.layout(idx.numpy(), w.E, w.R, w.align, w.capacity)
    return w, x, tw, res, L


@pytest.mark.parametrize("name,T", [("prefill", 300), ("decode", None), ("group_limited", 512)])
def test_prequantised_input(name, T):
    w, x, tw, res, L = setup(name, T)
    xq, xs = oracle.quantize_rows(x)
    xq_d = torch.from_numpy(xq).to(DEV).view(torch.float8_e4m3fn)
    xs_d = torch.from_numpy(xs).to(DEV)
    recv, sc, _ = ep.ep_dispatch_ex(res.handle, xq_d, True, x_scales=xs_d)
    torch.cuda.synchronize()
    q, s = oracle.dispatch_fp8_prequant(xq, xs, L.pos, L.n_rows)
    valid = L.src_idx >= 0
    assert (u8(recv)[valid] == q[valid]).all()
    assert (sc.cpu().numpy()[valid].view(np.uint32) == s[valid].view(np.uint32)).all()
    # and it is the fused FP8 dispatch, exactly
    q2, s2 = oracle.dispatch_fp8(x, L.pos, L.n_rows)
    assert (q[valid] == q2[valid]).all() and (s[valid] == s2[valid]).all()


@pytest.mark.parametrize("prequant", [False, True])
def test_column_major_scales(prequant):
    w, x, tw, res, L = setup("prefill", 257)
    rows = res.handle.num_recv_rows
    ld = (rows + 3) // 4 * 4
    if prequant:
        xq, xs = oracle.quantize_rows(x)
        xin = torch.from_numpy(xq).to(DEV).view(torch.float8_e4m3fn)
        xsd = torch.from_numpy(xs).to(DEV)
    else:
        xin, xsd = x.to(DEV), None
    sc_col = torch.full((w.H // 128, ld), -3.0, dtype=torch.float32, device=DEV)
    recv, sc, _ = ep.ep_dispatch_ex(res.handle, xin, True, x_scales=xsd, recv_scales=sc_col,
                                    scale_layout="col", scale_ld=ld)
    torch.cuda.synchronize()
    q, s = oracle.dispatch_fp8(x, L.pos, L.n_rows)
    valid = L.src_idx >= 0
    got = sc.cpu().numpy()
    assert (got[:, :rows].T[valid].view(np.uint32) == s[valid].view(np.uint32)).all()
    assert (got[:, :rows].T[~valid] == -3.0).all() and (got[:, rows:] == -3.0).all()
    assert (u8(recv)[valid] == q[valid]).all()


@pytest.mark.parametrize("num_sms", [1, 3, 16, 1000])
def test_sm_budget_changes_nothing(num_sms):
    for name, fp8 in (("group_limited", True), ("large_skewed", False)):
        w, x, tw, res, L = setup(name, 1024)
        h = res.handle
        xd = x.to(DEV)
        r0, s0, _ = ep.ep_dispatch_ex(h, xd, fp8)
        r1, s1, _ = ep.ep_dispatch_ex(h, xd, fp8, num_sms=num_sms)
        y = W.make_expert_out(h.num_recv_rows, w.H, seed=5).to(DEV)
        twd = tw.to(DEV)
        o0 = ep.ep_combine_ex(h, y, twd)
        o1 = ep.ep_combine_ex(h, y, twd, num_sms=num_sms)
        torch.cuda.synchronize()
        valid = torch.from_numpy(L.src_idx >= 0).to(DEV)
        assert torch.equal(r0.view(torch.uint8)[valid], r1.view(torch.uint8)[valid])
        if fp8:
            assert torch.equal(s0[valid], s1[valid])
        assert torch.equal(o0.view(torch.int16), o1.view(torch.int16))
        assert (u16(o0) == oracle.combine(y.cpu(), tw.numpy(), L.pos)).all()


@pytest.mark.parametrize("num_sms,T,H,k", [(1, 700, 8192 + 128, 8), (3, 700, 8192 + 128, 8),
                                            (2, 300, 1024, 32), (5, 333, 640, 1)])
def test_sm_budget_pipelined_kernels_against_the_oracle(num_sms, T, H, k):
    """The grid-stride kernels an SM budget runs (the next unit's inputs are
    loaded while the current unit is stored, row pointers double-buffered)
    against the oracle itself: FP8 quantising and pre-quantised dispatch, BF16
    dispatch and combine, with unused slots, a token with no slot and a
    padded layout; two chunks per token (H = 8320 > 8192 channels), so that
    every block walks many units of both chunk positions, and the extremes of
    top-k (32 slots: the whole first warp loads positions; 1 slot)."""
    w = W.WORKLOADS["prefill"].scaled(T=T, H=H, k=k)
    x, idx, tw = W.make_routing(w)
    idx = idx.clone()
    idx[::4, min(2, k - 1)] = -1
    idx[9, :] = -1
    for C in (0, 96 if k > 1 else 8):
        res = ep.ep_layout(idx.to(DEV), w.E, w.R, 1, C)
        st, L = oracle.layout(idx.numpy(), w.E, w.R, 1, C)
        assert st == 0
        h = res.handle
        rows = h.num_recv_rows
        valid = L.src_idx >= 0
        xd = x.to(DEV)
        recv, sc, _ = ep.ep_dispatch_ex(h, xd, True, num_sms=num_sms)
        xq, xs = oracle.quantize_rows(x)
        rq, sq, _ = ep.ep_dispatch_ex(h, torch.from_numpy(xq).to(DEV).view(torch.float8_e4m3fn), True,
                                      x_scales=torch.from_numpy(xs).to(DEV), num_sms=num_sms)
        rb, _, _ = ep.ep_dispatch_ex(h, xd, False, num_sms=num_sms)
        y = W.make_expert_out(rows, w.H, seed=7).to(DEV)
        out = ep.ep_combine_ex(h, y, tw.to(DEV), num_sms=num_sms)
        torch.cuda.synchronize()
        q, s = oracle.dispatch_fp8(x, L.pos, L.n_rows)
        assert (u8(recv)[valid] == q[valid]).all(), C
        assert (sc.cpu().numpy()[valid].view(np.uint32) == s[valid].view(np.uint32)).all(), C
        q2, s2 = oracle.dispatch_fp8_prequant(xq, xs, L.pos, L.n_rows)
        assert (u8(rq)[valid] == q2[valid]).all(), C
        assert (sq.cpu().numpy()[valid].view(np.uint32) == s2[valid].view(np.uint32)).all(), C
        b = oracle.dispatch_bf16(x, L.pos, L.n_rows)
        assert (u16(rb)[valid] == b[valid]).all(), C
        assert (u16(out) == oracle.combine(y.cpu(), tw.numpy(), L.pos)).all(), C
        h.free()


def test_option_errors():
    w, x, tw, res, L = setup("prefill", 64)
    h = res.handle
    xq, xs = oracle.quantize_rows(x)
    xq_d = torch.from_numpy(xq).to(DEV).view(torch.float8_e4m3fn)
    with pytest.raises(ValueError):
        ep.ep_dispatch_ex(h, xq_d, False, x_scales=torch.from_numpy(xs).to(DEV))
    L_ = ep.lib()
    import ctypes
    rows = h.num_recv_rows
    recv = torch.empty(rows, w.H, dtype=torch.float8_e4m3fn, device=DEV)
    sc = torch.empty(rows * (w.H // 128), dtype=torch.float32, device=DEV)
    P = ctypes.c_void_p
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    G = w.H // 128
    # overlapping scale strides (row stride smaller than the groups of a row)
    st = L_.ep_dispatch_ex(h.ptr, P(x.to(DEV).data_ptr()), None, w.H, 0, 1, P(recv.data_ptr()),
                           P(sc.data_ptr()), G - 1, 1, None, rows, 0, stream)
    assert st == ep.EP_ERR_INVALID_ARG
    # e4m3 input without scales
    st = L_.ep_dispatch_ex(h.ptr, P(xq_d.data_ptr()), None, w.H, 1, 1, P(recv.data_ptr()),
                           P(sc.data_ptr()), G, 1, None, rows, 0, stream)
    assert st == ep.EP_ERR_INVALID_ARG
    # negative SM budget
    st = L_.ep_dispatch_ex(h.ptr, P(x.to(DEV).data_ptr()), None, w.H, 0, 1, P(recv.data_ptr()),
                           P(sc.data_ptr()), G, 1, None, rows, -1, stream)
    assert st == ep.EP_ERR_INVALID_ARG


@pytest.mark.parametrize("prequant,num_sms,padded", [(False, 0, False), (True, 0, False), (False, 16, False),
                                                      (False, 0, True)])
def test_column_major_scales_large_batch(prequant, num_sms, padded):
    """Column-major scales on a batch of over 2^20 scale stores, fused or
    pre-quantised, with an SM budget and in padded mode: bit-exact against
    the oracle, with tokens whose first slots are unused, a token with no
    slot, padding rows and the leading dimension's slack untouched."""
    w = W.WORKLOADS["prefill"].scaled(T=2400)
    x, idx, _ = W.make_routing(w)
    idx = idx.clone()
    idx[::3, 0] = -1
    idx[5, :] = -1
    idx[7, :2] = -1
    C = 128 if padded else 0
    G = w.H // 128
    assert idx.shape[0] * w.k * G >= 1 << 20
    res = ep.ep_layout(idx.to(DEV), w.E, w.R, 1, C)
    st, L = oracle.layout(idx.numpy(), w.E, w.R, 1, C)
    assert st == 0
    rows = res.handle.num_recv_rows
    ld = (rows + 3) // 4 * 4 + 4
    if prequant:
        xq, xs = oracle.quantize_rows(x)
        xin = torch.from_numpy(xq).to(DEV).view(torch.float8_e4m3fn)
        xsd = torch.from_numpy(xs).to(DEV)
    else:
        xin, xsd = x.to(DEV), None
    sc = torch.full((G, ld), -3.0, dtype=torch.float32, device=DEV)
    recv, sc, _ = ep.ep_dispatch_ex(res.handle, xin, True, x_scales=xsd, recv_scales=sc, scale_layout="col",
                                    num_sms=num_sms)
    torch.cuda.synchronize()
    q, s = oracle.dispatch_fp8(x, L.pos, L.n_rows)
    valid = L.src_idx >= 0
    got = sc.cpu().numpy()
    assert (got[:, :rows].T[valid].view(np.uint32) == s[valid].view(np.uint32)).all()
    assert (got[:, :rows].T[~valid] == -3.0).all() and (got[:, rows:] == -3.0).all()
    assert (u8(recv)[valid] == q[valid]).all()
    assert res.handle.check() == ep.EP_OK


def test_binding_refuses_buffers_the_call_would_overrun():
    """The library cannot see a buffer's size; the binding checks every
    buffer indexed by receive row before anything is launched."""
    w, x, tw, res, L = setup("prefill", 64)
    h = res.handle
    rows, G = h.num_recv_rows, w.H // 128
    xd = x.to(DEV)
    with pytest.raises(ValueError, match="recv_scales"):
        ep.ep_dispatch(h, xd, True, recv_scales=torch.empty(rows - 1, G, device=DEV))
    with pytest.raises(ValueError, match="recv_src_idx"):
        ep.ep_dispatch(h, xd, False, recv_src_idx=torch.empty(rows - 1, dtype=torch.int32, device=DEV))
    with pytest.raises(ValueError, match="recv_scales"):
        ep.ep_dispatch_ex(h, xd, True, scale_layout="col", recv_scales=torch.empty(G, rows - 1, device=DEV))
    with pytest.raises(ValueError, match="recv_scales"):
        ep.ep_dispatch_ex(h, xd, True, scale_layout="col", scale_ld=rows + 8,
                          recv_scales=torch.empty(G, rows + 4, device=DEV))
    with pytest.raises(ValueError, match="recv_src_idx"):
        ep.ep_dispatch_ex(h, xd, False, recv_src_idx=torch.empty(rows - 1, dtype=torch.int32, device=DEV))
    with pytest.raises(ValueError, match="bf16 or float8_e4m3fn"):
        ep.ep_dispatch_ex(h, xd.float(), True)
    go = x.to(DEV)
    with pytest.raises(ValueError, match="y must be"):
        ep.ep_combine_backward(h, go, tw.to(DEV), y=torch.empty(rows - 1, w.H, dtype=torch.bfloat16, device=DEV))
    with pytest.raises(ValueError, match="grad_y must be"):
        ep.ep_combine_backward(h, go, tw.to(DEV), want_grad_weights=False,
                               grad_y=torch.empty(rows - 1, w.H, dtype=torch.bfloat16, device=DEV))
    with pytest.raises(ValueError, match="need y"):
        ep.ep_combine_backward(h, go, tw.to(DEV))
    # a column-major buffer wider than the rows, with its width as the leading dimension, is accepted
    sc = torch.full((G, rows + 12), -1.0, device=DEV)
    _, got, _ = ep.ep_dispatch_ex(h, xd, True, scale_layout="col", recv_scales=sc)
    torch.cuda.synchronize()
    _, s = oracle.dispatch_fp8(x, L.pos, L.n_rows)
    valid = L.src_idx >= 0
    assert (got.cpu().numpy()[:, :rows].T[valid].view(np.uint32) == s[valid].view(np.uint32)).all()
    assert h.check() == ep.EP_OK


@pytest.mark.parametrize("T,num_sms,padded,ld_pad", [(2400, 0, False, 0), (2400, 16, False, 4), (2400, 0, True, 8),
                                                     (257, 0, False, 0), (1, 0, False, 4)])
def test_column_major_scales_through_the_token_table(T, num_sms, padded, ld_pad):
    """ep_dispatch_fp8_colmajor (per-token scale table, then the column
    fill): codes, column-major scales and the token table bit-exact against
    the oracle, with unused first slots, a token with no slot, padding rows
    and the leading dimension's slack untouched, under an SM budget and in
    padded mode; a ragged last tile of rows (rows not a multiple of 128)."""
    w = W.WORKLOADS["prefill"].scaled(T=T)
    x, idx, _ = W.make_routing(w)
    idx = idx.clone()
    if T > 8:
        idx[::3, 0] = -1
        idx[5, :] = -1
        idx[7, :2] = -1
    C = 128 if padded else 0
    G = w.H // 128
    res = ep.ep_layout(idx.to(DEV), w.E, w.R, 1, C)
    st, L = oracle.layout(idx.numpy(), w.E, w.R, 1, C)
    assert st == 0
    rows = res.handle.num_recv_rows
    ld = (rows + 3) // 4 * 4 + ld_pad
    sc = torch.full((G, ld), -3.0, dtype=torch.float32, device=DEV)
    recv = torch.full((rows, w.H), 0x5A, dtype=torch.uint8, device=DEV).view(torch.float8_e4m3fn)
    tok = torch.full((T, G), -5.0, dtype=torch.float32, device=DEV)
    src = torch.empty(rows, dtype=torch.int32, device=DEV)
    ep.ep_dispatch_fp8_colmajor(res.handle, x.to(DEV), recv_x=recv, recv_scales=sc, token_scales=tok,
                                recv_src_idx=src, num_sms=num_sms)
    torch.cuda.synchronize()
    q, s = oracle.dispatch_fp8(x, L.pos, L.n_rows)
    _, ts = oracle.quantize_rows(x)
    valid = L.src_idx >= 0
    got = sc.cpu().numpy()
    assert (got[:, :rows].T[valid].view(np.uint32) == s[valid].view(np.uint32)).all()
    assert (got[:, :rows].T[~valid] == -3.0).all() and (got[:, rows:] == -3.0).all()
    assert (u8(recv)[valid] == q[valid]).all() and (u8(recv)[~valid] == 0x5A).all()
    assert (tok.cpu().numpy().view(np.uint32) == ts.view(np.uint32)).all()
    assert (src.cpu().numpy() == L.src_idx).all()
    assert res.handle.check() == ep.EP_OK


@pytest.mark.parametrize("H,align,num_sms", [(7168, 1, 0), (640, 1, 0), (8192 + 128, 1, 0), (7168, 4, 0),
                                              (1024, 1, 7)])
def test_column_major_scales_repeated_calls(H, align, num_sms):
    """Several ep_dispatch_fp8_colmajor calls on one handle with new x each
    time (the decode pattern), the table and scale buffers reused: every
    call bit-exact, for 56 groups (16-byte table pieces), 5 groups (scalar
    pieces), two chunks per token, an alignment and an SM budget."""
    w = W.WORKLOADS["prefill"].scaled(T=777, H=H)
    _, idx, _ = W.make_routing(w)
    idx = idx.clone()
    idx[::5, 1] = -1
    res = ep.ep_layout(idx.to(DEV), w.E, w.R, align, 0)
    st, L = oracle.layout(idx.numpy(), w.E, w.R, align, 0)
    assert st == 0
    rows, G = res.handle.num_recv_rows, H // 128
    valid = L.src_idx >= 0
    sc = torch.full((G, rows + 4), -3.0, device=DEV)
    tok = torch.empty(w.T, G, device=DEV)
    for step in range(3):
        x = W.make_x(w, 50 + step)
        recv, sc, tok, _ = ep.ep_dispatch_fp8_colmajor(res.handle, x.to(DEV), recv_scales=sc, token_scales=tok,
                                                       num_sms=num_sms)
        torch.cuda.synchronize()
        q, s = oracle.dispatch_fp8(x, L.pos, L.n_rows)
        got = sc.cpu().numpy()
        assert (got[:, :rows].T[valid].view(np.uint32) == s[valid].view(np.uint32)).all(), step
        assert (got[:, :rows].T[~valid] == -3.0).all() and (got[:, rows:] == -3.0).all(), step
        assert (u8(recv)[valid] == q[valid]).all(), step
    assert res.handle.check() == ep.EP_OK


def test_column_major_scales_through_the_token_table_full_size():
    """The metric workload (group-limited gating, T=8192, H=7168, E=256,
    R=64) at full size: every receive row's codes and every column-major
    scale against the oracle; equal to ep_dispatch_ex's scattered form."""
    w = W.WORKLOADS["group_limited"]
    x, idx, _ = W.make_routing(w)
    res = ep.ep_layout(idx.to(DEV), w.E, w.R)
    _, L = oracle.layout(idx.numpy(), w.E, w.R)
    rows, G = res.handle.num_recv_rows, w.H // 128
    xd = x.to(DEV)
    recv, sc, tok, _ = ep.ep_dispatch_fp8_colmajor(res.handle, xd)
    _, sc2, _ = ep.ep_dispatch_ex(res.handle, xd, True, scale_layout="col")
    torch.cuda.synchronize()
    assert torch.equal(sc[:, :rows], sc2[:, :rows])
    q, s = oracle.dispatch_fp8(x, L.pos, L.n_rows)
    assert (sc[:, :rows].cpu().numpy().T.view(np.uint32) == s.view(np.uint32)).all()
    got = recv.view(torch.uint8)
    for r0 in range(0, rows, 8192):
        assert (got[r0:r0 + 8192].cpu().numpy() == q[r0:r0 + 8192]).all(), r0
    _, ts = oracle.quantize_rows(x)
    assert (tok.cpu().numpy().view(np.uint32) == ts.view(np.uint32)).all()


def test_column_major_token_table_argument_errors():
    w, x, tw, res, L = setup("prefill", 64)
    h = res.handle
    rows, G = h.num_recv_rows, w.H // 128
    xd = x.to(DEV)
    with pytest.raises(ValueError, match="recv_scales"):
        ep.ep_dispatch_fp8_colmajor(h, xd, recv_scales=torch.empty(G, rows - 1, device=DEV))
    with pytest.raises(ValueError, match="token_scales"):
        ep.ep_dispatch_fp8_colmajor(h, xd, token_scales=torch.empty(w.T - 1, G, device=DEV))
    with pytest.raises(ValueError, match="H % 128"):
        ep.ep_dispatch_fp8_colmajor(h, torch.zeros(w.T, 136, dtype=torch.bfloat16, device=DEV))
    import ctypes
    P = ctypes.c_void_p
    recv = torch.empty(rows, w.H, dtype=torch.float8_e4m3fn, device=DEV)
    sc = torch.empty(G, rows, device=DEV)
    stream = P(torch.cuda.current_stream().cuda_stream)
    # no token table
    st = ep.lib().ep_dispatch_fp8_colmajor(h.ptr, P(xd.data_ptr()), w.H, P(recv.data_ptr()), P(sc.data_ptr()),
                                           rows, None, None, rows, 0, stream)
    assert st == ep.EP_ERR_INVALID_ARG
    # fewer rows than the layout may use
    tok = torch.empty(w.T, G, device=DEV)
    st = ep.lib().ep_dispatch_fp8_colmajor(h.ptr, P(xd.data_ptr()), w.H, P(recv.data_ptr()), P(sc.data_ptr()),
                                           rows - 1, P(tok.data_ptr()), None, rows - 1, 0, stream)
    assert st == ep.EP_ERR_INVALID_ARG


def test_column_major_prequantised_through_the_fill():
    """Pre-quantised input with column-major scales takes the fill pass with
    the input's own scale table: bit-exact, padding rows untouched."""
    w = W.WORKLOADS["decode"]
    x, idx, _ = W.make_routing(w)
    res = ep.ep_layout(idx.to(DEV), w.E, w.R, w.align, w.capacity)
    _, L = oracle.layout(idx.numpy(), w.E, w.R, w.align, w.capacity)
    rows, G = res.handle.num_recv_rows, w.H // 128
    xq, xs = oracle.quantize_rows(x)
    sc = torch.full((G, rows + 4), -3.0, device=DEV)
    recv, sc, _ = ep.ep_dispatch_ex(res.handle, torch.from_numpy(xq).to(DEV).view(torch.float8_e4m3fn), True,
                                    x_scales=torch.from_numpy(xs).to(DEV), recv_scales=sc, scale_layout="col")
    torch.cuda.synchronize()
    q, s = oracle.dispatch_fp8_prequant(xq, xs, L.pos, L.n_rows)
    valid = L.src_idx >= 0
    got = sc.cpu().numpy()
    assert (got[:, :rows].T[valid].view(np.uint32) == s[valid].view(np.uint32)).all()
    assert (got[:, :rows].T[~valid] == -3.0).all() and (got[:, rows:] == -3.0).all()
    assert (u8(recv)[valid] == q[valid]).all()



@pytest.mark.parametrize("prequant", [False, True])
def test_column_major_back_to_back_calls_and_graph_replays(prequant):
    """Column-major scales through the fill pass, four calls enqueued back to
    back on one handle (new x each, one shared token table for the quantising
    call, no synchronisation in between) and three replays of a captured call
    (new x copied in before each, results copied out after each, one
    synchronisation at the end): each bit-exact.  With pre-quantised input the
    fill pass starts before the copy kernel completes (its table is the
    input), so this also checks that it never runs ahead of what it needs."""
    w = W.WORKLOADS["prefill"].scaled(T=1500)
    _, idx, _ = W.make_routing(w)
    res = ep.ep_layout(idx.to(DEV), w.E, w.R)
    st, L = oracle.layout(idx.numpy(), w.E, w.R)
    assert st == 0
    h = res.handle
    rows, G = h.num_recv_rows, w.H // 128
    valid = L.src_idx >= 0
    xs = [W.make_x(w, 90 + i) for i in range(4)]
    if prequant:
        qs = [oracle.quantize_rows(x) for x in xs]
        ins = [(torch.from_numpy(xq).to(DEV).view(torch.float8_e4m3fn), torch.from_numpy(xsc).to(DEV))
               for xq, xsc in qs]
    else:
        ins = [(x.to(DEV), None) for x in xs]
    tok = torch.empty(w.T, G, device=DEV)

    def call(xin, sin, recv=None, sc=None):
        if prequant:
            return ep.ep_dispatch_ex(h, xin, True, x_scales=sin, recv_x=recv, recv_scales=sc, scale_layout="col")[:2]
        return ep.ep_dispatch_fp8_colmajor(h, xin, recv_x=recv, recv_scales=sc, token_scales=tok)[:2]

    def check(i, recv, sc, what):
        if prequant:
            q, s = oracle.dispatch_fp8_prequant(qs[i][0], qs[i][1], L.pos, L.n_rows)
        else:
            q, s = oracle.dispatch_fp8(xs[i], L.pos, L.n_rows)
        assert (sc.cpu().numpy()[:, :rows].T[valid].view(np.uint32) == s[valid].view(np.uint32)).all(), what
        assert (u8(recv)[valid] == q[valid]).all(), what

    torch.cuda.synchronize()
    outs = [call(xin, sin) for xin, sin in ins]
    torch.cuda.synchronize()
    for i, (recv, sc) in enumerate(outs):
        check(i, recv, sc, ("back to back", i))

    xin = torch.empty_like(ins[0][0])
    sin = torch.empty_like(ins[0][1]) if prequant else None
    recv = torch.empty(rows, w.H, dtype=torch.float8_e4m3fn, device=DEV)
    sc = torch.empty(G, (rows + 3) // 4 * 4, device=DEV)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        call(xin, sin, recv, sc)
    torch.cuda.current_stream().wait_stream(stream)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        call(xin, sin, recv, sc)
    snaps = []
    for xi, si in ins[:3]:
        xin.copy_(xi)
        if prequant:
            sin.copy_(si)
        graph.replay()
        snaps.append((recv.clone(), sc.clone()))
    torch.cuda.synchronize()
    for i, (r, s) in enumerate(snaps):
        check(i, r, s, ("replay", i))
    assert h.check() == ep.EP_OK
    del graph
