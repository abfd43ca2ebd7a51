"""Parity of the backward pair (through the C ABI) with the CPU oracle.

Bars: dispatch backward and grad_y bit-exact (same roundings as the oracle);
grad_weights (an fp32 dot product whose summation order the pages leave
open) within the bound that follows from its fixed reduction order:
|gpu - exact| <= (16 * ceil(H / 2048) + 37) * 2^-24 * sum_i |g_i * y_i|, the
oracle's binary64 value standing in for the exact one.
"""
import math

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


def u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def grad_w_bound(go, y, pos, H):
    g = go.double().numpy()
    yy = y.double().numpy()
    T, k = pos.shape
    s = np.zeros((T, k))
    for j in range(k):
        valid = pos[:, j] >= 0
        rows = np.where(valid, pos[:, j], 0)
        s[:, j] = np.where(valid, np.abs(g * yy[rows]).sum(1), 0.0)
    return (16 * math.ceil(H / 2048) + 37) * 2.0 ** -24 * s + 1e-30


def setup(name, T=None, H=None, k=None, unused=False):
    w = W.WORKLOADS[name]
    kw = {}
    if T:
        kw["T"] = T
    if H:
        kw["H"] = H
    if k:
        kw["k"] = k
    w = w.scaled(**kw) if kw else w
    _, idx, tw = W.make_routing(w)
    if unused:
        idx[::7, -1] = -1
    res = ep.ep_layout(idx.to(DEV), w.E, w.R, w.align, w.capacity)
    _, L = oracle.layout(idx.numpy(), w.E, w.R, w.align, w.capacity)
    return w, idx, tw, res, L


@pytest.mark.parametrize("name,T,H", [("tiny", None, None), ("prefill", 512, None), ("decode", None, None),
                                      ("large_skewed", 1024, None), ("tiny", None, 1000)])
def test_dispatch_backward(name, T, H):
    w, idx, tw, res, L = setup(name, T, H, unused=True)
    g = W.make_expert_out(L.n_rows, w.H, seed=31)
    gx = ep.ep_dispatch_backward(res.handle, g.to(DEV))
    torch.cuda.synchronize()
    assert (u16(gx) == oracle.dispatch_backward(g, L.pos)).all()


@pytest.mark.parametrize("name,T,H,k", [("tiny", None, None, None), ("prefill", 256, None, None),
                                        ("group_limited", 256, None, None), ("decode", None, None, None),
                                        ("tiny", None, 1000, None), ("tiny", 64, 24, 16),
                                        ("prefill", 64, 17408, 32)])
def test_combine_backward(name, T, H, k):
    w, idx, tw, res, L = setup(name, T, H, k, unused=True)
    y = W.make_expert_out(L.n_rows, w.H, seed=41)
    go = W.make_x(w, 42)
    gy0 = torch.full((L.n_rows, w.H), 7.0, dtype=torch.bfloat16, device=DEV)  # sentinel rows
    gy, gw = ep.ep_combine_backward(res.handle, go.to(DEV), tw.to(DEV), y=y.to(DEV), grad_y=gy0)
    torch.cuda.synchronize()
    want_gy, want_gw = oracle.combine_backward(go, y, tw.numpy(), L.pos)
    written = L.src_idx >= 0
    got = u16(gy)
    assert (got[written] == want_gy[written]).all()
    assert (got[~written] == 0x40E0).all(), "rows no slot maps to must be left untouched"
    gwn = gw.cpu().numpy().astype(np.float64)
    assert (np.abs(gwn - want_gw) <= grad_w_bound(go, y, L.pos, w.H)).all()
    assert (gwn[L.pos < 0] == 0).all()
    # grad_weights omitted: the same grad_y, y not needed
    gy2, gw2 = ep.ep_combine_backward(res.handle, go.to(DEV), tw.to(DEV), want_grad_weights=False)
    torch.cuda.synchronize()
    assert gw2 is None and (u16(gy2)[written] == want_gy[written]).all()
    # deterministic
    _, gw3 = ep.ep_combine_backward(res.handle, go.to(DEV), tw.to(DEV), y=y.to(DEV))
    assert torch.equal(gw.cpu(), gw3.cpu())


def test_backward_full_size_sampled():
    w, idx, tw, res, L = setup("group_limited")
    y = W.make_expert_out(L.n_rows, w.H, seed=51)
    go = W.make_x(w, 52)
    gy, gw = ep.ep_combine_backward(res.handle, go.to(DEV), tw.to(DEV), y=y.to(DEV))
    grecv = W.make_expert_out(L.n_rows, w.H, seed=53)
    gx = ep.ep_dispatch_backward(res.handle, grecv.to(DEV))
    torch.cuda.synchronize()
    sample = torch.randperm(w.T, generator=torch.Generator().manual_seed(8))[:64].tolist() + [0, w.T - 1]
    for t in sample:
        rows = torch.from_numpy(L.pos[t].astype(np.int64))
        pos1 = np.arange(w.k, dtype=np.int32)[None, :]
        want_gy, want_gw = oracle.combine_backward(go[t:t + 1], y[rows], tw[t:t + 1].numpy(), pos1)
        assert (u16(gy[rows.to(DEV)]) == want_gy).all()
        bound = grad_w_bound(go[t:t + 1], y[rows], pos1, w.H)
        assert (np.abs(gw[t].cpu().numpy().astype(np.float64) - want_gw[0]) <= bound[0]).all()
        want_gx = oracle.dispatch_backward(grecv[rows], pos1)
        assert (u16(gx[t:t + 1]) == want_gx).all()
