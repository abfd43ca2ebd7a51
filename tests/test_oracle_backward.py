"""Pins for the oracle's backward pair (CPU only).

The pages state that the backward of dispatch is a combine and the backward
of combine is a dispatch.  The oracle's gradients are checked against
  * torch autograd in float64 of the forward definitions (a library routine),
  * exact rational arithmetic for the rounding steps of grad_y,
  * exact small-integer cases, unused slots, and the k = 1 special case.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

from combine_ep_layout_10_b200 import workloads as W
from exact import bf16_bits, to_bf16, to_f32


def bf16_of(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16)


def u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def autograd_combine(y64, w64, pos, g64):
    """float64 autograd of out[t] = sum_j w[t,j] * y[pos[t,j]] with loss <g, out>."""
    y64 = y64.clone().requires_grad_(True)
    w64 = w64.clone().requires_grad_(True)
    T, k = pos.shape
    out = torch.zeros(T, y64.shape[1], dtype=torch.float64)
    for j in range(k):
        valid = pos[:, j] >= 0
        rows = torch.where(valid, pos[:, j], torch.zeros_like(pos[:, j])).long()
        out = out + torch.where(valid[:, None], w64[:, j:j + 1] * y64[rows], torch.zeros_like(out))
    (out * g64).sum().backward()
    return y64.grad, w64.grad


@pytest.mark.parametrize("name", ["tiny", "prefill"])
def test_combine_backward_vs_autograd(orc, name):
    w = W.WORKLOADS[name].scaled(T=40, H=256)
    _, idx, tw = W.make_routing(w)
    idx[3, 1] = -1  # an unused slot
    _, L = orc.layout(idx.numpy(), w.E, w.R)
    g = torch.Generator().manual_seed(2)
    y = torch.randn(L.n_rows, w.H, generator=g).to(torch.bfloat16)
    go = torch.randn(w.T, w.H, generator=g).to(torch.bfloat16)
    grad_y, grad_w = orc.combine_backward(go, y, tw.numpy(), L.pos)
    pos = torch.from_numpy(L.pos)
    gy64, gw64 = autograd_combine(y.double(), tw.double(), pos, go.double())
    # grad_w: float64 sums of exact products, any order -> ~1e-12 relative
    scale = (go.double().abs() @ y.double().abs().T).max().item()
    assert np.allclose(grad_w, gw64.numpy(), rtol=0, atol=1e-12 * scale)
    assert grad_w[3, 1] == 0.0
    # grad_y: each written row is w * g rounded to fp32 then to bf16; autograd's
    # float64 value differs from it by at most those two roundings
    written = L.src_idx >= 0
    ref = gy64.numpy()[written]
    got = orc.bits_to_f32(grad_y[written]).astype(np.float64)
    assert (np.abs(got - ref) <= np.abs(ref) * (2.0 ** -8 + 2.0 ** -23) + 1e-300).all()
    assert (grad_y[~written] == 0).all()


def test_combine_backward_rounding_is_fp32_then_bf16(orc):
    # w * g = 0.70507814..., fp32-rounded it is a bf16 tie that goes to the even
    # 0.703125; rounding the exact product to bf16 directly would give 0.70703125.
    w = np.array([[0.5277777910232544]], np.float32)
    go = bf16_of([[1.3359375]])
    y = bf16_of([[0.0]])
    grad_y, _ = orc.combine_backward(go, y, w, np.array([[0]], np.int32))
    exact = Fraction(float(w[0, 0])) * Fraction(1.3359375)
    assert orc.bf16_to_f32(int(grad_y[0, 0])) == to_bf16(Fraction(to_f32(exact))) == 0.703125
    assert to_bf16(exact) == 0.70703125


def test_combine_backward_exact_rationals(orc):
    rng = np.random.default_rng(9)
    T, k, H, n = 5, 3, 12, 20
    go = (torch.from_numpy(rng.standard_normal((T, H))) * 4).to(torch.bfloat16)
    y = (torch.from_numpy(rng.standard_normal((n, H))) * 2).to(torch.bfloat16)
    w = rng.random((T, k)).astype(np.float32)
    pos = np.ascontiguousarray(rng.permutation(n)[:T * k].reshape(T, k).astype(np.int32))  # injective, like a layout
    grad_y, grad_w = orc.combine_backward(go, y, w, pos)
    gf, yf = go.float().numpy(), y.float().numpy()
    for t in range(T):
        for j in range(k):
            p = pos[t, j]
            want_dot = sum(Fraction(float(gf[t, i])) * Fraction(float(yf[p, i])) for i in range(H))
            assert abs(Fraction(grad_w[t, j]) - want_dot) <= Fraction(1, 10 ** 12) * (1 + abs(want_dot))
            for i in range(H):
                v = to_bf16(Fraction(to_f32(Fraction(float(w[t, j])) * Fraction(float(gf[t, i])))))
                assert grad_y[p, i] == (bf16_bits(v) if v != 0 else grad_y[p, i] & 0x8000)


def test_dispatch_backward_vs_autograd(orc):
    w = W.WORKLOADS["tiny"]
    _, idx, _ = W.make_routing(w)
    _, L = orc.layout(idx.numpy(), w.E, w.R)
    # small integers: every fp32 partial sum is exact, so the bf16 result is too
    rng = np.random.default_rng(4)
    gr = rng.integers(-8, 9, size=(L.n_rows, w.H)).astype(np.float32)
    got = orc.dispatch_backward(bf16_of(gr.tolist()), L.pos)
    x64 = torch.zeros(w.T, w.H, dtype=torch.float64, requires_grad=True)
    src = torch.from_numpy(L.src_idx.astype(np.int64))
    recv = x64[src]
    (recv * torch.from_numpy(gr).double()).sum().backward()
    want = x64.grad.numpy()
    assert (orc.bits_to_f32(got).astype(np.float64) == want).all()


def test_dispatch_backward_k1_is_inverse_permutation(orc):
    w = W.WORKLOADS["tiny"].scaled(k=1)
    x, idx, _ = W.make_routing(w)
    _, L = orc.layout(idx.numpy(), w.E, w.R)
    recv = orc.dispatch_bf16(x, L.pos, L.n_rows)
    assert (orc.dispatch_backward(recv, L.pos) == u16(x)).all()
