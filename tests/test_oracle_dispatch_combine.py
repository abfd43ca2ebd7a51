"""Pins for the oracle's dispatch (BF16 and fused FP8) and combine (CPU only).

Independent checks:
  * hand-derived FP8 group (tests/golden/fp8_group_small.json);
  * the scale and codes recomputed with exact rational arithmetic
    (tests/exact.py) and torch's e4m3 conversion;
  * the combine's fp32 fused-multiply-add chain replayed with exact
    rationals and correct rounding after every step, in slot order;
  * closed forms: small-integer combines are exact; combine(dispatch(x)) with
    identity experts and weights summing to one returns x exactly under BF16
    and within the e4m3 error bound under FP8; k = 1 with weight 1 is the
    inverse permutation.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from combine_ep_layout_10_b200 import workloads as W
from exact import bf16_bits, f32_bits, to_bf16, to_f32

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_of(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16)


def u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# --- FP8 quantisation --------------------------------------------------------

def test_golden_fp8_group(orc):
    d = json.load(open(os.path.join(GOLDEN, "fp8_group_small.json")))
    x = torch.zeros(128)
    for i, v in d["x_nonzero"].items():
        x[int(i)] = v
    q, s = orc.quantize_group(x.to(torch.bfloat16))
    assert f32_bits(s) == int(d["scale_bits"], 16)
    want = np.zeros(128, np.uint8)
    for i, c in d["codes_nonzero"].items():
        want[int(i)] = c
    assert (q == want).all(), (q[:8], want[:8])
    q0, s0 = orc.quantize_group(torch.zeros(128, dtype=torch.bfloat16))
    assert s0 == 0.0 and (q0 == 0).all()
    # an all-negative-zero group is still the all-zero case
    q1, s1 = orc.quantize_group(torch.full((128,), -0.0).to(torch.bfloat16))
    assert s1 == 0.0 and (q1 == 0).all()


def exact_quantize(xg: torch.Tensor):
    """Scale and codes from exact rationals + torch's RNE e4m3 conversion."""
    xs = [Fraction(v) for v in xg.to(torch.float32).tolist()]
    amax = max(abs(v) for v in xs)
    if amax == 0:
        return [0] * 128, 0.0
    scale = to_f32(amax / 448)
    inv = Fraction(to_f32(Fraction(448) / amax))
    # IEEE product sign: a zero product keeps the sign of x (inv > 0); Fractions drop it.
    xf = xg.to(torch.float32).tolist()
    prod = torch.tensor([to_f32(v * inv) if v != 0 else xf[i] for i, v in enumerate(xs)],
                        dtype=torch.float32)
    codes = prod.to(torch.float8_e4m3fn).view(torch.uint8).tolist()
    return codes, scale


@pytest.mark.parametrize("mag", [1.0, 1e-3, 3e-6, 200.0, 6e4])
def test_quantize_vs_exact(orc, mag):
    g = torch.Generator().manual_seed(int(mag * 1000) % 997)
    for _ in range(8):
        xg = (torch.randn(128, generator=g) * mag)
        xg[torch.randint(0, 128, (4,), generator=g)] = -0.0
        xg = xg.to(torch.bfloat16)
        q, s = orc.quantize_group(xg)
        codes, scale = exact_quantize(xg)
        assert f32_bits(s) == f32_bits(scale)
        assert q.tolist() == codes


def test_quantize_error_bound(orc):
    """|decode(q)*s - x| <= 2^-4 |x| + 2^-10 * s * 448 / 448 ... i.e. half an e4m3 ulp."""
    g = torch.Generator().manual_seed(5)
    for _ in range(50):
        xg = (torch.randn(128, generator=g) * float(torch.rand(1, generator=g) * 10 + 1e-3)).to(torch.bfloat16)
        q, s = orc.quantize_group(xg)
        deq = np.array([orc.e4m3_decode(c) for c in q], np.float64) * s
        x = xg.to(torch.float64).numpy()
        # relative half-ulp 2^-4 for normals, absolute half-step 2^-10 * scale for subnormals,
        # plus the two fp32 roundings of the scale path
        assert (np.abs(deq - x) <= 2.0 ** -4 * np.abs(x) + 2.0 ** -10 * s + 1e-6 * np.abs(x)).all()


# --- dispatch ----------------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny", "prefill", "decode"])
def test_dispatch_bf16_is_gather_of_src(orc, name):
    w = W.WORKLOADS[name].scaled(T=min(W.WORKLOADS[name].T, 256))
    x, idx, _ = W.make_routing(w)
    _, L = orc.layout(idx.numpy(), w.E, w.R, capacity=w.capacity)
    recv = orc.dispatch_bf16(x, L.pos, L.n_rows)
    xs = u16(x)
    rows = np.nonzero(L.src_idx >= 0)[0]
    assert (recv[rows] == xs[L.src_idx[rows]]).all()
    pad = np.nonzero(L.src_idx < 0)[0]
    assert (recv[pad] == 0).all()


@pytest.mark.parametrize("name", ["prefill", "group_limited", "decode"])
def test_dispatch_fp8_rows(orc, name):
    w = W.WORKLOADS[name].scaled(T=48)
    x, idx, _ = W.make_routing(w)
    _, L = orc.layout(idx.numpy(), w.E, w.R, capacity=w.capacity)
    recv, scales = orc.dispatch_fp8(x, L.pos, L.n_rows)
    G = w.H // 128
    for t in range(w.T):
        qs, ss = zip(*[orc.quantize_group(x[t, g * 128:(g + 1) * 128]) for g in range(G)])
        q = np.concatenate(qs)
        for j in range(w.k):
            p = L.pos[t, j]
            assert (recv[p] == q).all()
            assert (scales[p] == np.array(ss, np.float32)).all()
    # spot-check one token fully against the exact recomputation
    codes, scale = exact_quantize(x[3, :128])
    assert recv[L.pos[3, 0], :128].tolist() == codes
    assert f32_bits(scales[L.pos[3, 0], 0]) == f32_bits(scale)


# --- combine -----------------------------------------------------------------

def exact_combine_elem(ws, ys):
    """fp32 fma chain: acc <- round32(w*y + acc) in slot order, then round to bf16."""
    acc = Fraction(0)
    for wv, yv in zip(ws, ys):
        acc = Fraction(to_f32(Fraction(wv) * Fraction(yv) + acc))
    return bf16_bits(to_bf16(acc)) if acc != 0 else 0


def test_combine_fma_chain_exact(orc):
    g = torch.Generator().manual_seed(11)
    T, k, H, n = 6, 5, 24, 40
    y = (torch.randn(n, H, generator=g) * 3).to(torch.bfloat16)
    w = torch.rand(T, k, generator=g) * 2 - 0.5
    pos = torch.randint(0, n, (T, k), generator=g).to(torch.int32)
    pos[1, 2] = -1
    pos[4, :] = -1
    out = orc.combine(y, w.numpy(), pos.numpy())
    yf = y.to(torch.float32)
    for t in range(T):
        for i in range(H):
            sl = [j for j in range(k) if pos[t, j] >= 0]
            want = exact_combine_elem([w[t, j].item() for j in sl],
                                      [yf[pos[t, j], i].item() for j in sl])
            assert out[t, i] == want, (t, i)


def test_combine_order_matters_and_is_slot_order(orc):
    """A case where summing in another order, or without fusing, gives another
    bf16: the oracle must follow the slot-order fma chain exactly."""
    y = bf16_of([[1.0], [2.0 ** -9], [-1.0], [2.0 ** -9]])
    w = np.array([[1.0, 1.0, 1.0, 1.0]], np.float32)
    pos = np.array([[0, 1, 2, 3]], np.int32)
    # slot order: 1 + 2^-9 = 1.001953125 (exact in fp32), -1 -> 2^-9, + 2^-9 = 2^-8
    out = orc.combine(y, w, pos)
    assert orc.bf16_to_f32(int(out[0, 0])) == 2.0 ** -8
    # the reverse order would also be 2^-8 here; make one where it is not:
    y2 = bf16_of([[2.0 ** 24], [1.0], [-(2.0 ** 24)]])
    w2 = np.array([[1.0, 1.0, 1.0]], np.float32)
    out2 = orc.combine(y2, w2, np.array([[0, 1, 2]], np.int32))
    assert orc.bf16_to_f32(int(out2[0, 0])) == 0.0      # 2^24 + 1 rounds to 2^24 in fp32
    out3 = orc.combine(y2, w2, np.array([[0, 2, 1]], np.int32))
    assert orc.bf16_to_f32(int(out3[0, 0])) == 1.0


def test_combine_small_integers_exact(orc):
    rng = np.random.default_rng(12)
    T, k, H, n = 20, 8, 64, 100
    yv = rng.integers(-64, 65, size=(n, H)).astype(np.float32)
    w = (rng.integers(-8, 9, size=(T, k)) / 8.0).astype(np.float32)
    pos = rng.integers(0, n, size=(T, k)).astype(np.int32)
    out = orc.combine(bf16_of(yv.tolist()), w, pos)
    want = np.zeros((T, H))
    for j in range(k):
        want += w[:, j:j + 1].astype(np.float64) * yv[pos[:, j]].astype(np.float64)
    # |sum| <= 8 * 64 = 512 with step 1/8: exactly representable in fp32; round to bf16 exactly
    wantb = np.array([[bf16_bits(to_bf16(Fraction(v))) if v != 0 else 0 for v in row] for row in want])
    got = out.astype(np.int64)
    got[got == 0x8000] = 0  # -0 and +0 are the same value here
    assert (got == wantb).all()


def test_combine_k1_inverse_permutation(orc):
    w = W.WORKLOADS["tiny"].scaled(k=1)
    x, idx, _ = W.make_routing(w)
    _, L = orc.layout(idx.numpy(), w.E, w.R)
    recv = orc.dispatch_bf16(x, L.pos, L.n_rows)
    out = orc.combine(recv, np.ones((w.T, 1), np.float32), L.pos)
    assert (out == u16(x)).all()


@pytest.mark.parametrize("name", ["tiny", "large_skewed"])
def test_roundtrip_bf16_exact(orc, name):
    w = W.WORKLOADS[name].scaled(T=min(W.WORKLOADS[name].T, 512))
    x, idx, tw = W.make_routing(w)
    _, L = orc.layout(idx.numpy(), w.E, w.R)
    recv = orc.dispatch_bf16(x, L.pos, L.n_rows)
    out = orc.combine(recv, tw.numpy(), L.pos)        # identity experts
    xs = u16(x).astype(np.int64)
    got = out.astype(np.int64)
    zero = (xs & 0x7FFF) == 0
    assert (got[~zero] == xs[~zero]).all()
    assert ((got[zero] & 0x7FFF) == 0).all()


@pytest.mark.parametrize("name", ["prefill", "group_limited"])
def test_roundtrip_fp8_bound(orc, name):
    w = W.WORKLOADS[name].scaled(T=32)
    x, idx, tw = W.make_routing(w)
    _, L = orc.layout(idx.numpy(), w.E, w.R)
    q, s = orc.dispatch_fp8(x, L.pos, L.n_rows)
    table = np.array([orc.e4m3_decode(c) for c in range(256)], np.float32)
    deq = table[q] * np.repeat(s, 128, axis=1)             # identity expert on dequantised rows
    y = torch.from_numpy(deq.astype(np.float32)).to(torch.bfloat16)
    out = orc.combine(y, tw.numpy(), L.pos)
    outf = orc.bits_to_f32(out).astype(np.float64)
    xf = x.to(torch.float64).numpy()
    sg = np.repeat(s[L.pos[:, 0]], 128, axis=1).astype(np.float64)
    assert (np.abs(outf - xf) <= 0.07 * np.abs(xf) + 2.0 ** -9 * sg).all()


def test_combine_golden_by_hand(orc):
    # 0.5 * 1.0 + 0.25 * 2.0 = 1.0; 0.5 * 3.0 + 0.25 * (-2.0) = 1.0; slot -1 skipped
    y = bf16_of([[1.0, 3.0], [2.0, -2.0], [100.0, 100.0]])
    w = np.array([[0.5, 0.25, 7.0]], np.float32)
    pos = np.array([[0, 1, -1]], np.int32)
    out = orc.combine(y, w, pos)
    assert out.tolist() == [[0x3F80, 0x3F80]]


def test_combine_is_fused(orc):
    """w*y rounded before the add would cancel to 0 here; the fused chain keeps
    the -2^-27 residual of the second product (exactly representable in bf16)."""
    y = bf16_of([[1.0 + 2.0 ** -7], [-(1.0 + 2.0 ** -7)]])
    w = np.array([[1.0 + 2.0 ** -20, 1.0 + 2.0 ** -20]], np.float32)
    out = orc.combine(y, w, np.array([[0, 1]], np.int32))
    assert orc.bf16_to_f32(int(out[0, 0])) == -(2.0 ** -27)


# --- pre-quantised FP8 input -------------------------------------------------

@pytest.mark.parametrize("name", ["prefill", "decode"])
def test_prequant_dispatch_equals_quantise_then_dispatch(orc, name):
    """Quantising each token first and dispatching the codes gives exactly the
    fused FP8 dispatch; and every received row is its source token's row."""
    w = W.WORKLOADS[name].scaled(T=64)
    x, idx, _ = W.make_routing(w)
    _, L = orc.layout(idx.numpy(), w.E, w.R, capacity=w.capacity)
    xq, xs = orc.quantize_rows(x)
    q1, s1 = orc.dispatch_fp8_prequant(xq, xs, L.pos, L.n_rows)
    q2, s2 = orc.dispatch_fp8(x, L.pos, L.n_rows)
    assert (q1 == q2).all() and (s1.view(np.uint32) == s2.view(np.uint32)).all()
    rows = np.nonzero(L.src_idx >= 0)[0]
    assert (q1[rows] == xq[L.src_idx[rows]]).all()
    assert (s1[rows] == xs[L.src_idx[rows]]).all()
