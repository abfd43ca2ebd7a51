"""Pins for the oracle's number formats (CPU only).

e4m3 (OCP FP8 E4M3, the "fn" variant: no infinities, max 448) and bf16
rounding are checked against
  * values that follow from the format definition by hand,
  * a library routine (torch.float8_e4m3fn / torch.bfloat16 conversions),
    exhaustively over the in-range binary32 inputs for e4m3,
  * exact rational rounding written in tests/exact.py.
"""
import numpy as np
import torch

from exact import f32, to_bf16
from fractions import Fraction


# --- e4m3 decode -----------------------------------------------------------

def test_e4m3_decode_anchor_values(orc):
    # From the format definition: bias 7, 3 mantissa bits, subnormal step 2^-9.
    assert orc.e4m3_decode(0x00) == 0.0
    assert orc.e4m3_decode(0x01) == 2.0 ** -9
    assert orc.e4m3_decode(0x07) == 7 * 2.0 ** -9
    assert orc.e4m3_decode(0x08) == 2.0 ** -6
    assert orc.e4m3_decode(0x38) == 1.0
    assert orc.e4m3_decode(0x39) == 1.125
    assert orc.e4m3_decode(0x40) == 2.0
    assert orc.e4m3_decode(0x76) == 224.0
    assert orc.e4m3_decode(0x7E) == 448.0
    assert orc.e4m3_decode(0xB8) == -1.0
    assert np.isnan(orc.e4m3_decode(0x7F)) and np.isnan(orc.e4m3_decode(0xFF))


def test_e4m3_decode_table_matches_torch(orc):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float32).numpy()
    mine = np.array([orc.e4m3_decode(c) for c in range(256)], np.float32)
    nan = np.isnan(ref)
    assert (np.isnan(mine) == nan).all()
    assert (mine[~nan].view(np.uint32) == ref[~nan].view(np.uint32)).all()  # incl. -0


def test_e4m3_roundtrip_all_codes(orc):
    for c in range(256):
        v = orc.e4m3_decode(c)
        if np.isnan(v):
            continue
        assert orc.e4m3_encode(v) == c, hex(c)


# --- e4m3 encode -------------------------------------------------------------

def test_e4m3_encode_ties_and_saturation(orc):
    enc = orc.e4m3_encode
    # Midpoint of 1.0 (0x38, even) and 1.125 (0x39): ties to even -> 1.0
    assert enc(1.0625) == 0x38
    # Midpoint of 1.125 (odd) and 1.25 (0x3A, even) -> 1.25
    assert enc(1.1875) == 0x3A
    # Just above / below a midpoint
    assert enc(np.nextafter(np.float32(1.0625), np.float32(2)).item()) == 0x39
    assert enc(np.nextafter(np.float32(1.0625), np.float32(0)).item()) == 0x38
    # Subnormal grid: 2^-10 is the midpoint of 0 and 2^-9 -> 0 (even)
    assert enc(2.0 ** -10) == 0x00
    # 3*2^-10 is the midpoint of 2^-9 (odd) and 2*2^-9 -> 2*2^-9
    assert enc(3 * 2.0 ** -10) == 0x02
    # Rounding up out of the subnormals into the smallest normal
    assert enc(7.5 * 2.0 ** -9) == 0x08
    # Binade carry: 1.9375 = midpoint of 1.875 (odd) and 2.0 -> 2.0
    assert enc(1.9375) == 0x40
    # Saturation: 448 is the largest finite; 464 is the 448/480 midpoint (448 even)
    for v in (448.0, 450.0, 464.0, 465.0, 480.0, 1e30, float("inf")):
        assert enc(v) == 0x7E and enc(-v) == 0xFE, v
    # Sign of zero kept, tiny values round to signed zero
    assert enc(0.0) == 0x00 and enc(-0.0) == 0x80
    assert enc(-(2.0 ** -12)) == 0x80
    assert enc(float("nan")) == 0x7F


def _binade(exp_biased: int) -> np.ndarray:
    m = np.arange(1 << 23, dtype=np.uint32)
    return ((np.uint32(exp_biased) << np.uint32(23)) | m).view(np.float32)


def test_e4m3_encode_exhaustive_vs_torch(orc):
    """Every positive binary32 below 464 (all of binades 0..135, i.e. < 512,
    restricted to <= 464) against torch's round-to-nearest-even conversion."""
    checked = 0
    for eb in range(0, 136):
        v = _binade(eb)
        v = v[v <= 464.0]
        mine = orc.e4m3_encode_array(v)
        ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        bad = np.nonzero(mine != ref)[0]
        assert bad.size == 0, (eb, v[bad[:4]], mine[bad[:4]], ref[bad[:4]])
        checked += v.size
    assert checked > 1_100_000_000


def test_e4m3_encode_negative_sample_vs_torch(orc):
    rng = np.random.default_rng(1)
    v = -np.abs(rng.standard_normal(2_000_000).astype(np.float32)) * np.float32(40)
    v = v[v >= -464.0]
    mine = orc.e4m3_encode_array(v)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert (mine == ref).all()


# --- bf16 ------------------------------------------------------------------

def test_bf16_widening_exact(orc):
    for h in (0x0000, 0x8000, 0x3F80, 0xBF80, 0x7F7F, 0x0001, 0x4049):
        b = orc.bf16_to_f32(h)
        assert np.float32(b).view(np.uint32) == np.uint32(h << 16)


def test_bf16_rounding_vs_torch(orc):
    rng = np.random.default_rng(2)
    highs = np.concatenate([rng.integers(0, 1 << 16, 200, dtype=np.uint32),
                            np.array([0x0000, 0x0001, 0x3F80, 0x3F81, 0x7F7F, 0x7F7E, 0x8000,
                                      0x807F, 0xBF80, 0xFF7F, 0x0080, 0x007F], np.uint32)])
    lows = np.arange(1 << 16, dtype=np.uint32)
    for hi in highs:
        bits = (hi << np.uint32(16)) | lows
        v = bits.view(np.float32)
        fin = np.isfinite(v)
        mine = orc.f32_to_bf16_array(v[fin])
        ref = torch.from_numpy(v[fin].copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert (mine == ref).all(), hex(int(hi))


def test_bf16_rounding_vs_exact(orc):
    rng = np.random.default_rng(3)
    v = rng.standard_normal(3000).astype(np.float32) * np.float32(1000)
    for x in v.tolist():
        want = to_bf16(Fraction(x))
        got = orc.bf16_to_f32(orc.f32_to_bf16(x))
        assert got == want, x
    # ties: 1 + 2^-8 is the midpoint of 1.0 (even) and 1 + 2^-7 -> 1.0
    assert orc.f32_to_bf16(1.0 + 2.0 ** -8) == 0x3F80
    assert orc.f32_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82
    assert f32(1.0 + 2.0 ** -8) == 1.0 + 2.0 ** -8
