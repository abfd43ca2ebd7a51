"""The hardware e4m3 conversion FP8 dispatch uses, against the oracle's
software encoder, over every finite fp32 bit pattern (GPU).

The oracle's encoder is written from the OCP FP8 E4M3 definition and pinned
on CPU (tests/test_oracle_formats.py).  ep_e4m3_encode runs the very
conversion the dispatch kernels use (round to nearest even, saturate finite
overflow to +-448).  Here every one of the 2^32 - 2^24 finite fp32 values is
encoded both ways and compared bit for bit, in chunks of 2^28.  Infinities
and NaN, which the oracle does not define, are checked against the stated
behaviour: +-inf gives +-448, NaN gives a NaN code.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_ep_layout_10_b200 import ep

pytestmark = pytest.mark.gpu
DEV = "cuda"
CHUNK = 1 << 28


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from combine_ep_layout_10_b200 import build
    build.build()
    ep.lib()
    oracle.lib()


def test_e4m3_conversion_matches_the_oracle_on_every_finite_fp32():
    mismatches = 0
    for start in range(0, 1 << 32, CHUNK):
        bits = np.arange(start, start + CHUNK, dtype=np.uint32)
        finite = (bits & np.uint32(0x7F800000)) != np.uint32(0x7F800000)
        v = bits.view(np.float32)
        got = ep.e4m3_encode(torch.from_numpy(v).to(DEV)).cpu().numpy()
        want = oracle.e4m3_encode_array(v[finite])
        mismatches += int((got[finite] != want).sum())
        assert mismatches == 0, "first mismatch in the chunk starting at bit pattern %#x" % start


def test_e4m3_conversion_specials_and_ragged_tail():
    x = torch.tensor([float("inf"), -float("inf"), float("nan"), 448.0, 464.0, -1e30, 0.0, -0.0, 2.0 ** -9,
                      2.0 ** -10, 3.0 * 2.0 ** -11], dtype=torch.float32, device=DEV)
    got = ep.e4m3_encode(x).cpu().numpy().tolist()
    assert got[0] == 0x7E and got[1] == 0xFE            # infinities saturate to +-448
    assert got[2] & 0x7F == 0x7F                        # NaN stays NaN
    assert got[3] == 0x7E and got[4] == 0x7E and got[5] == 0xFE
    assert got[6] == 0x00 and got[7] == 0x80            # signed zero kept
    assert got[8] == 0x01                               # smallest subnormal
    # 2^-10 is half the smallest subnormal: a tie, to even (zero); 1.5 * 2^-10 rounds up
    assert got[9] == 0x00 and got[10] == 0x01
    # lengths that are not a multiple of the 8-value vector take the scalar tail
    for n in (1, 7, 9, 1023):
        v = torch.randn(n, generator=torch.Generator().manual_seed(n)) * 100
        assert (ep.e4m3_encode(v.to(DEV)).cpu().numpy() == oracle.e4m3_encode_array(v.numpy())).all()
