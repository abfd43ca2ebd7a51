"""bench.py's byte accounting and throughput arithmetic (CPU only).

`value` and `roofline.achieved` are algorithmic bytes over device time, so
the byte counts are worked out here by hand from the sizes of every array a
call must read or write, and compared with bench.py's formulas:

  dispatch FP8:  x bf16 [T,H] read, pos int32 [T,k] read, e4m3 codes and one
                 fp32 scale per 128 channels written to each valid slot's row;
  dispatch BF16: x read, pos read, a bf16 row written per valid slot;
  combine:       a bf16 row read per valid slot, topk weights and pos read
                 (fp32 / int32 [T,k]), out bf16 [T,H] written;
  layout:        ids read, counts [E] and [R] and is_token_in_rank [T,R]
                 written, pos [T,k], src_idx [rows], seg [E+1], rank_off [R+1].
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from combine_ep_layout_10_b200 import workloads as W  # noqa: E402


def test_metric_workload_bytes_by_hand():
    w = W.WORKLOADS["group_limited"]
    T, H, k, E, R = 8192, 7168, 8, 256, 64
    assert (w.T, w.H, w.k, w.E, w.R, w.fp8) == (T, H, k, E, R, True)
    V = T * k                                   # group-limited routing uses every slot
    x, pos, codes, scales = T * H * 2, T * k * 4, V * H, V * (H // 128) * 4
    assert (x, pos, codes, scales) == (117_440_512, 262_144, 469_762_048, 14_680_064)
    got = bench.algorithmic_bytes(w, V, V)
    assert got["dispatch"] == x + pos + codes + scales == 602_144_768
    rows_in, weights, out = V * H * 2, T * k * 4, T * H * 2
    assert got["combine"] == rows_in + weights + pos + out == 1_057_488_896
    layout = T * k * 4 + E * 4 + R * 4 + T * R + T * k * 4 + V * 4 + (E + 1) * 4 + (R + 1) * 4
    assert got["layout"] == layout == 1_313_288
    assert got["step"] == got["layout"] + got["dispatch"] + got["combine"]


def test_bf16_workload_bytes_by_hand():
    w = W.WORKLOADS["large_skewed"]
    T, H, k = w.T, w.H, w.k
    assert not w.fp8
    V = T * k - 1000                            # some unused slots: only valid slots move rows
    got = bench.algorithmic_bytes(w, V, V)
    assert got["dispatch"] == T * H * 2 + T * k * 4 + V * H * 2
    assert got["combine"] == V * H * 2 + 2 * T * k * 4 + T * H * 2


def test_job_throughput_one_rank():
    # 2 GB per step, 10 steps of 0.25 ms: 8,000 GB/s (the multi-rank max / sum
    # over gloo ranks is tests/test_multirank.py)
    value, ms = bench.job_throughput(0.25, 2e9, 10, 1)
    assert ms == 0.25
    assert value == pytest.approx(8000.0)


def test_reference_sample_bytes():
    """The reference arm counts the layout of every token plus the dispatch
    and combine of its n-token sample (all slots valid in the sample)."""
    w = W.WORKLOADS["group_limited"]
    n = 1024
    rows_full = bench.algorithmic_bytes(w, w.T * w.k, w.T * w.k)
    sub = bench.algorithmic_bytes(w.scaled(T=n), n * w.k, n * w.k)
    assert bench.oracle_bytes(w, n, w.T * w.k) == rows_full["layout"] + sub["dispatch"] + sub["combine"]


def test_measured_peak_is_read_from_the_repository():
    p = bench.measured_peaks()
    if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
        assert p["source"] == "measured" and p["hbm_gbs"] > 1000
    else:
        assert p == {"hbm_gbs": bench.HBM_FALLBACK_GBS, "source": "fallback"}
