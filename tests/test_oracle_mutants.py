"""The oracle's pins catch plausible mistakes (CPU only).

Each case plants one mistake in a copy of the oracle's C source (never in the
source itself), builds the copy, points the oracle wrapper at it and runs the
pins that guard that part of the definition: at least one of them must fail.
"""
import os
import subprocess

import pytest

import oracle
from oracle import build as oracle_build

import test_oracle_backward as PB
import test_oracle_dispatch_combine as PD
import test_oracle_formats as PF
import test_oracle_layout as PL
import test_oracle_topk as PT

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "ep_oracle.c")

# (name, text in the oracle, replacement, pins as (function, kwargs))
MUTANTS = [
    ("positions in reversed slot order",
     "        for (int j = 0; j < k; ++j) {\n            int64_t s = (int64_t)t * k + j;\n            int e = valid_id(topk_idx[s], E);",
     "        for (int j = k - 1; j >= 0; --j) {\n            int64_t s = (int64_t)t * k + j;\n            int e = valid_id(topk_idx[s], E);",
     # slot order only matters when a token names one expert twice
     [(PL.test_duplicates_and_unused_slots, {})] + [(PL.test_bruteforce_tiny, {"trial": t}) for t in range(20)]),
    ("capacity overflow not reported",
     "                over = 1;",
     "                over = 0;",
     [(PL.test_golden_layout, {})]),
    ("invalid expert id not reported",
     "            bad_id = 1;",
     "            bad_id = 0;",
     [(PL.test_bruteforce_tiny, {"trial": 6}), (PL.test_errors, {})]),
    ("rank of an expert taken modulo R",
     "in_rank[(int64_t)t * R + e / experts_per_rank] = 1;",
     "in_rank[(int64_t)t * R + e % R] = 1;",
     [(PL.test_golden_layout, {}), (PL.test_invariants_full_workloads, {"name": "tiny"})]),
    ("expert alignment ignored",
     "seg[e + 1] = (int32_t)(seg[e] + align_up64(cnt[e], align));",
     "seg[e + 1] = (int32_t)(seg[e] + cnt[e]);",
     [(PL.test_golden_layout, {})]),
    ("padded segment start off by one",
     "seg[e + 1] = (int32_t)((int64_t)(e + 1) * capacity);",
     "seg[e + 1] = (int32_t)((int64_t)(e + 1) * capacity + 1);",
     [(PL.test_golden_layout, {})]),
    ("scale constant 440 instead of 448",
     "*scale = amax / 448.0f;", "*scale = amax / 440.0f;",
     [(PD.test_golden_fp8_group, {}), (PD.test_quantize_vs_exact, {"mag": 1.0})]),
    ("inverse scale rounded from another constant",
     "float inv = 448.0f / amax;", "float inv = 447.0f / amax;",
     [(PD.test_golden_fp8_group, {}), (PD.test_quantize_vs_exact, {"mag": 1.0})]),
    ("e4m3 ties rounded away from zero",
     "if (rest > 0x80000u || (rest == 0x80000u && (keep & 1u))) {",
     "if (rest >= 0x80000u) {",
     [(PF.test_e4m3_encode_ties_and_saturation, {})]),
    ("all-zero group through the general path",
     "    if (amax == 0.0f) {\n        *scale = 0.0f;",
     "    if (0) {\n        *scale = 0.0f;",
     [(PD.test_golden_fp8_group, {})]),
    ("bf16 rounding by truncation",
     "if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) {",
     "if (0) {",
     [(PF.test_bf16_rounding_vs_exact, {})]),
    ("combine summed in reversed slot order",
     "            float acc = 0.0f;\n            for (int j = 0; j < k; ++j) {",
     "            float acc = 0.0f;\n            for (int j = k - 1; j >= 0; --j) {",
     [(PD.test_combine_order_matters_and_is_slot_order, {}), (PD.test_combine_fma_chain_exact, {})]),
    ("combine with a rounded product (no fma)",
     "acc = fmaf(w[(int64_t)t * k + j], oracle_bf16_to_f32(y[(int64_t)p * H + i]), acc);",
     "acc = w[(int64_t)t * k + j] * oracle_bf16_to_f32(y[(int64_t)p * H + i]) + acc;",
     [(PD.test_combine_is_fused, {}), (PD.test_combine_fma_chain_exact, {})]),
    ("combine with the weights dropped",
     "acc = fmaf(w[(int64_t)t * k + j], oracle_bf16_to_f32(y[(int64_t)p * H + i]), acc);",
     "acc = fmaf(1.0f, oracle_bf16_to_f32(y[(int64_t)p * H + i]), acc);",
     [(PD.test_combine_golden_by_hand, {})]),
    ("grad_y without the weight",
     "float prod = w[s] * g;", "float prod = g;",
     [(PB.test_combine_backward_vs_autograd, {"name": "tiny"})]),
    ("pre-quantised scales copied from the next token",
     "memcpy(scales + (int64_t)p * G, xs + (int64_t)t * G, (size_t)G * sizeof(float));",
     "memcpy(scales + (int64_t)p * G, xs + (int64_t)(t + 1 < T ? t + 1 : t) * G, (size_t)G * sizeof(float));",
     [(PD.test_prequant_dispatch_equals_quantise_then_dispatch, {"name": "decode"}),
      (PD.test_prequant_dispatch_equals_quantise_then_dispatch, {"name": "prefill"})]),
    ("pre-quantised codes of half a row",
     "memcpy(recv + (int64_t)p * H, xq + (int64_t)t * H, (size_t)H);",
     "memcpy(recv + (int64_t)p * H, xq + (int64_t)t * H, (size_t)H / 2);",
     [(PD.test_prequant_dispatch_equals_quantise_then_dispatch, {"name": "decode"}),
      (PD.test_prequant_dispatch_equals_quantise_then_dispatch, {"name": "prefill"})]),
    ("per-row weight taken from the neighbouring slot",
     "if (recv_w) recv_w[p] = topk_w[s];",
     "if (recv_w) recv_w[p] = topk_w[s ^ 1];",
     [(PT.test_golden_dispatch_topk, {"case": PT.TOPK["cases"][0]}),
      (PT.test_packed_equals_stable_sort, {"name": "tiny"})]),
    ("per-row slot id without the token",
     "if (recv_slot) recv_slot[p] = (int32_t)s;",
     "if (recv_slot) recv_slot[p] = (int32_t)j;",
     [(PT.test_golden_dispatch_topk, {"case": PT.TOPK["cases"][0]}),
      (PT.test_packed_equals_stable_sort, {"name": "tiny"})]),
    ("padding rows keep a stale weight",
     "        if (recv_w) recv_w[r] = 0.0f;",
     "        if (recv_w) recv_w[r] = 1.0f;",
     [(PT.test_golden_dispatch_topk, {"case": PT.TOPK["cases"][1]})]),
    ("grad_w missing the last channel",
     "            double dot = 0.0;\n            for (int i = 0; i < H; ++i) {",
     "            double dot = 0.0;\n            for (int i = 0; i < H - 1; ++i) {",
     [(PB.test_combine_backward_vs_autograd, {"name": "tiny"})]),
]

# Saturation needs two edits at once: the early return for |x| >= 448 and the clamp.
SATURATION = [
    ("    if (a >= 448.0f) {\n        return (uint8_t)(sign | 0x7e);\n    }",
     "    if (a >= 1e30f) {\n        return (uint8_t)(sign | 0x7e);\n    }"),
    ("    if (code > 0x7eu) {\n        code = 0x7eu;\n    }",
     "    if (code > 0x7fu) {\n        code = 0x7fu;\n    }"),
]


def build_mutant(edits, tmp_path):
    src = open(SRC).read()
    for old, new in edits:
        assert src.count(old) == 1, "mutation site not found exactly once: %r" % old[:60]
        src = src.replace(old, new)
    c = tmp_path / "mutant.c"
    so = tmp_path / "libmutant.so"
    c.write_text(src)
    res = subprocess.run(["gcc", *oracle_build.CFLAGS, str(c), "-o", str(so), "-lm"],
                         capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    return oracle.load(str(so))


def caught(pins):
    for fn, kw in pins:
        try:
            fn(oracle, **kw)
        except (AssertionError, oracle.OracleError):
            return True
    return False


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda m: m[0])
def test_pins_catch_planted_mistake(mutant, tmp_path, monkeypatch):
    name, old, new, pins = mutant
    monkeypatch.setattr(oracle, "_LIB", build_mutant([(old, new)], tmp_path))
    assert caught(pins), "no pin failed for: " + name


def test_pins_catch_missing_saturation(tmp_path, monkeypatch):
    monkeypatch.setattr(oracle, "_LIB", build_mutant(SATURATION, tmp_path))
    assert caught([(PF.test_e4m3_encode_ties_and_saturation, {})])


def test_unmutated_copy_passes(tmp_path, monkeypatch):
    """Control: the same build route without a mistake passes the same pins."""
    monkeypatch.setattr(oracle, "_LIB", build_mutant([], tmp_path))
    pins = {id(fn): (fn, kw) for m in MUTANTS for fn, kw in m[3]}
    assert not caught(list(pins.values()))
