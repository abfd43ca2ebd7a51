"""Pins for the oracle's per-row routing outputs of dispatch (CPU only).

Dispatch also returns recv_topk_idx and recv_topk_weights ("DeepEP
(DeepEveryParallel) Documentation", item 10).  Each receive row of the
expert-major layout holds one slot, so the outputs are that slot's expert,
weight and flat index.  Checked against
  * a hand-derived golden fixture (tests/golden/dispatch_topk_small.json),
  * torch.sort(stable=True) of the flattened expert ids (a library routine
    whose stable order is exactly the (expert, token, slot) order),
  * invariants that hold at any size: segment membership, the bijection
    between filled rows and used slots, src_idx agreement, padding values.
"""
import json
import os

import numpy as np
import pytest
import torch

from combine_ep_layout_10_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
LAYOUT = json.load(open(os.path.join(GOLDEN, "layout_small.json")))
TOPK = json.load(open(os.path.join(GOLDEN, "dispatch_topk_small.json")))


@pytest.mark.parametrize("case", TOPK["cases"], ids=lambda c: "align%d_cap%d" % (c["align"], c["capacity"]))
def test_golden_dispatch_topk(orc, case):
    idx = np.array(LAYOUT["topk_idx"], np.int32)
    w = np.array(TOPK["topk_weights"], np.float32)
    pos = np.array(case["pos"], np.int32)
    ri, rw, rs = orc.dispatch_topk(idx, w, pos, case["n_rows"])
    assert ri.tolist() == case["recv_topk_idx"]
    assert rw.tolist() == [np.float32(v) for v in case["recv_topk_weights"]]
    assert rs.tolist() == case["recv_slot"]
    assert not np.any(rw == np.float32(0.3)), "the unused slot's weight must not appear"


def check_invariants(idx, w, res, ri, rw, rs):
    T, k = idx.shape
    L = res
    filled = L.src_idx >= 0
    # padding rows
    assert (ri[~filled] == -1).all() and (rs[~filled] == -1).all()
    assert (rw[~filled].view(np.uint32) == 0).all()
    # bijection between filled rows and used slots
    used = np.flatnonzero(L.pos.reshape(-1) >= 0)
    assert sorted(rs[filled].tolist()) == used.tolist()
    rows = np.flatnonzero(filled)
    s = rs[filled]
    assert (L.pos.reshape(-1)[s] == rows).all()
    assert (s // k == L.src_idx[filled]).all()
    assert (ri[filled] == idx.reshape(-1)[s]).all()
    assert (rw[filled].view(np.uint32) == w.reshape(-1)[s].view(np.uint32)).all()
    # every filled row lies in the segment of its expert
    e = ri[filled]
    assert (L.seg[e] <= rows).all() and (rows < L.seg[e + 1]).all()


@pytest.mark.parametrize("name,T,align,cap", [("tiny", None, 1, 0), ("tiny", None, 4, 0),
                                              ("prefill", 200, 1, 0), ("decode", None, 1, 128),
                                              ("group_limited", 256, 8, 0)])
def test_invariants(orc, name, T, align, cap):
    wl = W.WORKLOADS[name]
    wl = wl.scaled(T=T) if T else wl
    _, idx, tw = W.make_routing(wl)
    idx = idx.numpy().copy()
    idx[::5, -1] = -1                   # unused slots
    idx[1::7, 0] = idx[1::7, 1]         # a token naming one expert twice
    tw = tw.numpy()
    cap = cap if cap == 0 else max(cap, int(np.bincount(idx[idx >= 0], minlength=wl.E).max()))
    _, L = orc.layout(idx, wl.E, wl.R, align, cap)
    ri, rw, rs = orc.dispatch_topk(idx, tw, L.pos, L.n_rows)
    check_invariants(idx, tw, L, ri, rw, rs)


@pytest.mark.parametrize("name", ["tiny", "prefill", "group_limited"])
def test_packed_equals_stable_sort(orc, name):
    """Packed, alignment 1, no unused slot: the filled rows are the flattened
    slots stably sorted by expert id, so recv_slot is torch's stable argsort,
    recv_topk_idx the sorted ids and recv_topk_weights the weights gathered
    in that order."""
    wl = W.WORKLOADS[name]
    wl = wl.scaled(T=min(wl.T, 512))
    _, idx, tw = W.make_routing(wl)
    _, L = orc.layout(idx.numpy(), wl.E, wl.R)
    ri, rw, rs = orc.dispatch_topk(idx.numpy(), tw.numpy(), L.pos, L.n_rows)
    vals, order = torch.sort(idx.reshape(-1), stable=True)
    n = order.numel()
    assert (rs[:n] == order.numpy()).all()
    assert (ri[:n] == vals.numpy()).all()
    assert (rw[:n] == tw.reshape(-1)[order].numpy()).all()
    assert (rs[n:] == -1).all()
