"""Pins for the oracle's routing layout (CPU only).

The oracle computes positions with a running per-expert fill counter.  It is
checked here against formulations that share nothing with that loop:
  * a hand-derived golden fixture (tests/golden/layout_small.json),
  * brute-force counting on tiny inputs: pos(t,j) = seg[e] + the number of
    earlier slots (in (token, slot) order) that name the same expert,
  * torch.sort(stable=True) of the flattened expert ids, whose stable order is
    exactly (expert, token, slot),
  * invariants on the full-size workloads.
"""
import json
import os

import numpy as np
import pytest
import torch

from combine_ep_layout_10_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_golden_layout(orc):
    d = json.load(open(os.path.join(GOLDEN, "layout_small.json")))
    idx = np.array(d["topk_idx"], np.int32)
    for case in d["cases"]:
        st, L = orc.layout(idx, d["E"], d["R"], align=case["align"], capacity=case["capacity"],
                           check=False)
        assert st == case["status"], case
        assert L.num_tokens_per_expert.tolist() == case["num_tokens_per_expert"]
        assert L.num_tokens_per_rank.tolist() == case["num_tokens_per_rank"]
        assert L.is_token_in_rank.tolist() == case["is_token_in_rank"]
        assert L.seg.tolist() == case["seg"]
        assert L.rank_off.tolist() == case["rank_off"]
        assert L.pos.tolist() == case["pos"]
        assert L.src_idx.tolist() == case["src_idx"]


def brute_layout(idx, E, R, align, capacity):
    """Independent definition by counting (no running fill counter).  An id
    outside [-1, E) is an unused slot; a padded expert keeps its first
    `capacity` slots in (token, slot) order."""
    T, k = len(idx), len(idx[0]) if len(idx) else 0
    epr = E // R
    idx = [[e if 0 <= e < E else -1 for e in row] for row in idx]
    slots = [(t, j) for t in range(T) for j in range(k)]
    cnt = [sum(1 for (t, j) in slots if idx[t][j] == e) for e in range(E)]
    if capacity:
        seg = [e * capacity for e in range(E + 1)]
    else:
        seg = [sum(-(-cnt[f] // align) * align for f in range(e)) for e in range(E + 1)]
    pos = [[-1] * k for _ in range(T)]
    for (t, j) in slots:
        e = idx[t][j]
        if e < 0:
            continue
        before = sum(1 for (t2, j2) in slots if (t2, j2) < (t, j) and idx[t2][j2] == e)
        if capacity and before >= capacity:
            continue
        pos[t][j] = seg[e] + before
    in_rank = [[int(any(idx[t][j] >= 0 and idx[t][j] // epr == r for j in range(k)))
                for r in range(R)] for t in range(T)]
    rank_tok = [sum(in_rank[t][r] for t in range(T)) for r in range(R)]
    rank_off = [seg[r * epr] for r in range(R + 1)]
    return cnt, seg, pos, in_rank, rank_tok, rank_off


@pytest.mark.parametrize("trial", range(60))
def test_bruteforce_tiny(orc, trial):
    rng = np.random.default_rng(100 + trial)
    T = int(rng.integers(0, 9))
    k = int(rng.integers(1, 4))
    E = int(rng.choice([1, 2, 4, 6, 8]))
    R = int(rng.choice([r for r in (1, 2, 3, 4, 8) if E % r == 0]))
    align = int(rng.choice([1, 1, 2, 4]))
    capacity = 0
    if trial % 5 == 4:
        capacity = align * int(rng.integers(T * k // max(E, 1) + 1, T * k // max(E, 1) + 4))
    elif trial % 10 == 3:
        capacity = align            # tight: experts overflow and keep their first slots
    # ids in [-1, E): duplicates inside a token and unused slots on purpose
    idx = rng.integers(-1, E, size=(T, k)).astype(np.int32)
    if trial % 7 == 6 and T:
        idx[int(rng.integers(0, T)), int(rng.integers(0, k))] = [E, -2, E + 7][trial % 3]   # invalid id
    cnt_b, seg_b, pos_b, in_rank_b, rank_tok_b, rank_off_b = brute_layout(idx.tolist(), E, R, align, capacity)
    st, L = orc.layout(idx.reshape(T, k), E, R, align=align, capacity=capacity, check=False)
    bad = bool(((idx < -1) | (idx >= E)).any())
    over = bool(capacity) and max(cnt_b, default=0) > capacity
    assert st == (2 if bad else 3 if over else 0)
    assert L.num_tokens_per_expert.tolist() == cnt_b
    assert L.seg.tolist() == seg_b
    assert L.pos.reshape(T, k).tolist() == pos_b
    assert L.is_token_in_rank.reshape(T, R).tolist() == in_rank_b
    assert L.num_tokens_per_rank.tolist() == rank_tok_b
    assert L.rank_off.tolist() == rank_off_b
    # src_idx: the inverse of pos, -1 elsewhere
    want_src = [-1] * L.n_rows
    for t in range(T):
        for j in range(k):
            if pos_b[t][j] >= 0:
                want_src[pos_b[t][j]] = t
    assert L.src_idx.tolist() == want_src


def check_invariants(L, idx):
    T, k = idx.shape
    E, R = L.E, L.R
    epr = E // R
    valid = idx >= 0
    V = int(valid.sum())
    cnt = L.num_tokens_per_expert
    assert int(cnt.sum()) == V
    assert (cnt == np.bincount(idx[valid], minlength=E)).all()
    # is_token_in_rank <=> the token has an expert owned by that rank
    owner = np.where(valid, idx // epr, -1)
    want = np.zeros((T, R), np.uint8)
    for j in range(k):
        m = owner[:, j] >= 0
        want[np.nonzero(m)[0], owner[m, j]] = 1
    assert (L.is_token_in_rank == want).all()
    assert (L.num_tokens_per_rank == want.sum(0)).all()
    assert (L.num_tokens_per_rank <= T).all()
    if V == T * k:
        assert int(L.num_tokens_per_rank.sum()) >= T
    # segments: monotone, wide enough, aligned
    seg = L.seg
    assert seg[0] == 0 and (np.diff(seg) >= np.maximum(cnt, 0)).all()
    if L.capacity == 0:
        assert (np.diff(seg) % L.align == 0).all() and (np.diff(seg) < cnt + L.align).all()
    assert (L.rank_off == seg[np.arange(R + 1) * epr]).all()
    # pos / src_idx are mutual inverses; pos inside the expert's segment
    pos = L.pos
    assert ((pos >= 0) == valid).all()
    e = np.where(valid, idx, 0)
    assert ((pos >= seg[e]) & (pos < seg[e] + cnt[e]) | ~valid).all()
    t_of = np.repeat(np.arange(T), k).reshape(T, k)
    assert (L.src_idx[pos[valid]] == t_of[valid]).all()
    assert int((L.src_idx >= 0).sum()) == V
    # inside every segment, source tokens never decrease
    for ee in range(E):
        s = L.src_idx[seg[ee]:seg[ee] + cnt[ee]]
        assert (np.diff(s) >= 0).all()


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_invariants_full_workloads(orc, name):
    w = W.WORKLOADS[name]
    _, idx, _ = W.make_routing(w)
    idx = idx.numpy()
    st, L = orc.layout(idx, w.E, w.R, align=w.align, capacity=w.capacity, check=False)
    assert st == 0
    check_invariants(L, idx)


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_stable_sort_crosscheck(orc, name):
    """torch.sort(stable=True) of the flattened ids gives the slots in
    (expert, token, slot) order, i.e. the receive order; with segments packed
    (align 1) that order *is* src_idx and its inverse is pos."""
    w = W.WORKLOADS[name].scaled(capacity=0, align=1)
    _, idx, _ = W.make_routing(w)
    st, L = orc.layout(idx.numpy(), w.E, w.R)
    flat = idx.reshape(-1).to(torch.int64)
    order = torch.sort(flat, stable=True).indices          # slots by (expert, slot id)
    order = order[flat[order] >= 0]
    V = order.numel()
    assert (L.src_idx[:V] == (order // w.k).numpy()).all()
    pos = np.full(flat.numel(), -1, np.int64)
    pos[order.numpy()] = np.arange(V)
    assert (L.pos.reshape(-1) == pos).all()


def test_duplicates_and_unused_slots(orc):
    idx = np.array([[1, 1, -1], [-1, -1, -1], [0, 1, 0]], np.int32)
    st, L = orc.layout(idx, 2, 1)
    assert st == 0
    assert L.num_tokens_per_expert.tolist() == [2, 3]
    assert L.pos.tolist() == [[2, 3, -1], [-1, -1, -1], [0, 4, 1]]
    assert L.src_idx.tolist() == [2, 2, 0, 0, 2, -1, -1, -1, -1]
    assert L.is_token_in_rank.tolist() == [[1], [0], [1]]


def test_special_cases(orc):
    rng = np.random.default_rng(7)
    idx = np.stack([rng.permutation(16)[:4] for _ in range(50)]).astype(np.int32)
    # R = 1: every token with a valid slot is on the only rank
    _, L = orc.layout(idx, 16, 1)
    assert (L.is_token_in_rank == 1).all() and L.num_tokens_per_rank.tolist() == [50]
    # R = E: one expert per rank, so in_rank is the one-hot of the ids
    _, L = orc.layout(idx, 16, 16)
    oh = np.zeros((50, 16), np.uint8)
    for j in range(4):
        oh[np.arange(50), idx[:, j]] = 1
    assert (L.is_token_in_rank == oh).all()
    # k = 1: positions are the stable argsort's inverse
    idx1 = idx[:, :1].copy()
    _, L = orc.layout(idx1, 16, 4)
    order = np.argsort(idx1[:, 0], kind="stable")
    assert (L.src_idx == order).all()
    # T = 0
    st, L = orc.layout(np.zeros((0, 4), np.int32), 16, 4)
    assert st == 0 and L.n_rows == 0 and (L.seg == 0).all()


def test_errors(orc):
    idx = np.array([[0, 1], [2, 3]], np.int32)
    assert orc.layout(idx, 4, 3, check=False)[0] == orc.OR_ERR_INVALID_ARG       # E % R
    assert orc.layout(idx, 4, 2, align=0, check=False)[0] == orc.OR_ERR_INVALID_ARG
    assert orc.layout(idx, 4, 2, capacity=3, align=2, check=False)[0] == orc.OR_ERR_INVALID_ARG
    bad = np.array([[0, 4], [2, 3]], np.int32)
    assert orc.layout(bad, 4, 2, check=False)[0] == orc.OR_ERR_BAD_EXPERT_ID
    bad = np.array([[0, -2], [2, 3]], np.int32)
    assert orc.layout(bad, 4, 2, check=False)[0] == orc.OR_ERR_BAD_EXPERT_ID
    over = np.array([[0, 1], [0, 2], [0, 3]], np.int32)
    assert orc.layout(over, 4, 2, capacity=2, check=False)[0] == orc.OR_ERR_CAPACITY
    # both: the bad id is reported; the layout is still complete
    both = np.array([[0, 9], [0, 2], [0, 3]], np.int32)
    st, L = orc.layout(both, 4, 2, capacity=2, check=False)
    assert st == orc.OR_ERR_BAD_EXPERT_ID
    assert L.pos.tolist() == [[0, -1], [1, 4], [-1, 6]]
    assert L.num_tokens_per_expert.tolist() == [3, 0, 1, 1]
    assert orc.max_recv_rows(10, 8, 4, 1, 0) == 80
    assert orc.max_recv_rows(10, 8, 4, 4, 0) == 92
    assert orc.max_recv_rows(10, 8, 4, 1, 16) == 64
    assert orc.max_recv_rows(-1, 8, 4, 1, 0) == -1
