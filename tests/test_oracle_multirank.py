"""Pins for the multi-rank definition in oracle/multirank.py (CPU only).

The definition is "the single-GPU layout of the concatenated batch, sliced
by owner rank".  Pinned here, independently of that construction:
  * brute force: every rank's receive rows enumerated by explicit loops in
    (owned expert, source rank, source token, slot) order, with alignment
    padding, unused slots and duplicates, and different token counts per rank;
  * W = 1 reduces to the single-GPU oracle;
  * the identity-expert round trip: BF16 rows sent out and combined back with
    weights that sum to one return every token exactly (a closed form);
  * padded (capacity) mode places rows in concatenated token order and
    reports an overflow of the concatenated count.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import multirank as MR


def random_ids(rng, T, k, E, unused=0.0, dup=0.0):
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32) if T else \
        np.zeros((0, k), np.int32)
    if T and unused:
        idx[rng.random((T, k)) < unused] = -1
    if T and dup:
        rows = rng.random(T) < dup
        idx[rows, 0] = idx[rows, k - 1] if k > 1 else idx[rows, 0]
    return idx


def brute_rows(idx_list, E, W, align):
    """Rank r's receive rows as (source rank, token, slot) or None (padding), by loops."""
    epr = E // W
    out = []
    for r in range(W):
        rows = []
        for e in range(r * epr, (r + 1) * epr):
            n = 0
            for s, idx in enumerate(idx_list):
                for t in range(idx.shape[0]):
                    for j in range(idx.shape[1]):
                        if idx[t, j] == e:
                            rows.append((s, t, j))
                            n += 1
            while n % align:
                rows.append(None)
                n += 1
        out.append(rows)
    return out


@pytest.mark.parametrize("trial", range(12))
def test_bruteforce_rows_and_destinations(trial):
    rng = np.random.default_rng(100 + trial)
    W = [2, 3, 4][trial % 3]
    E = W * int(rng.integers(1, 4))
    k = int(rng.integers(1, min(E, 4) + 1))
    align = [1, 2, 4][trial % 3]
    idx_list = [random_ids(rng, int(rng.integers(0, 7)), k, E, unused=0.2, dup=0.2) for _ in range(W)]
    _, RL = MR.layout(idx_list, E, W, align)
    want = brute_rows(idx_list, E, W, align)
    for r in range(W):
        assert RL.recv_rows(r) == len(want[r])
    for s, idx in enumerate(idx_list):
        d = RL.destinations(s)
        for t in range(idx.shape[0]):
            for j in range(k):
                if idx[t, j] < 0:
                    assert tuple(d[t, j]) == (-1, -1)
                    continue
                owner = idx[t, j] // (E // W)
                assert d[t, j, 0] == owner
                assert want[owner][d[t, j, 1]] == (s, t, j)
    # the per-expert counts and segments each rank reports
    for r in range(W):
        seg = RL.recv_seg(r)
        for le in range(E // W):
            members = [x for x in want[r][seg[le]:seg[le + 1]] if x is not None]
            assert len(members) == RL.recv_counts(r)[le]
            assert all(idx_list[s][t, j] == r * (E // W) + le for s, t, j in members)


def test_single_rank_is_the_single_gpu_layout():
    rng = np.random.default_rng(5)
    idx = random_ids(rng, 40, 4, 16, unused=0.1)
    _, RL = MR.layout([idx], 16, 1, 2)
    _, L = oracle.layout(idx, 16, 1, 2)
    assert (RL.L.pos == L.pos).all() and RL.recv_rows(0) == L.seg[-1]
    assert (RL.destinations(0)[..., 1] == L.pos).all()


@pytest.mark.parametrize("W", [2, 4])
def test_identity_round_trip_is_exact(W):
    """BF16 dispatch, identity experts (y = received rows), weights summing to
    one: every source token comes back bit-exactly (the fp32 chain gives
    x(1 + d) with |d| far below half a bf16 ulp)."""
    rng = np.random.default_rng(W)
    E, k, H = 8 * W, 4, 64
    idx_list = [random_ids(rng, T, k, E) for T in (17, 5, 30, 1)[:W]]
    x_list = [torch.from_numpy(rng.standard_normal((i.shape[0], H))).to(torch.bfloat16) for i in idx_list]
    w_list = []
    for i in idx_list:
        w = rng.random((i.shape[0], k)).astype(np.float32) + 0.1
        w_list.append((w / w.sum(1, keepdims=True)).astype(np.float32))
    _, RL = MR.layout(idx_list, E, W)
    recv = MR.dispatch_bf16(RL, x_list)
    out = MR.combine(RL, recv, w_list)
    for s in range(W):
        assert (out[s] == oracle._u16(x_list[s])).all()


def test_padded_capacity_in_concatenated_token_order():
    # W = 2, E = 2 (one expert per rank).  Expert 0 is named by rank 0 tokens
    # 0, 1 and rank 1 tokens 0, 1: with capacity 4 they take rows 0..3 of rank
    # 0 in (source rank, token) order; with capacity 3 the concatenated count
    # 4 overflows and the layout reports it (positions are then unspecified).
    idx0 = np.array([[0], [0], [1]], np.int32)
    idx1 = np.array([[0], [0]], np.int32)
    st, RL = MR.layout([idx0, idx1], 2, 2, 1, 4)
    assert st == oracle.OR_OK
    assert RL.destinations(0)[:, 0].tolist() == [[0, 0], [0, 1], [1, 0]]
    assert RL.destinations(1)[:, 0].tolist() == [[0, 2], [0, 3]]
    assert RL.recv_rows(0) == RL.recv_rows(1) == 4
    assert RL.recv_counts(0).tolist() == [4] and RL.recv_counts(1).tolist() == [1]
    st, _ = MR.layout([idx0, idx1], 2, 2, 1, 3, check=False)
    assert st == oracle.OR_ERR_CAPACITY


def test_combine_backward_by_enumeration():
    """grad_y of the slot (s, t, j) sits on its owner at the row the brute-force
    enumeration gives it and equals bf16(fp32(w * g)); grad_w[s][t][j] is the
    dot product of g with that row of the owner's y (exact in binary64)."""
    rng = np.random.default_rng(21)
    W_, E, k, H = 3, 6, 2, 16
    idx_list = [random_ids(rng, T, k, E, unused=0.2) for T in (4, 0, 5)]
    _, RL = MR.layout(idx_list, E, W_)
    g_list = [torch.from_numpy(rng.standard_normal((i.shape[0], H))).to(torch.bfloat16) for i in idx_list]
    w_list = [rng.random(i.shape).astype(np.float32) for i in idx_list]
    y_list = [torch.from_numpy(rng.standard_normal((max(RL.recv_rows(r), 1), H))).to(torch.bfloat16)
              for r in range(W_)]
    gy, gw = MR.combine_backward(RL, g_list, y_list, w_list)
    want = brute_rows(idx_list, E, W_, 1)
    for r in range(W_):
        assert gy[r].shape[0] == RL.recv_rows(r)
        for row, who in enumerate(want[r]):
            s, t, j = who
            prod = torch.tensor(float(w_list[s][t, j]), dtype=torch.float32) * g_list[s][t].float()
            assert (gy[r][row] == oracle._u16(prod.to(torch.bfloat16))).all()
            dot = float((g_list[s][t].double() * y_list[r][row].double()).sum())
            assert abs(gw[s][t, j] - dot) <= 1e-12 * (1 + abs(dot))
    for s, idx in enumerate(idx_list):
        assert (gw[s][idx < 0] == 0).all()


def test_dispatch_topk_by_enumeration():
    """Every owner row's expert, weight, source rank and source slot are those
    of the (source rank, token, slot) the brute-force enumeration puts there;
    padding rows carry -1 / 0 / -1 / -1."""
    rng = np.random.default_rng(33)
    W_, E, k = 3, 9, 3
    idx_list = [random_ids(rng, T, k, E, unused=0.2, dup=0.2) for T in (5, 0, 7)]
    w_list = [rng.random(i.shape).astype(np.float32) for i in idx_list]
    _, RL = MR.layout(idx_list, E, W_, 2)
    got = MR.dispatch_topk(RL, idx_list, w_list)
    want = brute_rows(idx_list, E, W_, 2)
    for r in range(W_):
        ri, rw, rsrc, rslot = got[r]
        assert len(ri) == len(want[r])
        for row, who in enumerate(want[r]):
            if who is None:
                assert (ri[row], rw[row], rsrc[row], rslot[row]) == (-1, 0.0, -1, -1)
                continue
            s, t, j = who
            assert ri[row] == idx_list[s][t, j] and rw[row] == w_list[s][t, j]
            assert rsrc[row] == s and rslot[row] == t * k + j
