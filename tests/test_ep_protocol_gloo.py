"""The host protocol of expert parallelism across ranks, on CPU over gloo.

Across GPUs every rank knows only its own tokens.  The protocol the library
runs (combine_ep_layout_10_b200/group.py with the plan, peer dispatch and peer
combine kernels) is:

  1. the local layout of the rank's own ids over W ranks (per-expert counts,
     positions in token order);
  2. an all-gather of the per-expert counts of every rank;
  3. the plan: from its own positions and the gathered counts alone, each
     rank derives the (owner rank, row) of each of its slots;
  4. dispatch: rows stored into the owners' receive buffers; combine: each
     source rank reads its slots' rows back and reduces them.

Here the ranks are gloo processes and the stores and loads are object
all-gathers, so the protocol runs with no GPU.  The plan rule is restated
in numpy from its definition: inside expert e's segment on its owner, the
slots of source rank s start after those of ranks s' < s, and each keeps its
token order.  The receive buffers and combined outputs that every rank ends
up with must equal the multi-rank oracle, which builds the same result from
all ranks' tokens at once (the single-GPU layout of their concatenation,
sliced by owner).
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(s, T, k, E, H):
    """Rank s's ids (unused slots and duplicates included), bf16 x, weights."""
    rng = np.random.default_rng(1000 + s)
    idx = rng.integers(-1, E, (T, k)).astype(np.int32)
    x = torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)).to(torch.bfloat16)
    w = rng.random((T, k)).astype(np.float32)
    return idx, x.view(torch.int16).numpy().view(np.uint16), w


def _expert_out(o, rows, H):
    """Owner o's expert outputs, bf16 bits [rows, H]."""
    rng = np.random.default_rng(2000 + o)
    y = torch.from_numpy(rng.standard_normal((rows, H)).astype(np.float32)).to(torch.bfloat16)
    return y.view(torch.int16).numpy().view(np.uint16)


def plan_rule(pos, seg, idx, counts, s, W, align, capacity):
    """(owner, row) of every local slot from the local layout (pos, seg over
    W ranks, alignment 1, packed) and the gathered counts [W, E]; (-1, -1)
    for unused slots and slots past a padded expert's capacity."""
    E = counts.shape[1]
    epr = E // W
    total = counts.sum(axis=0)
    before = counts[:s].sum(axis=0)                  # slots of each expert on ranks < s
    start = np.zeros(E, np.int64)                    # expert segment start in its owner's buffer
    for o in range(W):
        run = 0
        for le in range(epr):
            e = o * epr + le
            start[e] = le * capacity if capacity else run
            run += -(-int(total[e]) // align) * align
    dest = np.full(idx.shape + (2,), -1, np.int32)
    for t in range(idx.shape[0]):
        for j in range(idx.shape[1]):
            e = idx[t, j]
            if e < 0:
                continue
            i = int(before[e]) + int(pos[t, j] - seg[e])     # index among all ranks' slots of e
            if capacity and i >= capacity:
                continue
            dest[t, j] = (e // epr, start[e] + i)
    return dest


def _worker(rank, W, port, cfg, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=W, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from oracle import multirank as MR
        Ts, k, E, H, align, capacity = cfg["T"], cfg["k"], cfg["E"], cfg["H"], cfg["align"], cfg["capacity"]
        epr = E // W
        idx, x, w = _inputs(rank, Ts[rank], k, E, H)

        # 1-2: local layout, all-gather of the per-expert counts
        _, L = oracle.layout(idx, E, W, 1, 0)
        c = torch.from_numpy(L.num_tokens_per_expert.astype(np.int64))
        parts = [torch.empty_like(c) for _ in range(W)]
        dist.all_gather(parts, c)
        counts = torch.stack(parts).numpy()

        # 3: the plan from local knowledge only
        dest = plan_rule(L.pos, L.seg, idx, counts, rank, W, align, capacity)
        total = counts.sum(axis=0)
        mine = total[rank * epr:(rank + 1) * epr]
        recv_rows = epr * capacity if capacity else int(sum(-(-int(n) // align) * align for n in mine))

        # 4a: dispatch -- every rank's (owner, row, x row) stores, delivered to the owners
        sends = [(int(dest[t, j, 0]), int(dest[t, j, 1]), x[t]) for t in range(idx.shape[0])
                 for j in range(k) if dest[t, j, 0] >= 0]
        got = [None] * W
        dist.all_gather_object(got, sends)
        recv = np.zeros((recv_rows, H), np.uint16)
        filled = np.zeros(recv_rows, bool)
        for stores in got:
            for o, row, data in stores:
                if o == rank:
                    assert not filled[row], "two slots stored into one row"
                    recv[row] = data
                    filled[row] = True

        # 4b: combine -- every owner exposes its expert outputs, each source
        # rank loads its slots' rows and reduces them in slot order
        y = _expert_out(rank, recv_rows, H)
        ys = [None] * W
        dist.all_gather_object(ys, y)
        flat_pos = np.where(dest[..., 0] >= 0, np.arange(idx.size).reshape(idx.shape), -1).astype(np.int32)
        gathered = np.zeros((max(idx.size, 1), H), np.uint16)
        for t in range(idx.shape[0]):
            for j in range(k):
                if dest[t, j, 0] >= 0:
                    gathered[t * k + j] = ys[dest[t, j, 0]][dest[t, j, 1]]
        out = oracle.combine(gathered[:idx.size], w, flat_pos)

        # the oracle, from every rank's inputs at once
        all_in = [_inputs(s, Ts[s], k, E, H) for s in range(W)]
        st, RL = MR.layout([a[0] for a in all_in], E, W, align, capacity, check=False)
        want_recv = MR.dispatch_bf16(RL, [a[1] for a in all_in])[rank]
        want_out = MR.combine(RL, [_expert_out(o, RL.recv_rows(o), H) for o in range(W)],
                              [a[2] for a in all_in])[rank]
        # an over-capacity expert keeps its first `capacity` slots in
        # concatenated (rank, token, slot) order; the oracle reports it
        overflow = bool((total > capacity).any()) if capacity else False
        q.put((rank, dict(
            rows=(recv_rows, RL.recv_rows(rank)),
            dest=bool((dest == RL.destinations(rank)).all()),
            recv=bool((recv[filled] == want_recv[filled]).all()) and bool((want_recv[~filled] == 0).all()),
            filled=int(filled.sum()),
            out=bool((out == want_out).all()),
            overflow=overflow, oracle_status=int(st))))
    except Exception as exc:  # report instead of hanging the other rank's collectives
        q.put((rank, {"error": repr(exc)}))
        raise
    finally:
        dist.destroy_process_group()


CASES = {
    "packed_align4_w2": dict(W=2, T=[37, 20], k=4, E=16, H=16, align=4, capacity=0, overflow=False),
    "packed_w3_empty_rank": dict(W=3, T=[25, 0, 31], k=3, E=12, H=8, align=1, capacity=0, overflow=False),
    "padded_w2": dict(W=2, T=[40, 40], k=4, E=8, H=8, align=1, capacity=48, overflow=False),
    "padded_overflow_w2": dict(W=2, T=[40, 40], k=4, E=8, H=8, align=1, capacity=16, overflow=True),
}


@pytest.mark.parametrize("name", list(CASES))
def test_protocol_over_gloo_matches_the_multirank_oracle(name):
    cfg = CASES[name]
    W = cfg["W"]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, W, port, cfg, q)) for r in range(W)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in range(W))
    for p in procs:
        p.join(timeout=60)
    for r in range(W):
        assert "error" not in res[r], res[r]
        assert procs[r].exitcode == 0
    for r in range(W):
        d = res[r]
        # every rank sees the overflow the oracle reports, in the gathered counts
        assert d["overflow"] == cfg["overflow"] and (d["oracle_status"] != 0) == cfg["overflow"]
        assert d["rows"][0] == d["rows"][1]
        assert d["dest"] and d["recv"] and d["out"]
    assert sum(res[r]["filled"] for r in range(W)) > 0
