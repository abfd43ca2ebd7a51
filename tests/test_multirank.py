"""The N>1 path of bench.py on CPU: world size 2 over gloo.

The path does not shard across GPUs (one GPU's expert-parallel ranks are
virtual), so `bench.py --gpus N` runs N independent replicas.  What needs
checking is the host logic around them: every replica draws its own batch,
and the job's throughput is all replicas' bytes over the slowest replica's
time.  Each replica here runs the oracle path on its batch (CPU only).
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


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import oracle
        from combine_ep_layout_10_b200 import workloads as W
        w = W.WORKLOADS["tiny"]
        seed = bench.replica_seed(0, rank)
        x, idx, tw = W.make_routing(w, seed)
        _, L = oracle.layout(idx.numpy(), w.E, w.R)
        recv = oracle.dispatch_bf16(x, L.pos, L.n_rows)
        out = oracle.combine(recv, tw.numpy(), L.pos)
        xs = x.view(torch.int16).numpy().view(np.uint16)
        nz = (xs & 0x7FFF) != 0
        roundtrip_ok = bool((out[nz] == xs[nz]).all())
        local_ms = 1.0 + rank          # a slower rank 1
        value, step_ms = bench.job_throughput(local_ms, 1000.0, 10, world)
        q.put((rank, value, step_ms, int(idx.sum()), roundtrip_ok))
    finally:
        dist.destroy_process_group()


def test_two_replicas_over_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    (_, v0, ms0, s0, ok0), (_, v1, ms1, s1, ok1) = res
    assert ok0 and ok1
    assert s0 != s1, "replicas must draw different batches"
    assert ms0 == ms1 == 2.0, "job time is the slowest rank's"
    want = (1000.0 * 10 * world) / (2.0 * 10 / 1e3) / 1e9
    assert v0 == pytest.approx(want) and v1 == pytest.approx(want)


def test_single_process_helpers():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    v, ms = bench.job_throughput(0.5, 2e6, 4, 1)
    assert ms == 0.5 and v == pytest.approx(2e6 * 4 / (0.5 * 4 / 1e3) / 1e9)
    assert bench.replica_seed(7, 3) == 10
