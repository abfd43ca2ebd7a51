"""The multi-GPU protocol end to end in separate processes (GPU).

Two ranks of an EpGroup, each its own process with its own CUDA context,
share their receive / scale / expert-output buffers through CUDA IPC and
order each other's stores and loads with gloo collectives -- the host logic
of the multi-GPU path (handle exchange, count all-gather, plan, barriers,
cached plan, release).  Both processes use the one GPU of this machine: no
kernel waits on the other process (every ordering point is a host
collective), so nothing depends on the two contexts running at once.
Results are compared bit-exactly with the multi-rank oracle.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TOKENS = [200, 131]


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q, backend="gloo", scale_layout="row"):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    kw = {"device_id": torch.device("cuda", 0)} if backend == "nccl" else {}
    dist.init_process_group(backend, rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60), **kw)
    result = {"rank": rank, "error": None}
    try:
        torch.cuda.set_device(0)
        from oracle import multirank as MR
        from combine_ep_layout_10_b200 import ep, group
        from combine_ep_layout_10_b200 import workloads as W
        base = W.WORKLOADS["prefill"]
        E, H, k = base.E, base.H, base.k
        tokens = TOKENS[:world]
        routed = [W.make_routing(base.scaled(T=T), seed=50 + r) for r, T in enumerate(tokens)]
        x_list = [r[0] for r in routed]
        idx_list = [r[1] for r in routed]
        w_list = [r[2] for r in routed]
        recv_rows = ep.ep_peer_max_recv_rows(sum(tokens), k, E, world)
        g = group.EpGroup(E, H, recv_rows, fp8=True, scale_layout=scale_layout)
        _, RL = MR.layout(idx_list, E, world)
        n = RL.recv_rows(rank)
        filled = RL.L.src_idx[RL.L.rank_off[rank]:RL.L.rank_off[rank] + n] >= 0

        def check_recv(xs):
            q_want, s_want = MR.dispatch_fp8(RL, xs)[rank]
            got_q = g.recv_x[:n].view(torch.uint8).cpu().numpy()
            got_s = (g.recv_scales[:n] if scale_layout == "row" else g.recv_scales[:, :n].T).cpu().numpy()
            return bool((got_q[filled] == q_want[filled]).all()
                        and (got_s[filled].view(np.uint32) == s_want[filled].view(np.uint32)).all())

        plan = g.dispatch(x_list[rank].cuda(), idx_list[rank].cuda(), topk_weights=w_list[rank].cuda())
        torch.cuda.synchronize()
        result["dispatch"] = check_recv(x_list)
        wi, ww, wsrc, wslot = MR.dispatch_topk(RL, idx_list, w_list)[rank]
        result["topk"] = bool((g.recv_topk_idx[:n].cpu().numpy() == wi).all()
                              and (g.recv_topk_weights[:n].cpu().numpy().view(np.uint32) == ww.view(np.uint32)).all()
                              and (g.recv_src_rank[:n].cpu().numpy() == wsrc).all()
                              and (g.recv_slot[:n].cpu().numpy() == wslot).all())
        result["rows"] = plan.recv_rows_host() == n
        ys = [W.make_expert_out(recv_rows, H, seed=900 + r) for r in range(world)]
        g.y.copy_(ys[rank].cuda())
        out = g.combine(plan, w_list[rank].cuda())
        torch.cuda.synchronize()
        want = MR.combine(RL, ys, w_list)[rank]
        result["combine"] = bool((out.view(torch.int16).cpu().numpy().view(np.uint16) == want).all())
        # second step: same routing (cached plan), new hidden states
        x2 = [W.make_x(base.scaled(T=T), 1000 + r) for r, T in enumerate(tokens)]
        g.dispatch(x2[rank].cuda(), plan=plan)
        torch.cuda.synchronize()
        result["cached"] = check_recv(x2)
        # backward: combine's (gradient rows to the owners), then dispatch's
        gos = [W.make_x(base.scaled(T=T), 2000 + r) for r, T in enumerate(tokens)]
        gw = g.combine_backward(plan, gos[rank].cuda(), w_list[rank].cuda())
        torch.cuda.synchronize()
        want_gy, want_gw = MR.combine_backward(RL, gos, ys, w_list)
        got_gy = g.grad_y[:n].view(torch.int16).cpu().numpy().view(np.uint16)
        scale = np.abs(gos[rank].double().numpy()).sum(1, keepdims=True) * 8.0
        result["combine_bwd"] = bool((got_gy[filled] == want_gy[rank][filled]).all()
                                     and (np.abs(gw.cpu().numpy() - want_gw[rank]) <= 1e-4 * scale).all())
        grs = [W.make_expert_out(recv_rows, H, seed=3000 + r) for r in range(world)]
        g.y.copy_(grs[rank].cuda())     # this rank's receive-row gradients
        gx = g.dispatch_backward(plan)
        torch.cuda.synchronize()
        ones = [np.ones(i.shape, np.float32) for i in idx_list]
        want_gx = MR.combine(RL, grs, ones)[rank]
        result["dispatch_bwd"] = bool((gx.view(torch.int16).cpu().numpy().view(np.uint16) == want_gx).all())
        g.close()
        plan.free()
    except Exception as e:  # reported to the parent, which fails the test
        result["error"] = repr(e)
    finally:
        q.put(result)
        dist.destroy_process_group()


def _run(world, backend, scale_layout="row"):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from combine_ep_layout_10_b200 import build
    build.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, backend, scale_layout)) for r in range(world)]
    for p in procs:
        p.start()
    results = []
    try:
        for _ in range(world):
            results.append(q.get(timeout=300))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    for r in sorted(results, key=lambda d: d["rank"]):
        assert r["error"] is None, r
        assert r["dispatch"] and r["rows"] and r["combine"] and r["cached"], r
        assert r["combine_bwd"] and r["dispatch_bwd"] and r["topk"], r


def test_two_processes_share_buffers_over_ipc():
    _run(2, "gloo")


def test_single_rank_group_over_nccl():
    """The NCCL branch of EpGroup (device-ordered all-reduce barriers and the
    all_gather_into_tensor of the counts) with one rank, whose peer table is
    its own buffers; FP8 scales in the column-major (grouped-GEMM) layout."""
    _run(1, "nccl", "col")
