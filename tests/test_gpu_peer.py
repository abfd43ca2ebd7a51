"""Expert parallelism across ranks (plan, peer dispatch, peer combine) against
the multi-rank oracle, with the W ranks emulated on one GPU (GPU).

Every rank's buffers live on the one GPU, and each rank's kernels run in
turn on one stream: no kernel waits for another, so the emulation exercises
exactly the per-rank addressing of the multi-GPU path (plan rows, stores into
another rank's buffer, loads from another rank's outputs) without standing in
for concurrency.  Bars: bit-exact receive rows, scales, destinations,
segments and counts; combine bit-exact against the oracle's fma chain.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import multirank as MR
from combine_ep_layout_10_b200 import ep
from combine_ep_layout_10_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"
SENTINEL = 0x5A


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from combine_ep_layout_10_b200 import build
    build.build()
    ep.lib()
    oracle.lib()


def routing(name, Ts, seed0=0, unused=False, H=None):
    base = W.WORKLOADS[name]
    if H:
        base = base.scaled(H=H)
    idx_list, x_list, w_list = [], [], []
    for r, T in enumerate(Ts):
        w = base.scaled(T=T)
        x, idx, tw = W.make_routing(w, seed=seed0 + 17 * r)
        if unused and T:
            idx[::3, -1] = -1
        idx_list.append(idx)
        x_list.append(x)
        w_list.append(tw)
    return base, idx_list, x_list, w_list


class Emulated:
    """W ranks on one GPU: per-rank layouts, gathered counts, plans, buffers."""

    def __init__(self, E, k, H, idx_list, fp8, align=1, capacity=0, recv_rows=None):
        self.W = len(idx_list)
        self.E, self.k, self.H, self.fp8 = E, k, H, fp8
        total = sum(int(i.shape[0]) for i in idx_list)
        self.recv_rows = recv_rows or ep.ep_peer_max_recv_rows(total, k, E, self.W, align, capacity)
        rows = self.recv_rows
        dt = torch.uint8 if fp8 else torch.int16
        self.recv = [torch.full((rows, H), SENTINEL, dtype=dt, device=DEV) for _ in range(self.W)]
        self.scales = [torch.full((rows, H // 128), -1.0, dtype=torch.float32, device=DEV) for _ in range(self.W)] \
            if fp8 else None
        self.y = [torch.zeros(rows, H, dtype=torch.bfloat16, device=DEV) for _ in range(self.W)]
        self.grad_y = [torch.full((rows, H), SENTINEL, dtype=torch.int16, device=DEV) for _ in range(self.W)]
        self.peers = ep.Peers(self.W, self.recv, self.scales, self.y, rows, grad_y=self.grad_y)
        self.idx_dev = [i.to(DEV) for i in idx_list]
        self.layouts = [ep.ep_layout(i, E, self.W) for i in self.idx_dev]
        counts = torch.stack([l.num_tokens_per_expert for l in self.layouts])  # the all-gather
        self.plans = [ep.ep_plan_create(l.handle, i, counts, r, self.W, rows, align, capacity)
                      for r, (l, i) in enumerate(zip(self.layouts, self.idx_dev))]

    def dispatch(self, x_list, x_scales=None):
        for r in range(self.W):
            x = x_list[r].to(DEV)
            xs = x_scales[r].to(DEV) if x_scales is not None else None
            ep.ep_dispatch_peer(self.plans[r], self.peers, x, self.fp8, x_scales=xs)
        torch.cuda.synchronize()

    def combine(self, w_list):
        outs = [ep.ep_combine_peer(self.plans[r], self.peers, w_list[r].to(DEV) if w_list else None, self.H)
                for r in range(self.W)]
        torch.cuda.synchronize()
        return outs


def u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def check_plans(em, RL):
    for r in range(em.W):
        ex = em.plans[r].export()
        assert (ex["dst"].cpu().numpy() == RL.destinations(r)).all()
        assert (ex["recv_seg"].cpu().numpy() == RL.recv_seg(r)).all()
        assert (ex["recv_counts"].cpu().numpy() == RL.recv_counts(r)).all()
        assert em.plans[r].recv_rows_host() == RL.recv_rows(r)
        assert em.plans[r].check() == ep.EP_OK


def filled_rows(RL, r):
    b = RL.L.rank_off[r]
    return RL.L.src_idx[b:b + RL.recv_rows(r)] >= 0


@pytest.mark.parametrize("name,Ts,fp8,align,cap,unused,H", [
    ("tiny", [40, 0, 17, 64], False, 1, 0, True, None),          # W = 4, an empty rank
    ("tiny", [128, 128], False, 4, 0, False, None),              # alignment
    ("prefill", [64, 256, 33, 100, 5, 90, 1, 77], True, 1, 0, False, None),  # W = 8, FP8
    ("group_limited", [512, 300], True, 8, 0, True, None),       # W = 2, skewed, aligned
    ("decode", [128] * 8, True, 1, 128, False, 512),             # W = 8, padded (capacity)
])
def test_peer_dispatch_and_combine(name, Ts, fp8, align, cap, unused, H):
    base, idx_list, x_list, w_list = routing(name, Ts, unused=unused, H=H)
    Wr = len(Ts)
    em = Emulated(base.E, base.k, base.H, idx_list, fp8, align, cap)
    _, RL = MR.layout(idx_list, base.E, Wr, align, cap)
    check_plans(em, RL)
    em.dispatch(x_list)
    if fp8:
        want = MR.dispatch_fp8(RL, x_list)
    else:
        want = MR.dispatch_bf16(RL, x_list)
    for r in range(Wr):
        n = RL.recv_rows(r)
        f = filled_rows(RL, r)
        if fp8:
            q, s = want[r]
            got_q = em.recv[r][:n].cpu().numpy()
            got_s = em.scales[r][:n].cpu().numpy()
            assert (got_q[f] == q[f]).all()
            assert (got_s[f].view(np.uint32) == s[f].view(np.uint32)).all()
            assert (got_q[~f] == SENTINEL).all(), "rows no slot fills are not written"
        else:
            got = em.recv[r][:n].cpu().numpy().view(np.uint16)
            assert (got[f] == want[r][f]).all()
        assert (em.recv[r][n:].cpu().numpy() == SENTINEL).all()
    # combine: every rank's expert outputs, read back through the peer table
    ys = []
    for r in range(Wr):
        y = W.make_expert_out(em.recv_rows, base.H, seed=900 + r)
        em.y[r].copy_(y.to(DEV))
        ys.append(y)
    outs = em.combine(w_list)
    want_out = MR.combine(RL, ys, w_list)
    for r in range(Wr):
        assert (u16(outs[r]) == want_out[r]).all()
    # unit weights: the backward of the peer dispatch
    outs1 = em.combine(None)
    ones = [torch.ones(i.shape, dtype=torch.float32).numpy() for i in idx_list]
    want1 = MR.combine(RL, ys, ones)
    for r in range(Wr):
        assert (u16(outs1[r]) == want1[r]).all()


def test_peer_dispatch_prequantised_fp8():
    base, idx_list, x_list, _ = routing("prefill", [100, 60, 1, 31])
    em = Emulated(base.E, base.k, base.H, idx_list, True)
    qs = [oracle.quantize_rows(x) for x in x_list]
    em.dispatch([torch.from_numpy(q).view(torch.float8_e4m3fn) for q, _ in qs],
                x_scales=[torch.from_numpy(s) for _, s in qs])
    _, RL = MR.layout(idx_list, base.E, 4)
    want = MR.dispatch_fp8(RL, x_list)
    for r in range(4):
        n = RL.recv_rows(r)
        f = filled_rows(RL, r)
        assert (em.recv[r][:n].cpu().numpy()[f] == want[r][0][f]).all()
        assert (em.scales[r][:n].cpu().numpy()[f].view(np.uint32) == want[r][1][f].view(np.uint32)).all()


def test_receive_buffer_too_small_is_an_error_not_a_write():
    base, idx_list, x_list, _ = routing("group_limited", [256, 256])
    _, RL = MR.layout(idx_list, base.E, 2)
    need = max(RL.recv_rows(0), RL.recv_rows(1))
    em = Emulated(base.E, base.k, base.H, idx_list, True, recv_rows=need - 5)
    assert any(p.check() == ep.EP_ERR_CAPACITY for p in em.plans)
    em.dispatch(x_list)
    for r in range(2):
        # every row actually written is a correct row of the oracle; nothing past the buffer
        n = min(RL.recv_rows(r), em.recv_rows)
        f = filled_rows(RL, r)[:n]
        got = em.recv[r][:n].cpu().numpy()
        want = MR.dispatch_fp8(RL, x_list)[r][0][:n]
        written = (got != SENTINEL).any(1)
        assert (written == f).all(), "exactly the rows inside the buffer that slots fill are written"
        assert (got[f] == want[f]).all()


def test_capacity_overflow_across_ranks():
    # one expert per rank, capacity 2: rank 0's two slots of expert 0 fit,
    # rank 1's slot of expert 0 is the third and gets no row
    idx0 = torch.tensor([[0], [0]], dtype=torch.int32)
    idx1 = torch.tensor([[0], [1]], dtype=torch.int32)
    em = Emulated(2, 1, 128, [idx0, idx1], True, 1, 2)
    assert em.plans[0].check() == ep.EP_ERR_CAPACITY  # every rank sees the same counts
    d1 = em.plans[1].export()["dst"].cpu().numpy()
    assert d1[:, 0].tolist() == [[-1, -1], [1, 0]]
    d0 = em.plans[0].export()["dst"].cpu().numpy()
    assert d0[:, 0].tolist() == [[0, 0], [0, 1]]


def test_plan_argument_errors():
    base, idx_list, _, _ = routing("tiny", [16, 16])
    idx = idx_list[0].to(DEV)
    counts = torch.zeros(2, base.E, dtype=torch.int32, device=DEV)
    res_wrong_r = ep.ep_layout(idx, base.E, 4)
    with pytest.raises(ep.EpError):
        ep.ep_plan_create(res_wrong_r.handle, idx, torch.zeros(2, base.E, dtype=torch.int32, device=DEV),
                          0, 2, 64)
    res_aligned = ep.ep_layout(idx, base.E, 2, 4)
    with pytest.raises(ep.EpError):
        ep.ep_plan_create(res_aligned.handle, idx, counts, 0, 2, 64)
    res = ep.ep_layout(idx, base.E, 2)
    with pytest.raises(ep.EpError):
        ep.ep_plan_create(res.handle, idx, counts, 2, 2, 64)  # rank out of range
    bad = torch.empty(64 * base.H + 8, dtype=torch.int16, device=DEV)[1:]
    with pytest.raises(ep.EpError):
        ep.Peers(2, [bad, bad], None, None, 64)  # misaligned buffer


@pytest.mark.parametrize("name,Ts,align,H", [("prefill", [64, 30, 0, 100], 1, None),
                                             ("group_limited", [300, 212], 8, None),
                                             ("tiny", [64, 64], 4, 1000)])
def test_peer_combine_backward(name, Ts, align, H):
    """grad_y rows land bit-exactly on their owners; grad_w equals the local
    kernel's on the concatenated layout bit for bit (the same per-token
    reduction order) and the oracle within the derived bound."""
    import math
    base, idx_list, _, w_list = routing(name, Ts, unused=True, H=H)
    Wr = len(Ts)
    em = Emulated(base.E, base.k, base.H, idx_list, False, align)
    _, RL = MR.layout(idx_list, base.E, Wr, align)
    ys = []
    for r in range(Wr):
        y = W.make_expert_out(em.recv_rows, base.H, seed=500 + r)
        em.y[r].copy_(y.to(DEV))
        ys.append(y)
    gos = [W.make_x(base.scaled(T=T), 600 + r) for r, T in enumerate(Ts)]
    gws = [ep.ep_combine_backward_peer(em.plans[r], em.peers, gos[r].to(DEV), w_list[r].to(DEV))
           for r in range(Wr)]
    torch.cuda.synchronize()
    want_gy, want_gw = MR.combine_backward(RL, gos, ys, w_list)
    for r in range(Wr):
        n = RL.recv_rows(r)
        f = filled_rows(RL, r)
        got = em.grad_y[r][:n].cpu().numpy().view(np.uint16)
        assert (got[f] == want_gy[r][f]).all()
        assert (em.grad_y[r][:n].cpu().numpy()[~f] == SENTINEL).all()
    # the local kernel on the concatenated batch
    idx_cat = torch.cat(idx_list)
    res = ep.ep_layout(idx_cat.to(DEV), base.E, Wr, align)
    y_cat = torch.zeros(res.handle.num_recv_rows, base.H, dtype=torch.bfloat16)
    for r in range(Wr):
        n = RL.recv_rows(r)
        y_cat[RL.L.rank_off[r]:RL.L.rank_off[r] + n] = ys[r][:n]
    _, gw_cat = ep.ep_combine_backward(res.handle, torch.cat(gos).to(DEV), torch.cat(w_list).to(DEV),
                                       y=y_cat.to(DEV))
    gw_cat = gw_cat.cpu()
    for r in range(Wr):
        b, T = RL.token_base[r], RL.T[r]
        assert torch.equal(gws[r].cpu(), gw_cat[b:b + T])
        g64 = gos[r].double().numpy()
        bound = (16 * math.ceil(base.H / 2048) + 37) * 2.0 ** -24
        d = RL.destinations(r)
        for t in range(T):
            for j in range(base.k):
                if d[t, j, 0] < 0:
                    assert gws[r][t, j].item() == 0.0
                    continue
                yrow = ys[d[t, j, 0]][d[t, j, 1]].double().numpy()
                lim = bound * np.abs(g64[t] * yrow).sum() + 1e-30
                assert abs(float(gws[r][t, j]) - want_gw[r][t, j]) <= lim


def test_metric_batch_over_eight_ranks_sampled():
    """The benchmark's batch split over 8 emulated ranks of 1,024 tokens:
    every slot's (owner, row) exactly the oracle's, every rank's segments and
    counts too; FP8 rows and combined outputs exact on a sample of tokens
    the oracle computes one by one."""
    base = W.WORKLOADS["group_limited"]
    Wr, Tr = 8, base.T // 8
    parts = [W.make_routing(base.scaled(T=Tr), seed=7000 + r) for r in range(Wr)]
    x_list = [p[0] for p in parts]
    idx_list = [p[1] for p in parts]
    w_list = [p[2] for p in parts]
    em = Emulated(base.E, base.k, base.H, idx_list, True)
    _, RL = MR.layout(idx_list, base.E, Wr)
    check_plans(em, RL)
    em.dispatch(x_list)
    gy = torch.Generator(device=DEV).manual_seed(910)
    for r in range(Wr):   # expert outputs drawn on the device; the checks read them back
        em.y[r].copy_(torch.randn(em.recv_rows, base.H, generator=gy, device=DEV).to(torch.bfloat16))
    outs = em.combine(w_list)
    g = torch.Generator().manual_seed(12)
    for s in range(Wr):
        d = RL.destinations(s)
        sample = torch.randperm(Tr, generator=g)[:8].tolist() + ([0, Tr - 1] if s in (0, Wr - 1) else [])
        for t in sample:
            q1, s1 = oracle.dispatch_fp8(x_list[s][t:t + 1], np.zeros((1, 1), np.int32), 1)
            rows = []
            for j in range(base.k):
                o, row = int(d[t, j, 0]), int(d[t, j, 1])
                assert (em.recv[o][row].cpu().numpy() == q1[0]).all()
                assert (em.scales[o][row].cpu().numpy().view(np.uint32) == s1[0].view(np.uint32)).all()
                rows.append(em.y[o][row].cpu())
            want = oracle.combine(torch.stack(rows), w_list[s][t:t + 1].numpy(),
                                  np.arange(base.k, dtype=np.int32)[None, :])
            assert (u16(outs[s][t:t + 1]) == want).all()


@pytest.mark.parametrize("name,Ts,align,cap", [("tiny", [40, 0, 17, 64], 4, 0),
                                               ("prefill", [64, 30, 0, 100], 1, 0),
                                               ("decode", [128] * 8, 1, 128)])
def test_peer_dispatch_topk(name, Ts, align, cap):
    """Per-row outputs on the owners: expert, weight, source rank and slot of
    every received row exactly the oracle's; padding rows -1 / 0 / -1 / -1;
    rows past the received ones untouched."""
    base, idx_list, _, w_list = routing(name, Ts, unused=True, H=512 if name == "decode" else None)
    Wr = len(Ts)
    em = Emulated(base.E, base.k, base.H, idx_list, False, align, cap)
    rows = em.recv_rows
    t_idx = [torch.full((rows,), -7, dtype=torch.int32, device=DEV) for _ in range(Wr)]
    t_w = [torch.full((rows,), -7.0, dtype=torch.float32, device=DEV) for _ in range(Wr)]
    t_src = [torch.full((rows,), -7, dtype=torch.int32, device=DEV) for _ in range(Wr)]
    t_slot = [torch.full((rows,), -7, dtype=torch.int32, device=DEV) for _ in range(Wr)]
    em.peers.set_topk(t_idx, t_w, t_src, t_slot)
    for r in range(Wr):
        ep.ep_dispatch_topk_peer(em.plans[r], em.peers, em.idx_dev[r], w_list[r].to(DEV))
    torch.cuda.synchronize()
    _, RL = MR.layout(idx_list, base.E, Wr, align, cap)
    want = MR.dispatch_topk(RL, idx_list, w_list)
    for r in range(Wr):
        n = RL.recv_rows(r)
        wi, ww, ws, wsl = want[r]
        assert (t_idx[r][:n].cpu().numpy() == wi).all()
        assert (t_w[r][:n].cpu().numpy().view(np.uint32) == ww.view(np.uint32)).all()
        assert (t_src[r][:n].cpu().numpy() == ws).all()
        assert (t_slot[r][:n].cpu().numpy() == wsl).all()
        for t in (t_idx, t_src, t_slot):
            assert (t[r][n:].cpu().numpy() == -7).all()
        assert (t_w[r][n:].cpu().numpy() == -7.0).all()


def test_peer_dispatch_column_major_scales():
    """FP8 scales written column-major ([H/128, ld] per owner, the FP8 grouped
    GEMM layout) hold exactly the row-major scales, transposed; padding
    columns and the columns past the received rows stay untouched."""
    base, idx_list, x_list, _ = routing("prefill", [100, 0, 57, 31])
    Wr, H = 4, base.H
    em = Emulated(base.E, base.k, H, idx_list, True)
    rows = em.recv_rows
    ld = (rows + 3) // 4 * 4
    cols = [torch.full((H // 128, ld), -3.0, dtype=torch.float32, device=DEV) for _ in range(Wr)]
    peers = ep.Peers(Wr, em.recv, cols, None, rows)
    for r in range(Wr):
        ep.ep_dispatch_peer(em.plans[r], peers, x_list[r].to(DEV), True, scale_layout="col", scale_ld=ld)
    torch.cuda.synchronize()
    _, RL = MR.layout(idx_list, base.E, Wr)
    want = MR.dispatch_fp8(RL, x_list)
    for r in range(Wr):
        n = RL.recv_rows(r)
        f = filled_rows(RL, r)
        got = cols[r].cpu().numpy()
        assert (got[:, :n].T[f].view(np.uint32) == want[r][1][f].view(np.uint32)).all()
        assert (got[:, :n].T[~f] == -3.0).all() and (got[:, n:] == -3.0).all()
        assert (em.recv[r][:n].cpu().numpy()[f] == want[r][0][f]).all()
    # a scale layout that would overlap is refused on the host
    with pytest.raises(ep.EpError):
        ep.ep_dispatch_peer(em.plans[0], peers, x_list[0].to(DEV), True, scale_layout="col", scale_ld=ld - 8)


@pytest.mark.parametrize("num_sms,H,fp8", [(1, None, True), (7, None, True), (3, 8192 + 128, True),
                                            (3, 8192 + 128, False)])
def test_peer_sm_budget_changes_nothing(num_sms, H, fp8):
    """The SM budget changes the peer kernels' launch shape, never the result
    (FP8 and BF16; two chunks per token at H = 8320, so that the pipelined
    grid-stride kernels walk both chunk positions)."""
    base, idx_list, x_list, w_list = routing("group_limited", [300, 128, 77, 40], H=H)
    Wr = 4
    em = Emulated(base.E, base.k, base.H, idx_list, fp8)
    em.dispatch(x_list)
    ref_q = [r.clone() for r in em.recv]
    ref_s = [s.clone() for s in em.scales] if fp8 else None
    for r in em.recv:
        r.fill_(SENTINEL)
    for r in range(Wr):
        ep.ep_dispatch_peer(em.plans[r], em.peers, x_list[r].to(DEV), fp8, num_sms=num_sms)
    gy = torch.Generator(device=DEV).manual_seed(5)
    for r in range(Wr):
        em.y[r].copy_(torch.randn(em.recv_rows, base.H, generator=gy, device=DEV).to(torch.bfloat16))
    outs0 = [ep.ep_combine_peer(em.plans[r], em.peers, w_list[r].to(DEV), base.H) for r in range(Wr)]
    outs1 = [ep.ep_combine_peer(em.plans[r], em.peers, w_list[r].to(DEV), base.H, num_sms=num_sms)
             for r in range(Wr)]
    torch.cuda.synchronize()
    for r in range(Wr):
        assert torch.equal(em.recv[r], ref_q[r])
        if fp8:
            assert torch.equal(em.scales[r], ref_s[r])
        assert torch.equal(outs0[r].view(torch.int16), outs1[r].view(torch.int16))
