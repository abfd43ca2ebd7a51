"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bars: layout, indices, FP8 codes and scales bit-exact; BF16 combine within
1 bf16 ulp (ordered-bit distance, +0 == -0) -- and, since both sides run the
same fp32 fma chain in slot order, bit-exact as well.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_ep_layout_10_b200 import ep
from combine_ep_layout_10_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from combine_ep_layout_10_b200 import build
    build.build()
    ep.lib()
    oracle.lib()


def u8(t):
    return t.contiguous().view(torch.uint8).cpu().numpy()


def u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_ulp_distance(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    def ordered(x):
        x = x.astype(np.int64)
        mag = x & 0x7FFF
        return np.where(x & 0x8000, -mag, mag)
    return np.abs(ordered(a) - ordered(b))


def run_layout(idx_cpu, E, R, align=1, capacity=0):
    res = ep.ep_layout(idx_cpu.to(DEV), E, R, align, capacity)
    md = res.handle.export()
    torch.cuda.synchronize()
    return res, md


def assert_layout_equal(res, md, L):
    assert (res.num_tokens_per_expert.cpu().numpy() == L.num_tokens_per_expert).all()
    assert (res.num_tokens_per_rank.cpu().numpy() == L.num_tokens_per_rank).all()
    assert (res.is_token_in_rank.cpu().numpy() == L.is_token_in_rank).all()
    assert (md["seg"].cpu().numpy() == L.seg).all()
    assert (md["rank_off"].cpu().numpy() == L.rank_off).all()
    assert (md["pos"].cpu().numpy() == L.pos).all()
    assert (md["src_idx"].cpu().numpy() == L.src_idx).all()


# --- layout ------------------------------------------------------------------

@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_layout_full_workloads(name):
    w = W.WORKLOADS[name]
    _, idx, _ = W.make_routing(w)
    res, md = run_layout(idx, w.E, w.R, w.align, w.capacity)
    _, L = oracle.layout(idx.numpy(), w.E, w.R, w.align, w.capacity)
    assert_layout_equal(res, md, L)
    assert res.handle.check() == ep.EP_OK
    assert res.handle.counts_host() == L.num_tokens_per_expert.tolist()


LAYOUT_EDGE = [
    # (T, k, E, R, align, capacity, id_low)  id_low=-1 adds unused slots
    (1, 1, 1, 1, 1, 0, 0),
    (1, 8, 256, 64, 1, 0, 0),
    (129, 8, 256, 8, 1, 0, 0),        # one full tile + ragged tail
    (300, 3, 16, 4, 1, 0, -1),        # unused slots, duplicates
    (1000, 8, 64, 64, 4, 0, -1),      # R == E, alignment 4
    (777, 4, 32, 1, 2, 0, 0),         # R == 1
    (513, 2, 8, 2, 1, 256, 0),        # padded, fits
    (70000, 2, 64, 16, 1, 0, -1),     # > 512 tiles of 128: larger tiles
    (64, 32, 4096, 4096, 1, 0, -1),   # maximum k, E, R
    (2048, 6, 96, 12, 8, 0, -1),      # E not a power of two
    (5000, 2, 16, 4, 1, 1024, 0),     # padded, tiled path (more than 8192 slots)
    (1537, 1, 8, 2, 1, 0, -1),        # one slot past the packed one-CTA limit
    (1536, 1, 8, 2, 1, 0, -1),        # exactly at the packed one-CTA limit
    (2048, 8, 256, 64, 1, 0, -1),     # 16K slots: 16 tiles, position kernel at 512 threads
    (1000, 8, 2048, 2048, 1, 0, -1),  # tiles doubled to 2K slots: position kernel at 1024 threads
    (1024, 8, 256, 64, 1, 0, -1),     # 8K slots packed: tiled
    (8193, 1, 8, 2, 1, 2048, 0),      # one slot past the padded one-CTA limit
    (8192, 1, 8, 2, 1, 2048, 0),      # exactly at the padded one-CTA limit
    (9000, 2, 96, 48, 1, 0, -1),      # tiled, 16-flag vectors across mask-word halves
]


@pytest.mark.parametrize("case", LAYOUT_EDGE)
def test_layout_edge_cases(case):
    T, k, E, R, A, C, low = case
    g = torch.Generator().manual_seed(T * 131 + k)
    idx = torch.randint(low, E, (T, k), generator=g, dtype=torch.int32)
    if C:
        # keep every expert within capacity
        idx = (torch.arange(T * k, dtype=torch.int32) % E).reshape(T, k)
    res, md = run_layout(idx, E, R, A, C)
    st, L = oracle.layout(idx.numpy(), E, R, A, C)
    assert st == 0
    assert_layout_equal(res, md, L)
    assert res.handle.check() == ep.EP_OK
    h = res.handle
    if _one_cta_layout(T, k, E, R, C):
        assert h.layout_path == ep.EP_LAYOUT_PATH_ONE_CTA and h.layout_kernels == 1
    else:
        assert h.layout_path == ep.EP_LAYOUT_PATH_TILED
        assert h.layout_kernels == (2 if h.layout_path == ep.EP_LAYOUT_PATH_TILED else 1)


def _one_cta_layout(T, k, E, R, C):
    """The stated rule for the one-CTA layout: at most 1536 slots packed or
    8192 padded, at most 512 experts, and its shared-memory plan within
    40000 words (ids, counts, offsets, per-warp histograms, in-rank masks)."""
    a4 = lambda n: (n + 3) // 4 * 4  # noqa: E731
    words = a4(T * k) + a4(E) + a4(E + 1) + a4(R) + 32 * (E + 1) + T * ((R + 31) // 32)
    return 0 < T * k <= (8192 if C else 1536) and E <= 512 and words <= 40000


def test_layout_empty():
    idx = torch.zeros(0, 8, dtype=torch.int32)
    for C in (0, 4):
        res, md = run_layout(idx, 16, 4, 1, C)
        _, L = oracle.layout(idx.numpy(), 16, 4, 1, C)
        assert_layout_equal(res, md, L)
        assert res.handle.layout_kernels == 1 and res.handle.layout_path == ep.EP_LAYOUT_PATH_EMPTY


def test_layout_bad_expert_id_reported():
    idx = torch.tensor([[0, 1], [2, 99], [-3, 1]], dtype=torch.int32)
    res = ep.ep_layout(idx.to(DEV), 4, 2)
    assert res.handle.check() == ep.EP_ERR_BAD_EXPERT_ID
    # the valid slots still get a consistent layout; the bad ones none
    pos = res.handle.export()["pos"].cpu().numpy()
    assert pos[1, 1] == -1 and pos[2, 0] == -1
    # ... and the whole layout is the oracle's, which takes a bad id as an unused slot
    st, L = oracle.layout(idx.numpy(), 4, 2, check=False)
    assert st == 2
    assert_layout_equal(res, res.handle.export(), L)


@pytest.mark.parametrize("T,k,C,bad", [(10, 1, 4, False), (700, 8, 16, True), (9000, 1, 4, False),
                                       (5000, 2, 64, True)])
def test_layout_data_errors_match_the_oracle(T, k, C, bad):
    """Padded overflow (an expert keeps its first `capacity` slots in (token,
    slot) order) and invalid ids (unused slots), on the one-CTA and the tiled
    path: the complete layout equals the oracle's and the status is the same."""
    E, R = 16, 4
    g = torch.Generator().manual_seed(T + k)
    idx = torch.randint(-1, E, (T, k), generator=g, dtype=torch.int32)
    idx[: T // 2, 0] = 3                      # expert 3 overflows
    if bad:
        idx[T // 3, k - 1] = E + 5
        idx[T - 1, 0] = -7
    res, md = run_layout(idx, E, R, 1, C)
    st, L = oracle.layout(idx.numpy(), E, R, 1, C, check=False)
    assert st == (2 if bad else 3)
    assert res.handle.check() == (ep.EP_ERR_BAD_EXPERT_ID if bad else ep.EP_ERR_CAPACITY)
    assert_layout_equal(res, md, L)


def test_layout_errors_on_tiled_path():
    g = torch.Generator().manual_seed(5)
    idx = torch.randint(0, 16, (4096, 4), generator=g, dtype=torch.int32)
    idx[1000, 2] = 16
    res = ep.ep_layout(idx.to(DEV), 16, 4)
    assert res.handle.check() == ep.EP_ERR_BAD_EXPERT_ID
    assert res.handle.export()["pos"].cpu().numpy()[1000, 2] == -1
    over = torch.zeros(9000, 1, dtype=torch.int32)
    res = ep.ep_layout(over.to(DEV), 4, 2, 1, 4)
    assert res.handle.check() == ep.EP_ERR_CAPACITY
    pos = res.handle.export()["pos"].cpu().numpy().ravel()
    assert pos[:4].tolist() == [0, 1, 2, 3] and (pos[4:] == -1).all()


def test_layout_capacity_overflow_reported():
    idx = torch.zeros(10, 1, dtype=torch.int32)  # 10 tokens to expert 0, capacity 4
    res = ep.ep_layout(idx.to(DEV), 4, 2, 1, 4)
    assert res.handle.check() == ep.EP_ERR_CAPACITY
    md = res.handle.export()
    pos = md["pos"].cpu().numpy().ravel()
    assert pos[:4].tolist() == [0, 1, 2, 3] and (pos[4:] == -1).all()
    assert md["src_idx"].cpu().numpy()[:4].tolist() == [0, 1, 2, 3]


# --- dispatch ----------------------------------------------------------------

def gpu_dispatch(x, res, fp8, sentinel=True):
    h = res.handle
    rows = h.num_recv_rows
    H = x.shape[1]
    dt = torch.float8_e4m3fn if fp8 else torch.bfloat16
    recv = torch.empty(rows, H, dtype=dt, device=DEV)
    sc = torch.empty(rows, H // 128, dtype=torch.float32, device=DEV) if fp8 else None
    if sentinel:
        recv.view(torch.uint8).fill_(0xA5)
        if sc is not None:
            sc.fill_(-7.0)
    src = torch.empty(rows, dtype=torch.int32, device=DEV)
    ep.ep_dispatch(h, x.to(DEV), fp8, recv, sc, src)
    torch.cuda.synchronize()
    return recv, sc, src


@pytest.mark.parametrize("name,T", [("tiny", None), ("large_skewed", 2048), ("decode", None)])
def test_dispatch_bf16(name, T):
    w = W.WORKLOADS[name]
    w = w.scaled(T=T) if T else w
    x, idx, _ = W.make_routing(w)
    res, md = run_layout(idx, w.E, w.R, w.align, w.capacity)
    _, L = oracle.layout(idx.numpy(), w.E, w.R, w.align, w.capacity)
    recv, _, src = gpu_dispatch(x, res, False)
    want = oracle.dispatch_bf16(x, L.pos, L.n_rows)
    got = u16(recv)
    valid = L.src_idx >= 0
    assert (got[valid] == want[valid]).all()
    assert (got[~valid] == 0xA5A5).all(), "padding rows must be left untouched"
    assert (src.cpu().numpy() == L.src_idx).all()


@pytest.mark.parametrize("name,T", [("prefill", 512), ("group_limited", 640), ("decode", None)])
def test_dispatch_fp8(name, T):
    w = W.WORKLOADS[name]
    w = w.scaled(T=T) if T else w
    x, idx, _ = W.make_routing(w)
    res, md = run_layout(idx, w.E, w.R, w.align, w.capacity)
    _, L = oracle.layout(idx.numpy(), w.E, w.R, w.align, w.capacity)
    recv, sc, _ = gpu_dispatch(x, res, True)
    q, s = oracle.dispatch_fp8(x, L.pos, L.n_rows)
    valid = L.src_idx >= 0
    got_q = u8(recv)
    got_s = sc.cpu().numpy()
    assert (got_q[valid] == q[valid]).all()
    assert (got_s[valid].view(np.uint32) == s[valid].view(np.uint32)).all()
    assert (got_q[~valid] == 0xA5).all() and (got_s[~valid] == -7.0).all()


@pytest.mark.parametrize("H", [8, 24, 1000, 8192 + 8, 16384 + 24])
def test_dispatch_bf16_hidden_sizes(H):
    w = W.WORKLOADS["tiny"].scaled(T=37, H=H)
    x, idx, _ = W.make_routing(w)
    res, _ = run_layout(idx, w.E, w.R)
    _, L = oracle.layout(idx.numpy(), w.E, w.R)
    recv, _, _ = gpu_dispatch(x, res, False)
    assert (u16(recv) == oracle.dispatch_bf16(x, L.pos, L.n_rows)).all()


def special_rows(T, H, seed):
    """Rows exercising the e4m3 corners: zero groups, -0, subnormal codes,
    saturation near 448, huge and tiny magnitudes, one dominant channel."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, H, generator=g)
    G = H // 128
    for t in range(T):
        mode = t % 6
        if mode == 0:
            x[t, :128] = 0.0
        elif mode == 1:
            x[t] = -0.0
            x[t, 5] = 1e-3
        elif mode == 2:
            x[t] *= 1e-30
        elif mode == 3:
            x[t] *= 3e38 / 8
        elif mode == 4:
            x[t, ::128] = 1000.0   # every group: one big channel, the rest to subnormal codes
        else:
            x[t] = torch.round(x[t] * 64) / 64
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("H", [128, 256, 7168, 8192 + 128, 20480])
def test_dispatch_fp8_special_values(H):
    T, k, E, R = 48, 4, 32, 4
    x = special_rows(T, H, H)
    g = torch.Generator().manual_seed(H + 1)
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)
    res, _ = run_layout(idx, E, R)
    _, L = oracle.layout(idx.numpy(), E, R)
    recv, sc, _ = gpu_dispatch(x, res, True)
    q, s = oracle.dispatch_fp8(x, L.pos, L.n_rows)
    assert (u8(recv) == q).all()
    assert (sc.cpu().numpy().view(np.uint32) == s.view(np.uint32)).all()


def test_dispatch_fp8_every_bf16_value():
    """Every finite bf16 bit pattern, quantised under several group maxima."""
    allb = torch.from_numpy(np.arange(1 << 16, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)
    fin = torch.isfinite(allb.float())
    vals = allb[fin]
    amaxes = [448.0, 1.0, 3.0, 1e-3, 7.0e4, 2.0 ** -100, 1.7e38]
    rows = []
    for am in amaxes:
        v = vals.float()
        v = v[v.abs() <= am]
        pad = (-v.numel()) % 127
        v = torch.cat([v, torch.zeros(pad)]).reshape(-1, 127)
        col = torch.full((v.shape[0], 1), am)  # the group max in every group
        rows.append(torch.cat([col, v], dim=1).reshape(-1))
    flat = torch.cat(rows)
    H = 1024
    flat = torch.cat([flat, torch.zeros((-flat.numel()) % H)])
    x = flat.reshape(-1, H).to(torch.bfloat16)
    T = x.shape[0]
    idx = torch.zeros(T, 1, dtype=torch.int32)
    res, _ = run_layout(idx, 1, 1)
    _, L = oracle.layout(idx.numpy(), 1, 1)
    recv, sc, _ = gpu_dispatch(x, res, True)
    q, s = oracle.dispatch_fp8(x, L.pos, L.n_rows)
    assert (u8(recv) == q).all()
    assert (sc.cpu().numpy().view(np.uint32) == s.view(np.uint32)).all()


# --- combine -----------------------------------------------------------------

def check_combine(out_gpu, want):
    got = u16(out_gpu)
    d = bf16_ulp_distance(got, want)
    assert int(d.max()) <= 1, "combine off by more than 1 bf16 ulp"
    return got


@pytest.mark.parametrize("name,T", [("tiny", None), ("prefill", 1024), ("group_limited", 512),
                                    ("decode", None), ("large_skewed", 2048)])
def test_combine(name, T):
    w = W.WORKLOADS[name]
    w = w.scaled(T=T) if T else w
    _, idx, tw = W.make_routing(w)
    res, _ = run_layout(idx, w.E, w.R, w.align, w.capacity)
    _, L = oracle.layout(idx.numpy(), w.E, w.R, w.align, w.capacity)
    y = W.make_expert_out(L.n_rows, w.H, seed=w.seed + 1)
    out = ep.ep_combine(res.handle, y.to(DEV), tw.to(DEV))
    torch.cuda.synchronize()
    want = oracle.combine(y, tw.numpy(), L.pos)
    got = check_combine(out, want)
    assert (got == want).all(), "same fma chain on both sides: expected bit-exact"


@pytest.mark.parametrize("H", [8, 136, 1000, 4096 + 8])
def test_combine_hidden_sizes_and_unused_slots(H):
    T, k, E, R = 300, 5, 16, 4
    g = torch.Generator().manual_seed(H)
    idx = torch.randint(-1, E, (T, k), generator=g, dtype=torch.int32)
    idx[7] = -1  # a token with no valid slot -> +0
    res, _ = run_layout(idx, E, R)
    _, L = oracle.layout(idx.numpy(), E, R)
    y = W.make_expert_out(L.n_rows, H, seed=3)
    tw = torch.rand(T, k, generator=g) * 2 - 0.5
    out = ep.ep_combine(res.handle, y.to(DEV), tw.to(DEV))
    want = oracle.combine(y, tw.numpy(), L.pos)
    got = check_combine(out, want)
    assert (got == want).all()
    assert (got[7] == 0).all()


def test_roundtrip_identity_experts_bf16():
    w = W.WORKLOADS["large_skewed"].scaled(T=4096)
    x, idx, tw = W.make_routing(w)
    res, _ = run_layout(idx, w.E, w.R)
    xd = x.to(DEV)
    recv, _, _ = ep.ep_dispatch(res.handle, xd, False)
    out = ep.ep_combine(res.handle, recv, tw.to(DEV))
    torch.cuda.synchronize()
    a, b = u16(out).astype(np.int64), u16(x).astype(np.int64)
    nz = (b & 0x7FFF) != 0
    assert (a[nz] == b[nz]).all() and ((a[~nz] & 0x7FFF) == 0).all()


# --- full sizes, element by element --------------------------------------------

def assert_rows_equal(got_dev, want, valid, what, chunk=8192):
    """Every valid row of a device tensor equals the oracle's (compared as raw
    bits, a chunk of rows at a time to bound host memory)."""
    n = want.shape[0]
    assert got_dev.shape[0] >= n
    for r0 in range(0, n, chunk):
        r1 = min(n, r0 + chunk)
        g = got_dev[r0:r1].contiguous()
        if g.dtype == torch.bfloat16:
            g = u16(g)
        elif g.dtype == torch.float32:
            g = g.cpu().numpy().view(np.uint32)
        else:
            g = u8(g)
        w = want[r0:r1]
        if w.dtype == np.float32:
            w = w.view(np.uint32)
        v = valid[r0:r1]
        bad = np.nonzero(~(g[v] == w[v]).all(axis=1))[0]
        assert bad.size == 0, "%s: %d rows differ, first receive row %d" % (
            what, bad.size, r0 + int(np.nonzero(v)[0][bad[0]]))


def test_group_limited_full_size_exact():
    """The benchmark's workload (group-limited gating, T=8192, H=7168, top-8,
    E=256, R=64, FP8 dispatch, BF16 combine) at full size: the layout, every
    receive row's codes and scales, and every element of the combined output
    against the oracle, with random expert outputs."""
    w = W.WORKLOADS["group_limited"]
    x, idx, tw = W.make_routing(w)
    res, md = run_layout(idx, w.E, w.R)
    _, L = oracle.layout(idx.numpy(), w.E, w.R)
    assert_layout_equal(res, md, L)
    recv, sc, src = gpu_dispatch(x, res, True)
    q, s = oracle.dispatch_fp8(x, L.pos, L.n_rows)
    valid = L.src_idx >= 0
    assert valid.all(), "packed layout without alignment: every row is used"
    assert_rows_equal(recv, q, valid, "FP8 codes")
    assert_rows_equal(sc, s, valid, "FP8 scales")
    assert (src.cpu().numpy() == L.src_idx).all()
    del q, s, recv, sc
    y = W.make_expert_out(L.n_rows, w.H, seed=9)
    out = ep.ep_combine(res.handle, y.to(DEV), tw.to(DEV))
    torch.cuda.synchronize()
    want = oracle.combine(y, tw.numpy(), L.pos)
    assert (u16(out) == want).all(), "combine differs from the oracle"
    assert res.handle.check() == ep.EP_OK


def test_prefill_full_size_exact():
    w = W.WORKLOADS["prefill"]
    x, idx, tw = W.make_routing(w)
    res, _ = run_layout(idx, w.E, w.R)
    _, L = oracle.layout(idx.numpy(), w.E, w.R)
    recv, sc, _ = gpu_dispatch(x, res, True, sentinel=False)
    q, s = oracle.dispatch_fp8(x, L.pos, L.n_rows)
    assert (u8(recv) == q).all()
    assert (sc.cpu().numpy().view(np.uint32) == s.view(np.uint32)).all()
    y = W.make_expert_out(L.n_rows, w.H, seed=10)
    out = ep.ep_combine(res.handle, y.to(DEV), tw.to(DEV))
    want = oracle.combine(y, tw.numpy(), L.pos)
    assert (u16(out) == want).all()


def test_large_skewed_full_size_exact():
    """Large skewed routing (T=32768, H=4096, E=128, Zipf 1.2, BF16) at full
    size: every receive row against the oracle's dispatch, every element of
    the combine of random expert outputs against the oracle's, and the
    identity round trip (combine of the received rows returns x)."""
    w = W.WORKLOADS["large_skewed"]
    x, idx, tw = W.make_routing(w)
    res, md = run_layout(idx, w.E, w.R)
    _, L = oracle.layout(idx.numpy(), w.E, w.R)
    assert_layout_equal(res, md, L)
    xd = x.to(DEV)
    twd = tw.to(DEV)
    recv, _, _ = ep.ep_dispatch(res.handle, xd, False)
    torch.cuda.synchronize()
    want_recv = oracle.dispatch_bf16(x, L.pos, L.n_rows)
    assert_rows_equal(recv, want_recv, L.src_idx >= 0, "BF16 receive rows")
    del want_recv
    out_id = ep.ep_combine(res.handle, recv, twd)   # identity experts
    torch.cuda.synchronize()
    a, b = u16(out_id).astype(np.int64), u16(x).astype(np.int64)
    nz = (b & 0x7FFF) != 0
    assert (a[nz] == b[nz]).all() and ((a[~nz] & 0x7FFF) == 0).all()
    del recv, out_id, a, b
    y = W.make_expert_out(L.n_rows, w.H, seed=11)
    out = ep.ep_combine(res.handle, y.to(DEV), twd)
    torch.cuda.synchronize()
    want = oracle.combine(y, tw.numpy(), L.pos)
    assert (u16(out) == want).all(), "combine differs from the oracle"
    assert res.handle.check() == ep.EP_OK


# --- decode: cached handle, CUDA graph, determinism ---------------------------

def test_decode_cached_handle_and_graph():
    w = W.WORKLOADS["decode"]
    _, idx, tw = W.make_routing(w)
    res, _ = run_layout(idx, w.E, w.R, w.align, w.capacity)
    h = res.handle
    _, L = oracle.layout(idx.numpy(), w.E, w.R, w.align, w.capacity)
    rows = h.num_recv_rows
    xb = torch.empty(w.T, w.H, dtype=torch.bfloat16, device=DEV)
    recv = torch.zeros(rows, w.H, dtype=torch.float8_e4m3fn, device=DEV)
    sc = torch.zeros(rows, w.H // 128, dtype=torch.float32, device=DEV)
    y = W.make_expert_out(rows, w.H, seed=21).to(DEV)
    twd = tw.to(DEV)
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device=DEV)

    def step():
        ep.ep_dispatch(h, xb, True, recv, sc)
        ep.ep_combine(h, y, twd, out)

    # plain launches
    for s in (0, 1, 99):
        xs = W.make_x(w, 1000 + s)
        xb.copy_(xs)
        step()
        torch.cuda.synchronize()
        q, scl = oracle.dispatch_fp8(xs, L.pos, L.n_rows)
        valid = L.src_idx >= 0
        assert (u8(recv)[valid] == q[valid]).all()
        assert (sc.cpu().numpy()[valid] == scl[valid]).all()
    want_out = oracle.combine(y.cpu(), tw.numpy(), L.pos)
    assert (u16(out) == want_out).all()

    # CUDA graph of dispatch + combine, replayed with new x each step
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        step()
    torch.cuda.current_stream().wait_stream(stream)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    for s in (5, 6):
        xs = W.make_x(w, 1000 + s)
        xb.copy_(xs)
        recv.view(torch.uint8).zero_()
        graph.replay()
        torch.cuda.synchronize()
        q, scl = oracle.dispatch_fp8(xs, L.pos, L.n_rows)
        valid = L.src_idx >= 0
        assert (u8(recv)[valid] == q[valid]).all()
    assert h.check() == ep.EP_OK
    del graph


def test_deterministic_runs():
    w = W.WORKLOADS["group_limited"].scaled(T=2048)
    x, idx, tw = W.make_routing(w)
    outs = []
    for _ in range(2):
        res, md = run_layout(idx, w.E, w.R)
        recv, sc, _ = gpu_dispatch(x, res, True, sentinel=False)
        y = W.make_expert_out(res.handle.num_recv_rows, w.H, seed=2).to(DEV)
        out = ep.ep_combine(res.handle, y, tw.to(DEV))
        torch.cuda.synchronize()
        outs.append((md["pos"].cpu(), u8(recv), sc.cpu(), u16(out)))
    a, b = outs
    assert torch.equal(a[0], b[0]) and (a[1] == b[1]).all()
    assert torch.equal(a[2], b[2]) and (a[3] == b[3]).all()


# --- argument errors through the binding --------------------------------------

def test_argument_errors():
    w = W.WORKLOADS["tiny"]
    x, idx, tw = W.make_routing(w)
    res, _ = run_layout(idx, w.E, w.R)
    h = res.handle
    xd = x.to(DEV)
    small = torch.empty(h.num_recv_rows - 1, w.H, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ep.EpError) as e:
        ep.ep_dispatch(h, xd, False, small)
    assert e.value.status == ep.EP_ERR_INVALID_ARG
    buf = torch.empty(h.num_recv_rows * w.H + 1, dtype=torch.bfloat16, device=DEV)
    mis = buf[1:].view(h.num_recv_rows, w.H)  # 2-byte offset: not 16-byte aligned
    with pytest.raises(ep.EpError):
        ep.ep_dispatch(h, xd, False, mis)
    xs = torch.zeros(w.T, 136, dtype=torch.bfloat16, device=DEV)  # FP8 needs H % 128 == 0
    with pytest.raises(ep.EpError):
        ep.ep_dispatch(h, xs, True)
