"""The seeded workload generators: deterministic, the stated shapes and structure."""
import pytest
import torch

from combine_ep_layout_10_b200 import workloads as W


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_shapes_and_determinism(name):
    w = W.WORKLOADS[name]
    x, idx, tw = W.make_routing(w)
    assert x.dtype == torch.bfloat16 and tuple(x.shape) == (w.T, w.H)
    assert idx.dtype == torch.int32 and tuple(idx.shape) == (w.T, w.k)
    assert tw.dtype == torch.float32 and tuple(tw.shape) == (w.T, w.k)
    assert int(idx.min()) >= 0 and int(idx.max()) < w.E
    s, _ = idx.sort(dim=1)
    assert not bool((s[:, 1:] == s[:, :-1]).any()), "experts of a token must be distinct"
    assert torch.allclose(tw.sum(1), torch.ones(w.T), atol=1e-6)
    x2, idx2, tw2 = W.make_routing(w)
    assert torch.equal(x.view(torch.int16), x2.view(torch.int16))
    assert torch.equal(idx, idx2) and torch.equal(tw, tw2)


def test_group_limited_structure():
    w = W.WORKLOADS["group_limited"].scaled(T=512)
    _, idx, _ = W.make_routing(w)
    groups = idx // (w.E // w.groups)
    for t in range(w.T):
        assert len(set(groups[t].tolist())) <= w.topk_groups
    st = W.load_stats(idx, w.E)
    assert st["hot_over_mean"] > 10  # Zipf bias makes expert 0 hot


def test_skew_and_capacity():
    st = W.load_stats(W.make_routing(W.WORKLOADS["large_skewed"].scaled(T=4096))[1], 128)
    assert 8 < st["hot_over_mean"] <= 16
    w = W.WORKLOADS["decode"]
    _, idx, _ = W.make_routing(w)
    assert int(torch.bincount(idx.flatten().long(), minlength=w.E).max()) <= w.capacity


def test_decode_steps_differ():
    w = W.WORKLOADS["decode"]
    a, b = W.make_x(w, 1000), W.make_x(w, 1001)
    assert a.shape == (w.T, w.H) and not torch.equal(a, b)


def test_expert_out_blocks_are_deterministic():
    """Expert outputs are drawn in seeded blocks: the same seed gives the same
    tensor (whatever the thread schedule), another seed another one, and the
    values are N(0,1) rounded to bf16."""
    a = W.make_expert_out(9000, 4096, seed=3)   # several blocks of 4096 rows
    b = W.make_expert_out(9000, 4096, seed=3)
    c = W.make_expert_out(9000, 4096, seed=4)
    assert a.dtype == torch.bfloat16 and tuple(a.shape) == (9000, 4096)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert not torch.equal(a.view(torch.int16), c.view(torch.int16))
    # blocks differ from each other (no block reuses another's seed)
    assert not torch.equal(a[:4096].view(torch.int16), a[4096:8192].view(torch.int16))
    f = a.float()
    assert abs(f.mean().item()) < 0.01 and abs(f.std().item() - 1.0) < 0.01
    assert W.make_expert_out(0, 8, seed=1).shape == (0, 8)
