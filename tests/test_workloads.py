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
