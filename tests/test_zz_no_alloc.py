"""ep_layout_noalloc against ep_layout (GPU).

ep_layout_noalloc serves callers that cannot allocate device memory (static
memory planners, code running under another framework's allocator, loops that
cannot afford cudaMalloc's implicit synchronisation): it writes the layout into
caller buffers and keeps its scratch in a fixed array inside the library.  Its
results must equal those of ep_layout (+ ep_handle_export) bit for bit, also
on the second of two calls in a row, when the shared scratch still holds the
first call's contents.  This file is collected last on purpose.
"""
import pytest
import torch

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


def buffers(T, k, E, R, rows):
    return dict(pos=torch.full((T, k), 7, dtype=torch.int32, device=DEV),
                src_idx=torch.full((rows,), 7, dtype=torch.int32, device=DEV),
                seg=torch.full((E + 1,), 7, dtype=torch.int32, device=DEV),
                rank_off=torch.full((R + 1,), 7, dtype=torch.int32, device=DEV),
                num_tokens_per_expert=torch.full((E,), 7, dtype=torch.int32, device=DEV),
                num_tokens_per_rank=torch.full((R,), 7, dtype=torch.int32, device=DEV),
                is_token_in_rank=torch.full((T, R), 7, dtype=torch.uint8, device=DEV),
                error_word=torch.full((1,), 7, dtype=torch.int32, device=DEV))


def reference(idx, E, R, A, C, want_status=ep.EP_OK):
    res = ep.ep_layout(idx, E, R, A, C)
    md = res.handle.export()
    torch.cuda.synchronize()
    assert res.handle.check() == want_status
    out = dict(md, num_tokens_per_expert=res.num_tokens_per_expert,
               num_tokens_per_rank=res.num_tokens_per_rank, is_token_in_rank=res.is_token_in_rank)
    res.handle.free()
    return out


def noalloc(idx, E, R, A, C, b, with_error_word=True):
    ep.ep_layout_noalloc(idx, E, R, b["pos"], b["src_idx"], b["seg"], b["rank_off"], A, C,
                         num_tokens_per_expert=b["num_tokens_per_expert"],
                         num_tokens_per_rank=b["num_tokens_per_rank"],
                         is_token_in_rank=b["is_token_in_rank"],
                         error_word=b["error_word"] if with_error_word else None)
    torch.cuda.synchronize()


def assert_same(b, want, what):
    for key, ref in want.items():
        assert torch.equal(b[key].cpu(), ref.cpu()), (what, key)


def test_noalloc_matches_layout_on_two_calls_in_a_row():
    cases = [W.WORKLOADS["group_limited"], W.WORKLOADS["decode"]]
    for w in cases:
        _, idx_cpu, _ = W.make_routing(w)
        idx = idx_cpu.to(DEV)
        rows = ep.ep_max_recv_rows(w.T, w.k, w.E, w.align, w.capacity)
        want = reference(idx, w.E, w.R, w.align, w.capacity)
        b = buffers(w.T, w.k, w.E, w.R, rows)
        ep.ep_layout_noalloc(idx, w.E, w.R, b["pos"], b["src_idx"], b["seg"], b["rank_off"],
                             w.align, w.capacity,
                             num_tokens_per_expert=b["num_tokens_per_expert"],
                             num_tokens_per_rank=b["num_tokens_per_rank"],
                             is_token_in_rank=b["is_token_in_rank"], error_word=b["error_word"])
        torch.cuda.synchronize()
        assert int(b["error_word"].item()) == 0, w.name
        for key, ref in want.items():
            assert torch.equal(b[key].cpu(), ref.cpu()), (w.name, key)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # One expert, one rank: 12288 tiles of 128 tokens; the per-tile words
    # (2 count words + 1 flag word per tile) exceed the 2^15-word scratch.
    T, k, E, R = 12288 * 128, 1, 1, 1
    idx = torch.zeros(T, k, dtype=torch.int32, device=DEV)
    rows = ep.ep_max_recv_rows(T, k, E)
    b = buffers(T, k, E, R, rows)
    with pytest.raises(ep.EpError) as e:
        ep.ep_layout_noalloc(idx, E, R, b["pos"], b["src_idx"], b["seg"], b["rank_off"])
    assert e.value.status == ep.EP_ERR_SCRATCH_LIMIT
    assert int(b["pos"][0, 0].item()) == 7, "nothing may be enqueued on rejection"


def data_error_ids(T, k, E, seed):
    """Ids with an invalid id and, in padded mode, expert 3 named by half the
    tokens (an overflow of any capacity below T / 2)."""
    g = torch.Generator().manual_seed(seed)
    idx = torch.randint(-1, E, (T, k), generator=g, dtype=torch.int32)
    idx[: T // 2, 0] = 3
    idx[T // 3, k - 1] = E + 5
    return idx


def test_noalloc_tiled_calls_back_to_back_and_data_errors():
    """Several calls in a row on the tiled path, with different tile counts,
    expert and rank counts, each reading the per-tile counts the previous call
    left in the shared scratch: every result equals ep_layout's, and the error
    word carries the same device-detected errors as the handle (an invalid id;
    an invalid id plus a padded expert over capacity)."""
    cases = [
        # (workload or (T, k, E, R), align, capacity, ids, expected handle status, error-word bits)
        ("prefill", 1, 0, None, ep.EP_OK, 0),
        ("group_limited", 1, 0, None, ep.EP_OK, 0),
        ((9000, 2, 96, 48), 4, 0, "bad", ep.EP_ERR_BAD_EXPERT_ID, 1),
        ((5000, 2, 16, 4), 1, 64, "bad", ep.EP_ERR_BAD_EXPERT_ID, 1 | 2),
        ((5000, 2, 16, 4), 1, 64, "over", ep.EP_ERR_CAPACITY, 2),
        ("large_skewed", 1, 0, None, ep.EP_OK, 0),
    ]
    for i, (shape, A, C, kind, status, bits) in enumerate(cases):
        if isinstance(shape, str):
            w = W.WORKLOADS[shape]
            T, k, E, R = w.T, w.k, w.E, w.R
            _, idx_cpu, _ = W.make_routing(w)
        else:
            T, k, E, R = shape
            idx_cpu = data_error_ids(T, k, E, seed=i)
            if kind == "over":
                idx_cpu[idx_cpu >= E] = 0
        idx = idx_cpu.to(DEV)
        rows = ep.ep_max_recv_rows(T, k, E, A, C)
        want = reference(idx, E, R, A, C, status)
        b = buffers(T, k, E, R, rows)
        noalloc(idx, E, R, A, C, b)
        assert int(b["error_word"].item()) == bits, (shape, kind)
        assert_same(b, want, (shape, kind))


def test_noalloc_without_error_word():
    """error_word = NULL: the device-detected errors go to a word inside the
    scratch array and are not reported; the layout itself is unchanged (here
    right after a call that set both error bits)."""
    T, k, E, R, C = 5000, 2, 16, 4, 64
    idx = data_error_ids(T, k, E, seed=77).to(DEV)
    rows = ep.ep_max_recv_rows(T, k, E, 1, C)
    want = reference(idx, E, R, 1, C, ep.EP_ERR_BAD_EXPERT_ID)
    b = buffers(T, k, E, R, rows)
    noalloc(idx, E, R, 1, C, b)
    assert int(b["error_word"].item()) == 3
    for _ in range(2):   # two calls in a row without an error word
        b = buffers(T, k, E, R, rows)
        noalloc(idx, E, R, 1, C, b, with_error_word=False)
        assert int(b["error_word"].item()) == 7, "an absent error word must not be written"
        assert_same(b, want, "error_word=None")
    w = W.WORKLOADS["group_limited"]
    _, idx_cpu, _ = W.make_routing(w)
    idx = idx_cpu.to(DEV)
    want = reference(idx, w.E, w.R, 1, 0)
    b = buffers(w.T, w.k, w.E, w.R, ep.ep_max_recv_rows(w.T, w.k, w.E))
    noalloc(idx, w.E, w.R, 1, 0, b, with_error_word=False)
    assert_same(b, want, "group_limited, error_word=None")
