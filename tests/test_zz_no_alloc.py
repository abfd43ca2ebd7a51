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


def reference(idx, E, R, A, C):
    res = ep.ep_layout(idx, E, R, A, C)
    md = res.handle.export()
    torch.cuda.synchronize()
    assert res.handle.check() == ep.EP_OK
    out = dict(md, num_tokens_per_expert=res.num_tokens_per_expert,
               num_tokens_per_rank=res.num_tokens_per_rank, is_token_in_rank=res.is_token_in_rank)
    res.handle.free()
    return out


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
