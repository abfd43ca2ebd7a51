"""Expert parallelism over real GPUs: one process per GPU, W ranks.

The routing contract is the one of the single-GPU library, with the virtual
ranks made physical: rank r owns experts [r*E/W, (r+1)*E/W) and its receive
buffer holds the rows the single-GPU layout would give rank r for all ranks'
tokens concatenated in rank order.  Every step of the data path runs in the
library's kernels (layout, plan, peer dispatch, peer combine); this module is
plumbing only: it allocates the buffers every rank exposes, exchanges their
CUDA IPC handles, all-gathers the per-expert counts, and places the
collectives that order one rank's stores before another rank's reads:

    dispatch:  layout -> all-gather counts -> plan -> peer stores -> barrier
    combine:   barrier (every y written) -> peer loads
    backward:  combine_backward: barrier -> peer stores of grad_y (+ grad_w
               from the owners' y) -> barrier; dispatch_backward: barrier
               (every owner wrote its receive-row gradients into its y
               buffer) -> peer loads with unit weights

The next dispatch's all-gather (or, with a cached plan, its barrier) orders
its stores after every rank's reads of the previous step.  No kernel waits
on another rank, so a rank that fails shows up as a collective error or
timeout on the host.  With the NCCL backend the collectives are ordered on
the current stream; with gloo (tests) the stream is synchronised around them.
"""
from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist

from . import ep


class EpGroup:
    """This rank's side of an expert-parallel group.

    recv_rows: rows of every rank's receive buffer (the same on all ranks);
    ep.ep_peer_max_recv_rows() gives a bound that always suffices.
    fp8: receive buffers hold e4m3 codes + fp32 scales (else bf16).
    scale_layout: "row" (scales [recv_rows, H/128]) or "col" ([H/128, ld],
    ld = recv_rows rounded up to 4: the FP8 grouped-GEMM layout).
    """

    def __init__(self, num_experts: int, hidden: int, recv_rows: int, fp8: bool = True,
                 group: Optional[dist.ProcessGroup] = None, device: Optional[torch.device] = None,
                 scale_layout: str = "row"):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        if num_experts % self.world:
            raise ValueError("num_experts must be a multiple of the group size")
        self.E, self.H, self.recv_rows, self.fp8 = num_experts, hidden, recv_rows, fp8
        self.device = device or torch.device("cuda", torch.cuda.current_device())
        self.nccl = dist.get_backend(group) == "nccl"
        dev = self.device
        self.recv_x = torch.empty(recv_rows, hidden, dtype=torch.float8_e4m3fn if fp8 else torch.bfloat16,
                                  device=dev)
        if scale_layout not in ("row", "col"):
            raise ValueError("scale_layout must be 'row' or 'col'")
        self.scale_layout = scale_layout
        self.scale_ld = (recv_rows + 3) // 4 * 4
        if not fp8:
            self.recv_scales = None
        elif scale_layout == "row":
            self.recv_scales = torch.empty(recv_rows, hidden // 128, dtype=torch.float32, device=dev)
        else:
            self.recv_scales = torch.empty(hidden // 128, self.scale_ld, dtype=torch.float32, device=dev)
        self.y = torch.empty(recv_rows, hidden, dtype=torch.bfloat16, device=dev)
        self.grad_y = torch.empty(recv_rows, hidden, dtype=torch.bfloat16, device=dev)
        # per-row routing outputs of each received row: expert, weight, source rank, source slot
        self.recv_topk_idx = torch.empty(recv_rows, dtype=torch.int32, device=dev)
        self.recv_topk_weights = torch.empty(recv_rows, dtype=torch.float32, device=dev)
        self.recv_src_rank = torch.empty(recv_rows, dtype=torch.int32, device=dev)
        self.recv_slot = torch.empty(recv_rows, dtype=torch.int32, device=dev)
        mine = [self.recv_x, self.recv_scales, self.y, self.grad_y,
                self.recv_topk_idx, self.recv_topk_weights, self.recv_src_rank, self.recv_slot]
        handles = [ep.ipc_export(t) if t is not None else None for t in mine]
        torch.cuda.synchronize(dev)
        everyone = [None] * self.world
        dist.all_gather_object(everyone, handles, group=group)
        # Several buffers can live in one allocation (the caching allocator
        # packs small ones together): each distinct handle is opened once and
        # the buffers are addressed by their offsets inside it.
        self._imported = []   # base addresses of opened handles, to release
        opened = {}
        tables = [[] for _ in mine]
        for r in range(self.world):
            for i, t in enumerate(mine):
                if t is None:
                    continue
                if r == self.rank:
                    tables[i].append(t.data_ptr())
                    continue
                blob, off = everyone[r][i]
                if blob not in opened:
                    opened[blob] = ep.ipc_import(blob, 0)
                    self._imported.append(opened[blob])
                tables[i].append(opened[blob] + off)
        self.peers = ep.Peers(self.world, tables[0], tables[1] if fp8 else None, tables[2], recv_rows,
                              grad_y=tables[3])
        self.peers.set_topk(*tables[4:8])

    # -- collectives -------------------------------------------------------

    def _barrier(self) -> None:
        if self.nccl:
            t = torch.zeros(1, dtype=torch.int32, device=self.device)
            dist.all_reduce(t, group=self.group)   # ordered on the current stream
        else:
            torch.cuda.current_stream(self.device).synchronize()
            dist.barrier(group=self.group)

    def _gather_counts(self, counts: torch.Tensor) -> torch.Tensor:
        if self.nccl:
            out = torch.empty(self.world, self.E, dtype=torch.int32, device=self.device)
            dist.all_gather_into_tensor(out, counts, group=self.group)
            return out
        parts = [torch.empty(self.E, dtype=torch.int32) for _ in range(self.world)]
        dist.all_gather(parts, counts.cpu(), group=self.group)
        return torch.stack(parts).to(self.device)

    # -- the data path -----------------------------------------------------

    def make_plan(self, topk_idx: torch.Tensor, expert_alignment: int = 1, capacity: int = 0) -> ep.Plan:
        """Layout of this rank's tokens, counts of every rank, and the plan."""
        res = ep.ep_layout(topk_idx, self.E, self.world)
        counts = self._gather_counts(res.num_tokens_per_expert)
        plan = ep.ep_plan_create(res.handle, topk_idx, counts, self.rank, self.world, self.recv_rows,
                                 expert_alignment, capacity)
        res.handle.free()   # stream-ordered: after the plan has read it
        return plan

    def dispatch(self, x: torch.Tensor, topk_idx: Optional[torch.Tensor] = None,
                 plan: Optional[ep.Plan] = None, expert_alignment: int = 1, capacity: int = 0,
                 x_scales: Optional[torch.Tensor] = None, num_sms: int = 0,
                 topk_weights: Optional[torch.Tensor] = None) -> ep.Plan:
        """Sends this rank's tokens to their experts' owners.  Pass `plan` (a
        cached handle) when the routing has not changed.  On return, in stream
        order, this rank's receive buffer holds its rows from every rank; with
        `topk_weights` (and `topk_idx`) recv_topk_idx / recv_topk_weights /
        recv_src_rank / recv_slot also describe every received row."""
        if plan is None:
            if topk_idx is None:
                raise ValueError("dispatch needs topk_idx or a plan")
            plan = self.make_plan(topk_idx, expert_alignment, capacity)   # its all-gather orders our stores
        else:
            self._barrier()   # peers have finished reading the previous step
        ep.ep_dispatch_peer(plan, self.peers, x, self.fp8, x_scales=x_scales, num_sms=num_sms,
                            scale_layout=self.scale_layout, scale_ld=self.scale_ld)
        if topk_weights is not None:
            if topk_idx is None:
                raise ValueError("per-row outputs need topk_idx")
            ep.ep_dispatch_topk_peer(plan, self.peers, topk_idx, topk_weights)
        self._barrier()       # every rank's stores are complete
        return plan

    def combine(self, plan: ep.Plan, topk_weights: Optional[torch.Tensor], num_sms: int = 0) -> torch.Tensor:
        """Each local token's weighted sum of its expert outputs, read from the
        owners' `y` buffers (the caller has written its own `y` rows)."""
        self._barrier()       # every rank's y is written
        return ep.ep_combine_peer(plan, self.peers, topk_weights, self.H, num_sms=num_sms)

    def combine_backward(self, plan: ep.Plan, grad_out: torch.Tensor, topk_weights: torch.Tensor,
                         want_grad_weights: bool = True) -> Optional[torch.Tensor]:
        """Backward of `combine`: every local slot's gradient row
        bf16(w * grad_out[t]) lands in its owner's `grad_y` buffer; returns
        grad_weights [T, k] (dot products with the owners' y rows) or None."""
        self._barrier()       # owners have finished with the previous grad_y
        gw = ep.ep_combine_backward_peer(plan, self.peers, grad_out, topk_weights, want_grad_weights)
        self._barrier()       # every rank's gradient rows are stored
        return gw

    def dispatch_backward(self, plan: ep.Plan) -> torch.Tensor:
        """Backward of `dispatch`: each local token's sum of its receive-row
        gradients, read from the owners' `y` buffers, into which every rank's
        expert backward has written its receive-row gradients (y is no longer
        needed once combine_backward has run)."""
        self._barrier()       # every owner's receive-row gradients are written
        return ep.ep_combine_peer(plan, self.peers, None, self.H)

    def close(self) -> None:
        """Release the peer mappings (after a final barrier, so no rank still
        reads or writes through them)."""
        if self.peers is None:
            return
        self._barrier()
        torch.cuda.synchronize(self.device)
        self.peers.free()
        self.peers = None
        for base in self._imported:
            ep.ipc_release(base, 0)
        self._imported = []
