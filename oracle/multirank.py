"""Expert parallelism over several real ranks, defined from the single-GPU oracle.

TEST INFRASTRUCTURE ONLY (same rules as the rest of ``oracle/``).

The pages describe dispatch as sending every token to its experts on all
ranks and combine as reducing the expert outputs back to the rank each token
came from ("DeepSeek publica DeepEP, una biblioteca open source para
entrenamiento e inferencia MoE", news.hada.io, "Patrones de uso en
entrenamiento, prefill y decoding"; "DeepEP (DeepEveryParallel)
Documentation", item 10).  They do not fix an order for the received rows.
This library takes the single-GPU order over the concatenation of all ranks'
tokens in rank order: rank r owns experts [r*E/W, (r+1)*E/W) and receives
exactly the rows [rank_off[r], rank_off[r+1]) of the single-GPU layout of the
concatenated batch, so inside one expert's segment rows are ordered by
(source rank, source token, slot).  Each function below is that definition:
concatenate, run the single-GPU oracle, slice.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

import oracle


@dataclass
class RankedLayout:
    """The concatenated layout plus where every rank's tokens start in it."""
    L: oracle.Layout
    W: int
    token_base: list      # first concatenated token of each source rank
    T: list               # tokens of each source rank

    @property
    def epr(self) -> int:
        return self.L.E // self.W

    def recv_rows(self, r: int) -> int:
        """Rows rank r receives (its slice of the concatenated layout)."""
        return int(self.L.rank_off[r + 1] - self.L.rank_off[r])

    def recv_seg(self, r: int) -> np.ndarray:
        """Segment starts of rank r's experts inside its own receive buffer [E/W + 1]."""
        e0 = r * self.epr
        return (self.L.seg[e0:e0 + self.epr + 1] - self.L.rank_off[r]).astype(np.int32)

    def recv_counts(self, r: int) -> np.ndarray:
        """Slots routed to each of rank r's experts, over all source ranks [E/W]."""
        e0 = r * self.epr
        return self.L.num_tokens_per_expert[e0:e0 + self.epr].copy()

    def destinations(self, s: int) -> np.ndarray:
        """int32 [T_s, k, 2]: (owner rank, row in the owner's receive buffer)
        of every slot of source rank s; (-1, -1) for unused or over-capacity slots."""
        b, T = self.token_base[s], self.T[s]
        pos = self.L.pos[b:b + T]
        d = np.full(pos.shape + (2,), -1, np.int32)
        valid = pos >= 0
        owner = np.searchsorted(self.L.rank_off, pos, side="right") - 1
        d[..., 0] = np.where(valid, owner, -1)
        d[..., 1] = np.where(valid, pos - self.L.rank_off[np.clip(owner, 0, self.W)], -1)
        return d


def layout(idx_list, E: int, W: int, align: int = 1, capacity: int = 0, check: bool = True):
    """Layout of W ranks' top-k ids (list of int32 [T_s, k]); returns (status, RankedLayout)."""
    T = [int(a.shape[0]) for a in idx_list]
    base = list(np.cumsum([0] + T[:-1]).astype(int))
    idx = np.ascontiguousarray(np.concatenate([np.asarray(a, np.int32) for a in idx_list]), np.int32)
    st, L = oracle.layout(idx, E, W, align, capacity, check=check)
    return st, RankedLayout(L, W, base, T)


def _concat_u16(xs):
    return np.concatenate([oracle._u16(x) for x in xs])


def dispatch_bf16(RL: RankedLayout, x_list):
    """Per-rank receive buffers (uint16 [recv_rows(r), H]); rows no slot fills are zero."""
    recv = oracle.dispatch_bf16(_concat_u16(x_list), RL.L.pos, RL.L.n_rows)
    return [recv[RL.L.rank_off[r]:RL.L.rank_off[r + 1]] for r in range(RL.W)]


def dispatch_fp8(RL: RankedLayout, x_list):
    """Per-rank (codes uint8 [recv_rows(r), H], scales float32 [recv_rows(r), H/128])."""
    q, s = oracle.dispatch_fp8(_concat_u16(x_list), RL.L.pos, RL.L.n_rows)
    return [(q[RL.L.rank_off[r]:RL.L.rank_off[r + 1]], s[RL.L.rank_off[r]:RL.L.rank_off[r + 1]])
            for r in range(RL.W)]


def combine(RL: RankedLayout, y_list, w_list):
    """y_list[r]: bf16 [>= recv_rows(r), H] expert outputs on rank r, rows in
    its receive order; w_list[s]: float32 [T_s, k].  Returns the combined
    uint16 [T_s, H] of every source rank."""
    w = np.concatenate([np.asarray(a, np.float32) for a in w_list])
    out = oracle.combine(_concat_y(RL, y_list), w, RL.L.pos)
    return [out[b:b + T] for b, T in zip(RL.token_base, RL.T)]


def _concat_y(RL: RankedLayout, y_list):
    H = oracle._u16(y_list[0]).shape[1]
    y = np.zeros((max(RL.L.n_rows, 1), H), np.uint16)
    for r in range(RL.W):
        n = RL.recv_rows(r)
        y[RL.L.rank_off[r]:RL.L.rank_off[r] + n] = oracle._u16(y_list[r])[:n]
    return y[:RL.L.n_rows]


def combine_backward(RL: RankedLayout, grad_out_list, y_list, w_list):
    """The backward of `combine` across ranks (the pages: a combine's backward
    is a dispatch).  grad_out_list[s]: bf16 [T_s, H]; y_list[r]: the owner's
    expert outputs.  Returns (grad_y per owner rank, uint16 [recv_rows(r), H],
    rows no slot fills are 0; grad_w per source rank, float64 [T_s, k])."""
    g = _concat_u16(grad_out_list)
    w = np.concatenate([np.asarray(a, np.float32) for a in w_list])
    gy, gw = oracle.combine_backward(g, _concat_y(RL, y_list), w, RL.L.pos)
    return ([gy[RL.L.rank_off[r]:RL.L.rank_off[r + 1]] for r in range(RL.W)],
            [gw[b:b + T] for b, T in zip(RL.token_base, RL.T)])


def dispatch_topk(RL: RankedLayout, idx_list, w_list):
    """Per-row routing outputs on every owner rank: (recv_topk_idx int32,
    recv_topk_weights float32, recv_src_rank int32, recv_slot int32), each
    [recv_rows(r)]; recv_slot is the slot's flat index t*k + j on its source
    rank.  Rows no slot fills get -1, 0, -1, -1."""
    idx = np.concatenate([np.asarray(a, np.int32) for a in idx_list])
    w = np.concatenate([np.asarray(a, np.float32) for a in w_list])
    ri, rw, rs = oracle.dispatch_topk(idx, w, RL.L.pos, RL.L.n_rows)
    k = RL.L.k
    rank_of_token = np.repeat(np.arange(RL.W, dtype=np.int64), RL.T)   # concatenated token -> source rank
    base = np.asarray(RL.token_base, np.int64)
    out = []
    for r in range(RL.W):
        a, b = RL.L.rank_off[r], RL.L.rank_off[r + 1]
        slot_g = rs[a:b].astype(np.int64)
        filled = slot_g >= 0
        src = np.where(filled, rank_of_token[np.where(filled, slot_g // k, 0)], -1)
        slot = np.where(filled, slot_g - base[np.where(filled, src, 0)] * k, -1)
        out.append((ri[a:b].copy(), rw[a:b].copy(), src.astype(np.int32), slot.astype(np.int32)))
    return out
