"""Sequence-parallel attention over several GPUs: sequence shards in, sequence shards out.

"OSP-Next" page, "Method": Sparse Sequence Parallelism partitions the (sub)sequences across
ranks and switches between the layouts that the sparse patterns need with a single
all-to-all.  In one attention call of this library every head's pattern reaches all N
tokens of that head (a spatial head keeps a window of whole frames, a temporal head every
frame of a window of positions), while heads never interact.  So the call's layout switch is
the one between token shards and head shards:

  1. one all-to-all takes this rank's token shard of Q, K and V (all heads, packed into one
     buffer) to the ranks that own each head, so every rank holds all N tokens of its heads;
  2. the rank runs the whole single-GPU call (profiling, permutation, masks, block-sparse
     attention) on its heads;
  3. one all-to-all takes the output rows back to the ranks that own each token shard.

Heads are split as evenly as the count allows (12 heads on 8 ranks: 2,2,2,2,1,1,1,1) and so
are tokens (contiguous shards in natural order).  The exchange uses torch.distributed
(NCCL over NVLink on GPUs, gloo on CPU for the tests); packing and unpacking are plain
tensor copies.  The local call is a parameter only so that the exchange can be tested on CPU
ranks; by default it is this library's SparseAttention on the rank's device.
"""
from __future__ import annotations

from typing import Callable, List, Optional

import torch
import torch.distributed as dist


def split_even(n: int, parts: int) -> List[int]:
    """Sizes of `parts` contiguous pieces of n, the remainder going to the first pieces."""
    base, rem = divmod(n, parts)
    return [base + (1 if i < rem else 0) for i in range(parts)]


def _offsets(sizes: List[int]) -> List[int]:
    out, acc = [], 0
    for s in sizes:
        out.append(acc)
        acc += s
    return out


class SequenceParallelAttention:
    """One attention call over a B x H x (F x Hl x Wl) x d problem whose tokens are sharded
    across the ranks of `group`: rank r passes q, k, v of shape [B, H, n_r, d] (its contiguous
    token shard, every head) and receives o of the same shape.

    local_attention: callable(q, k, v) -> o on [B, h_r, N, d] tensors holding this rank's
        heads (global heads head_offset .. head_offset + h_r - 1).  Default: a SparseAttention
        for those heads on `device`, built with **attention_kwargs.
    """

    def __init__(self, B: int, H: int, F: int, Hl: int, Wl: int, d: int, block: int = 128, *,
                 group: Optional[dist.ProcessGroup] = None,
                 local_attention: Optional[Callable[[torch.Tensor, torch.Tensor, torch.Tensor], torch.Tensor]] = None,
                 device=None, **attention_kwargs):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.B, self.H, self.d = B, H, d
        self.N = F * Hl * Wl
        self.heads = split_even(H, self.world)
        self.head0 = _offsets(self.heads)
        self.tokens = split_even(self.N, self.world)
        self.token0 = _offsets(self.tokens)
        self.head_offset = self.head0[self.rank]
        h = self.heads[self.rank]
        if local_attention is None and h > 0:
            from . import SparseAttention
            plan = SparseAttention(B, h, F, Hl, Wl, d, block, device=device, **attention_kwargs)
            local_attention = plan
            self.plan = plan
        self.local = local_attention

    def __call__(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor) -> torch.Tensor:
        r, W, B, d = self.rank, self.world, self.B, self.d
        n_r, h_r = self.tokens[r], self.heads[r]
        for x in (q, k, v):
            if tuple(x.shape) != (B, self.H, n_r, d):
                raise ValueError(f"rank {r} expects [B, H, n_r, d] = {(B, self.H, n_r, d)}, got {tuple(x.shape)}")
        # 1. token shard (all heads) -> head shard (all tokens): Q, K, V in one exchange
        send = torch.cat([torch.stack([x[:, self.head0[p]:self.head0[p] + self.heads[p]] for x in (q, k, v)])
                          .reshape(-1) for p in range(W)])
        in_splits = [3 * B * self.heads[p] * n_r * d for p in range(W)]
        out_splits = [3 * B * h_r * self.tokens[p] * d for p in range(W)]
        recv = torch.empty(sum(out_splits), dtype=q.dtype, device=q.device)
        dist.all_to_all_single(recv, send, out_splits, in_splits, group=self.group)
        # 2. the whole call on this rank's heads
        if h_r > 0:
            parts = [c.view(3, B, h_r, self.tokens[p], d) for p, c in enumerate(recv.split(out_splits))]
            qkv = torch.cat(parts, dim=3)                     # [3, B, h_r, N, d]
            o_local = self.local(qkv[0].contiguous(), qkv[1].contiguous(), qkv[2].contiguous())
            if isinstance(o_local, tuple):
                o_local = o_local[0]
            send_o = torch.cat([o_local[:, :, self.token0[p]:self.token0[p] + self.tokens[p]].reshape(-1)
                                for p in range(W)])
        else:
            send_o = torch.empty(0, dtype=q.dtype, device=q.device)
        # 3. head shard -> token shard: O in one exchange
        in_o = [B * h_r * self.tokens[p] * d for p in range(W)]
        out_o = [B * self.heads[p] * n_r * d for p in range(W)]
        recv_o = torch.empty(sum(out_o), dtype=q.dtype, device=q.device)
        dist.all_to_all_single(recv_o, send_o, out_o, in_o, group=self.group)
        return torch.cat([c.view(B, self.heads[p], n_r, d) for p, c in enumerate(recv_o.split(out_o))], dim=1)

    def exchange_bytes(self, element_size: int) -> int:
        """Bytes this rank sends per call (both exchanges, to other ranks only)."""
        r, B, d = self.rank, self.B, self.d
        qkv = sum(3 * B * self.heads[p] * self.tokens[r] * d for p in range(self.world) if p != r)
        o = sum(B * self.heads[r] * self.tokens[p] * d for p in range(self.world) if p != r)
        return (qkv + o) * element_size
