"""Sequence-parallel attention (token shards in, token shards out, head shards for the call;
"OSP-Next" page, "Method": Sparse Sequence Parallelism) run as world-size-2 gloo process
groups on CPU.  The local call on each rank is the fp64 oracle for that rank's heads, so the
gathered output must equal the single-process oracle result exactly: the exchange only moves
values."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from block_sparse_attention_31_b200.sequence_parallel import SequenceParallelAttention, split_even

F, HL, WL, D, BLOCK, H = 3, 5, 7, 16, 32, 3     # N = 105 tokens: shards of 53 and 52; heads 2 and 1
W_S, W_T = 0, 2


def _inputs():
    g = torch.Generator().manual_seed(4)
    N = F * HL * WL
    return [torch.randn(1, H, N, D, generator=g, dtype=torch.float64) for _ in range(3)]


def _oracle_head(q, k, v, h):
    """Head h (global index): even heads spatial, odd temporal, fixed windows."""
    kind = oracle.SPATIAL if h % 2 == 0 else oracle.TEMPORAL
    keep = oracle.pattern_keep(kind, F, HL, WL, BLOCK, W_S if kind == oracle.SPATIAL else W_T)
    slots = oracle.layout_slots(kind, F, HL, WL)
    out, _ = oracle.attention_rows(q, k, v, slots, BLOCK, keep, scale=1.0 / math.sqrt(D))
    return torch.from_numpy(out)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v = _inputs()
        holder = {}

        def local(ql, kl, vl):
            h0 = holder["ssp"].head_offset
            return torch.stack([_oracle_head(ql[0, i], kl[0, i], vl[0, i], h0 + i) for i in range(ql.shape[1])])[None]

        ssp = SequenceParallelAttention(1, H, F, HL, WL, D, BLOCK, local_attention=local)
        holder["ssp"] = ssp
        t0, n = ssp.token0[rank], ssp.tokens[rank]
        o = ssp(*(x[:, :, t0:t0 + n].contiguous() for x in (q, k, v)))
        out[rank] = (t0, n, o.numpy(), ssp.exchange_bytes(8))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_split_even():
    assert split_even(12, 8) == [2, 2, 2, 2, 1, 1, 1, 1]
    assert split_even(24, 8) == [3] * 8
    assert split_even(105, 2) == [53, 52]
    assert split_even(3, 4) == [1, 1, 1, 0]


def test_sequence_parallel_gloo_matches_single_process_oracle():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    q, k, v = _inputs()
    want = torch.stack([_oracle_head(q[0, h], k[0, h], v[0, h], h) for h in range(H)]).numpy()
    got = np.zeros_like(want)
    for rank in range(world):
        t0, n, o, _ = out[rank]
        assert o.shape == (1, H, n, D)
        got[:, t0:t0 + n] = o[0]
    assert np.array_equal(got, want)
    # bytes sent per call: rank 0 sends Q, K, V rows of head 2 (rank 1's) and O rows of heads 0-1
    # for rank 1's tokens
    assert out[0][3] == (3 * 1 * 1 * 53 * D + 1 * 2 * 52 * D) * 8
