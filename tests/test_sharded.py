"""Head-sharded forward for sequence-sharded inputs (the pages' 14B recipe
splits the token sequence over 4 GPUs): the seq -> heads -> seq exchange on
CPU ranks over gloo.  Bit-exact against slicing the unsharded tensor; no GPU
needed (the attention between the two exchanges is covered by the GPU parity
tests, which run the same library calls on a head subset)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_attention_30_b200 import sharded


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, shape, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, N, heads, d = shape
        g = torch.Generator().manual_seed(7)
        full = torch.randn(shape, generator=g).to(torch.bfloat16)    # same on every rank
        Nl, hl = N // world, heads // world
        mine = full[:, rank * Nl:(rank + 1) * Nl].contiguous()
        hs = sharded.seq_to_heads(mine)
        ok_heads = torch.equal(hs, full[:, :, rank * hl:(rank + 1) * hl])
        back = sharded.heads_to_seq(hs)
        ok_back = torch.equal(back, mine)
        # a head-wise operation between the exchanges lands on the right tokens
        scaled = sharded.heads_to_seq(hs * (rank + 2))
        want = torch.cat([full[:, rank * Nl:(rank + 1) * Nl, r * hl:(r + 1) * hl] * (r + 2)
                          for r in range(world)], dim=2)
        ok_op = torch.equal(scaled, want)
        results[rank] = (ok_heads, ok_back, ok_op, tuple(hs.shape), tuple(back.shape))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,shape", [(2, (1, 24, 4, 8)), (2, (2, 20, 6, 16)), (4, (1, 32, 8, 8))])
def test_seq_heads_exchange_is_exact(world, shape):
    ctx = mp.get_context("spawn")
    results = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, shape, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    B, N, heads, d = shape
    for r in range(world):
        ok_heads, ok_back, ok_op, hs_shape, back_shape = results[r]
        assert ok_heads and ok_back and ok_op, (r, results[r])
        assert hs_shape == (B, N, heads // world, d) and back_shape == (B, N // world, heads, d)


def test_exchange_bytes():
    # 14B-480P on 4 ranks: each rank sends 3/4 of its three input shards and
    # of its output shard
    shard = 29120 // 4 * 40 * 128 * 2
    assert sharded.exchange_bytes(1, 29120, 40, 128, 4) == 4 * shard * 3 // 4
    assert sharded.exchange_bytes(1, 29120, 40, 128, 1) == 0
