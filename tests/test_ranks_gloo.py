"""Multi-rank logic on CPU: two gloo ranks shard a batch by request and must
reproduce the single-call result (the oracle stands in for each rank's GPU
verification); the timing reduction takes the max over ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from speculative_decoding_verification_86_b200 import ranks


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(B, k, V, seed):
    g = torch.Generator().manual_seed(seed)
    target = torch.randn(B, k + 1, V, generator=g) * 2
    draft = target[:, :k] + torch.randn(B, k, V, generator=g)
    tokens = torch.randint(0, V, (B, k), generator=g, dtype=torch.int32)
    temp = torch.tensor([0.0, 0.7, 1.0], dtype=torch.float32)[torch.randint(0, 3, (B,), generator=g)]
    vlen = torch.randint(0, k + 1, (B,), generator=g, dtype=torch.int32)
    return [t.numpy() for t in (target.float(), draft.float(), tokens, temp, vlen)]


def _verify(oracle, inp, lo, hi, offset):
    target, draft, tokens, temp, vlen = inp
    return oracle.verify(target[lo:hi], draft[lo:hi], tokens[lo:hi], dtype=oracle.DTYPE_F32,
                         verify_len=vlen[lo:hi], temperature=temp[lo:hi], seed=77,
                         request_offset=offset)


def _worker(rank, world, port, B, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        inp = _inputs(B, 4, 48, seed=3)
        # strong split of one batch
        lo, hi = ranks.shard_bounds(B, world, rank)
        part = _verify(oracle, inp, lo, hi, lo)
        parts = [None] * world
        dist.all_gather_object(parts, {k: part[k] for k in ("accepted", "tokens", "p_x")})
        # weak scaling: every rank verifies the same B inputs as its own block
        # of a world*B batch
        weak = _verify(oracle, inp, 0, B, ranks.weak_offset(B, rank))
        weaks = [None] * world
        dist.all_gather_object(weaks, {k: weak[k] for k in ("accepted", "tokens")})
        m = ranks.max_over_ranks(10.0 + rank)
        if rank == 0:
            q.put((parts, weaks, m))
    finally:
        dist.destroy_process_group()


def test_sharded_batch_equals_single_call(oracle_lib):
    world, B = 2, 13
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, B, q)) for r in range(world)]
    for p in procs:
        p.start()
    parts, weaks, m = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp = _inputs(B, 4, 48, seed=3)
    full = _verify(oracle_lib, inp, 0, B, 0)
    for key in ("accepted", "tokens", "p_x"):
        np.testing.assert_array_equal(np.concatenate([p[key] for p in parts]), full[key])
    # the weak-scaling batch is the inputs repeated once per rank
    rep = [np.concatenate([a] * world) for a in inp]
    big = _verify(oracle_lib, rep, 0, world * B, 0)
    for key in ("accepted", "tokens"):
        np.testing.assert_array_equal(np.concatenate([w[key] for w in weaks]), big[key])
    assert m == 11.0


def test_shard_bounds_cover_the_batch():
    for total in (0, 1, 7, 256, 1000):
        for world in (1, 2, 3, 8):
            b = [ranks.shard_bounds(total, world, r) for r in range(world)]
            assert b[0][0] == 0 and b[-1][1] == total
            assert all(b[r][1] == b[r + 1][0] for r in range(world - 1))
            assert max(h - l for l, h in b) - min(h - l for l, h in b) <= 1
    with pytest.raises(ValueError):
        ranks.shard_bounds(4, 2, 2)
    assert ranks.max_over_ranks(3.5) == 3.5
