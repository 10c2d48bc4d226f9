"""The collective choreography of vocabulary-parallel verification, on CPU with
two gloo ranks.  The per-rank phases (CUDA kernels, tested on the GPU against
the single-rank run) are replaced by stand-ins that record what they were given,
so this checks what only the multi-rank path does: the block sizes and order of
the all-gathers, the MAX of the votes, and the gathering of a request's full
rows (shards of unequal widths, padded and cut back) for a whole redo."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from speculative_decoding_verification_86_b200 import binding

B, K, V = 6, 2, 40000  # fp32: 3 segments of 16384 -> two ranks of unequal width


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _full_logits():
    g = torch.Generator().manual_seed(3)
    return (torch.randn(B, K + 1, V, generator=g), torch.randn(B, K, V, generator=g))


class _FakeVerifier:
    device = torch.device("cpu")

    def __init__(self, log):
        self.log = log

    def _outputs(self, B_, k, with_pq=True):
        return dict(accepted=torch.zeros(B_, dtype=torch.int32),
                    tokens=torch.full((B_, k + 1), -1, dtype=torch.int32),
                    status=torch.zeros(B_, dtype=torch.int32),
                    p=torch.zeros((B_, k)), q=torch.zeros((B_, k)))

    def run(self, target, draft, tokens, **kw):
        self.log.append(("redo", target.clone(), draft.clone(), kw["request_offset"]))
        o = self._outputs(1, K)
        o["accepted"][0] = 77
        return o


class _FakeRank:
    """Phases that leave recognisable bytes in the exchange blocks."""

    def __init__(self, rank, n):
        self.rank, self.n = rank, n
        self.log = []
        self.ver = _FakeVerifier(self.log)
        self.device = torch.device("cpu")

    def stats(self, target, draft, tokens, V_, block1, **kw):
        block1.fill_(10 + self.rank)
        self.log.append(("shard", target.shape[2]))

    def decide(self, blocks1, target, draft, tokens, V_, out, block2, **kw):
        n1 = blocks1.numel() // self.n
        for r in range(self.n):  # every rank's block, in rank order
            assert torch.all(blocks1[r * n1:(r + 1) * n1] == 10 + r)
        out["accepted"].fill_(1)
        block2.fill_(20 + self.rank)

    def locate(self, blocks2, target, draft, tokens, V_, votes, **kw):
        n2 = blocks2.numel() // self.n
        for r in range(self.n):
            assert torch.all(blocks2[r * n2:(r + 1) * n2] == 20 + r)
        # request i's token is held by rank i % n; request 0 needs refinement
        for i in range(B):
            votes[i] = (100 * self.rank + i) if (i % self.n == self.rank and i != 0) else -2
        votes[0] = -1

    def finish(self, votes_max, out):
        self.log.append(("votes", votes_max.clone()))
        redo = torch.zeros(B, dtype=torch.int32)
        redo[0] = 2
        return redo

    def refine_partials(self, target, draft, tokens, V_, block3, **kw):
        block3.fill_(30 + self.rank)

    def refine_locate(self, blocks3, target, draft, tokens, V_, votes, **kw):
        n3 = blocks3.numel() // self.n
        for r in range(self.n):
            assert torch.all(blocks3[r * n3:(r + 1) * n3] == 30 + r)
        votes.fill_(-2)
        votes[0] = -1  # the refinement could not settle it: redo request 0 whole

    def refine_finish(self, votes_max, out):
        redo = torch.zeros(B, dtype=torch.int32)
        redo[0] = 1
        return redo


def _worker(rank, n, port, q, redo_whole=True):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=n)
    try:
        target, draft = _full_logits()
        bounds, _, _, _ = binding.shard_layout(B, K, V, torch.float32, n)
        lo, hi = bounds[rank], bounds[rank + 1]
        rk = _FakeRank(rank, n)
        tokens = torch.zeros((B, K), dtype=torch.int32)
        out = binding.verify_vocab_parallel(rk, target[:, :, lo:hi].contiguous(),
                                            draft[:, :, lo:hi].contiguous(), tokens, V,
                                            seed=5, request_offset=40, redo_whole=redo_whole)
        votes = [e[1] for e in rk.log if e[0] == "votes"][0]
        redo = [e for e in rk.log if e[0] == "redo"]
        q.put((rank, bounds, votes.tolist(), out["accepted"].tolist(),
               [(t.numpy(), d.numpy(), off) for _, t, d, off in redo], out["redo"].tolist()))
    finally:
        dist.destroy_process_group()


def test_two_rank_choreography():
    n = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, n, port, q)) for r in range(n)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(n)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    target, draft = _full_logits()
    for rank, bounds, votes, accepted, redo, flags in got:
        assert bounds[0] == 0 and bounds[-1] == V and bounds[1] - bounds[0] != bounds[2] - bounds[1]
        # the MAX picks the holder's vote; request 0 went on to the refinement
        assert votes[0] == -1
        assert votes[1:] == [100 * (i % n) + i for i in range(1, B)]
        # the whole redo of request 0 saw its full rows, gathered in vocabulary order
        assert len(redo) == 1
        t, d, off = redo[0]
        np.testing.assert_array_equal(t, target[0:1].numpy())
        np.testing.assert_array_equal(d, draft[0:1].numpy())
        assert off == 40
        assert accepted[0] == 77 and accepted[1:] == [1] * (B - 1)


def test_two_rank_step_without_host_redo():
    """redo_whole=False: every phase runs (the refinement included) and the
    request that needs rows of every rank is only flagged in out["redo"]."""
    n = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, n, port, q, False)) for r in range(n)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(n)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, bounds, votes, accepted, redo, flags in got:
        assert len(redo) == 0                     # nothing verified whole on the host
        assert flags[0] == 1 and flags[1:] == [0] * (B - 1)
        assert accepted == [1] * B
