"""Vocabulary-parallel verification (logits split by vocabulary over ranks),
run on one device: every rank is its own context with its slice of the
logits, the all-gathers are concatenations and the max over ranks a torch.max
(no kernel waits on another).  Every case is checked twice: against the fp64
CPU oracle on the same inputs (the same bar as the single-rank parity tests),
and against the single-rank run element for element, since the merged
statistics records of the ranks equal the single-rank records exactly."""
import numpy as np
import pytest
import torch

from parity_helpers import compare, host, run_oracle
from speculative_decoding_verification_86_b200 import binding, build, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def single(cuda_device):
    build.build()
    v = binding.SpecVerifier(cuda_device, max_batch=1024, max_k=8, max_vocab=262144, mode="dense")
    yield v
    v.close()


def _ranks(dev, n, B, k, V):
    return [binding.ShardRank(dev, r, n, max_batch=B, max_k=max(k, 1), max_vocab=V) for r in range(n)]


def _check_equal(single_out, final, label):
    for key in ("accepted", "tokens", "status", "p", "q"):
        a = single_out[key].cpu().numpy()
        b = final[key].cpu().numpy()
        np.testing.assert_array_equal(a, b, err_msg="%s: %s" % (label, key))


def _run(single, w, n):
    dev = single.device
    B, kp1, V = w["target"].shape
    ranks = _ranks(dev, n, B, kp1 - 1, V)
    try:
        kw = dict(verify_len=w.get("verify_len"), temperature=w.get("temperature"), conf=w.get("conf"),
                  seed=w["seed"])
        ref = single.run(w["target"], w.get("draft"), w["tokens"], **kw)
        outs, final, info, votes = binding.emulate_vocab_parallel(ranks, w["target"], w.get("draft"),
                                                                  w["tokens"], **kw)
        torch.cuda.synchronize()
        # every rank reaches the same decisions before the token exchange
        for o in outs[1:]:
            for key in ("accepted", "status", "p", "q"):
                np.testing.assert_array_equal(o[key].cpu().numpy(), outs[0][key].cpu().numpy())
        # at most one rank answers with a token for each request
        v = votes.cpu().numpy()
        assert np.all((v >= 0).sum(axis=0) <= 1)
        _check_equal(ref, final, "n=%d" % n)
        # the sharded result against the oracle directly
        compare(host(final), run_oracle(w))
        return info
    finally:
        for r in ranks:
            r.close()


@pytest.mark.parametrize("n", [2, 3, 5])
def test_stochastic_b64_matches_single_rank(single, n):
    w = workloads.stochastic("cuda", seed=1)
    _run(single, w, n)


def test_headline_two_ranks(single):
    w = workloads.headline("cuda", seed=1)
    info = _run(single, w, 2)
    # the fp32 filter certifies most samples; the others go through the
    # vocabulary-parallel fp64 refinement, and none needs a whole redo here
    assert 0 < len(info["refined"]) < 64
    assert len(info["redone"]) == 0


def test_mixed_temperatures_and_greedy(single):
    w = workloads.sweep("cuda", seed=4, B=128)
    _run(single, w, 4)


def test_fp32_ragged_vocabulary(single):
    g = torch.Generator(device="cuda").manual_seed(11)
    B, k, V = 16, 3, 40000  # 3 segments of 16384 fp32 logits, the last ragged
    target = torch.randn(B, k + 1, V, generator=g, device="cuda") * 2
    draft = target[:, :k] + torch.randn(B, k, V, generator=g, device="cuda")
    tokens = torch.randint(0, V, (B, k), generator=g, device="cuda", dtype=torch.int32)
    w = dict(target=target.contiguous(), draft=draft.contiguous(), tokens=tokens, seed=5)
    for n in (2, 3):
        _run(single, w, n)


def test_confidence_head_and_errors(single):
    w = workloads.confidence("cuda", seed=3, B=32)
    # plant a NaN in one shard's half of a verified row and a bad token
    w["target"][3, 0, 200000] = float("nan")
    w["tokens"][5, 0] = -7
    _run(single, w, 2)


def test_layout_refuses_too_many_shards():
    with pytest.raises(binding.SpecVerifyError):
        binding.shard_layout(4, 2, 40000, torch.float32, 4)  # only 3 segments


def test_refinement_three_ranks(single):
    """The vocabulary-parallel fp64 refinement with the drawn sub-chunks spread
    over three ranks (the headline batch: 18 uncertified samples)."""
    w = workloads.headline("cuda", seed=1)
    info = _run(single, w, 3)
    assert len(info["refined"]) > 0 and len(info["redone"]) == 0
