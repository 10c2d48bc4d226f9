"""The prefix order's dense tail (spec_verify_set_prefix_tail) against the fp64
oracle: from every switch position the outputs are the oracle's, element by
element -- the tail changes which rows are read and when, never the result.

Position 1 reads all of a request's later positions together once position 0
accepted; position k reads the bonus row alone; 17 (above every k here) reads
each position separately, the plain prefix order; 0 lets the library choose.
"""
import numpy as np
import pytest
import torch

from parity_helpers import compare, run_oracle
from speculative_decoding_verification_86_b200 import binding, build, workloads

pytestmark = pytest.mark.gpu

TAILS = [0, 1, 2, 3, 5, 17]


@pytest.fixture(scope="module")
def ver(cuda_device):
    build.build()
    v = binding.SpecVerifier(cuda_device, max_batch=256, max_k=16, max_vocab=262144, mode="prefix")
    yield v
    v.close()


def run_gpu(ver, w, tail):
    ver.set_prefix_tail(tail)
    o = ver.run(w["target"], w.get("draft"), w["tokens"], verify_len=w.get("verify_len"),
                temperature=w.get("temperature"), conf=w.get("conf"), seed=w["seed"])
    torch.cuda.synchronize()
    c = ver.last_counters()
    assert c["engine_error"] == 0 and c["wait_fail"] == 0
    return {k: v.cpu().numpy() for k, v in o.items()}


@pytest.mark.parametrize("tail", TAILS)
def test_stochastic_mixed_lengths(ver, tail):
    w = workloads.stochastic("cuda", seed=1)
    compare(run_gpu(ver, w, tail), run_oracle(w))


@pytest.mark.parametrize("tail", TAILS)
def test_every_position_accepted_mixed_temperatures(ver, tail):
    """draft == target: every verified position of a sampled request is
    accepted, so each with L_i >= tail runs its whole tail; greedy requests
    (T = 0, which accept only the target's arg-max) mixed in."""
    w = workloads.stochastic("cuda", seed=5, B=48, k=5, V=20000)
    w["draft"] = w["target"][:, :5].contiguous()
    temps = [0.0, 0.7, 1.0, 1.3] * 12
    w["temperature"] = torch.tensor(temps, device="cuda")
    g, o = run_gpu(ver, w, tail), run_oracle(w)
    compare(g, o)
    sampled = np.array(temps) > 0
    full = np.clip(w["verify_len"].cpu().numpy(), 0, 5)
    assert np.array_equal(g["accepted"][sampled], full[sampled])


@pytest.mark.parametrize("tail", [1, 3, 17])
def test_greedy_b256(ver, tail):
    w = workloads.greedy("cuda", seed=2)
    g, o = run_gpu(ver, w, tail), run_oracle(w)
    np.testing.assert_array_equal(g["accepted"], o["accepted"])
    np.testing.assert_array_equal(g["tokens"], o["tokens"])


@pytest.mark.parametrize("tail", [1, 3])
def test_headline_b256(ver, tail):
    w = workloads.headline("cuda", seed=1)
    compare(run_gpu(ver, w, tail), run_oracle(w))


@pytest.mark.parametrize("tail", [1, 2, 8])
def test_confidence_head(ver, tail):
    """The head's budgets are known only once position 0 is in; the tail's
    plan takes them from there."""
    w = workloads.confidence("cuda", seed=3)
    compare(run_gpu(ver, w, tail), run_oracle(w))


@pytest.mark.parametrize("tail", [1, 2, 4])
def test_errors_inside_the_tail(ver, tail):
    """Every position accepted (draft == target), with a fault planted at a
    later position, where the tail's walk meets it."""
    w = workloads.stochastic("cuda", seed=9, B=8, k=5, V=4096, fixed_len=5)
    w["draft"] = w["target"][:, :5].contiguous().clone()
    t, d = w["target"], w["draft"]
    t[0, 4, 17] = float("nan")   # NaN in target row 4
    d[1, 3, 5] = float("inf")    # +inf in draft row 3
    t[2, 5, :] = float("-inf")   # the bonus row all masked
    w["tokens"][3, 3] = 4096     # out of range at position 3
    w["tokens"][4, 4] = -1       # negative at position 4
    g, o = run_gpu(ver, w, tail), run_oracle(w)
    compare(g, o)
    assert list(g["status"][:5]) == [2, 2, 2, 1, 1]
    assert np.all(g["status"][5:] == 0) and np.all(g["accepted"][5:] == 5)


def test_out_of_range_positions_are_refused(ver):
    for bad in (-1, 18):
        with pytest.raises(binding.SpecVerifyError):
            ver.set_prefix_tail(bad)
    ver.set_prefix_tail(0)
