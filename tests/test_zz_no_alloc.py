"""spec_verify_greedy_noalloc -- greedy verification for callers that may not
allocate device memory (for example a serving engine that has already reserved
nearly all free GPU memory for its KV cache, or a plugin host that only lends a
stream and buffers).  Its working space is a fixed array inside the library.

Checked through the C ABI against spec_verify_greedy (which uses a context's
workspace) on two calls in a row with different inputs, so a stale array from
the first call would show up in the second, and against the fp64 CPU oracle at
temperature 0 directly: the greedy benchmark batch, a bf16 batch with many tied
maxima, the failure paths (tokens out of range, NaN and +inf in a row the chain
reads, a row of only masked logits, NaN in a row it does not read), k = 0 with
no drafted tokens, and fp32 logits at the largest accepted vocabulary.  Greedy
results must match exactly.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from parity_helpers import host, run_oracle
from speculative_decoding_verification_86_b200 import binding, build, workloads

pytestmark = pytest.mark.gpu


def _host(o):
    return {k: v.cpu().numpy() for k, v in o.items()}


def test_noalloc_greedy_matches_context_entry_point(cuda_device):
    build.build()
    calls = [
        workloads.greedy(cuda_device, seed=31, B=256, k=5, V=151936),
        workloads.greedy(cuda_device, seed=32, B=40, k=8, V=262144),
    ]
    calls[1]["verify_len"] = torch.randint(0, 9, (40,), dtype=torch.int32, device=cuda_device)
    with binding.SpecVerifier(cuda_device, max_batch=256, max_k=8, max_vocab=262144) as ver:
        for w in calls:
            ref = _host(ver.greedy(w["target"], w["tokens"], verify_len=w["verify_len"]))
            # outputs start as garbage, so every element must be written
            B, k = w["tokens"].shape
            out = dict(accepted=torch.full((B,), 77, dtype=torch.int32, device=cuda_device),
                       tokens=torch.full((B, k + 1), 77, dtype=torch.int32, device=cuda_device),
                       status=torch.full((B,), 77, dtype=torch.int32, device=cuda_device))
            got = _host(binding.greedy_noalloc(w["target"], w["tokens"], verify_len=w["verify_len"],
                                               out=out))
            torch.cuda.synchronize()
            for key in ("accepted", "tokens", "status"):
                np.testing.assert_array_equal(got[key], ref[key], err_msg=key)
            assert np.all(got["status"] == 0)


def test_noalloc_rejects_sizes_beyond_its_array(cuda_device):
    build.build()
    t = torch.zeros((257, 2, 64), dtype=torch.bfloat16, device=cuda_device)
    x = torch.zeros((257, 1), dtype=torch.int32, device=cuda_device)
    with pytest.raises(binding.SpecVerifyError) as e:
        binding.greedy_noalloc(t, x)
    assert e.value.status == binding.SPEC_ERR_INVALID_ARG
    t = torch.zeros((256, 9, 8), dtype=torch.float32, device=cuda_device)   # k = 8, V fine
    x = torch.zeros((256, 8), dtype=torch.int32, device=cuda_device)
    binding.greedy_noalloc(t, x)
    big = torch.zeros((4, 10, 8), dtype=torch.float32, device=cuda_device)  # k = 9 > 8
    with pytest.raises(binding.SpecVerifyError):
        binding.greedy_noalloc(big, torch.zeros((4, 9), dtype=torch.int32, device=cuda_device))


def _noalloc_vs_oracle(w):
    """Run the allocation-free entry point on workload ``w`` (greedy) and
    compare every output with the oracle at T = 0, bit for bit."""
    B, kp1, _ = w["target"].shape
    got = host(binding.greedy_noalloc(w["target"], w["tokens"], verify_len=w.get("verify_len")))
    torch.cuda.synchronize()
    o = run_oracle(dict(w, draft=None, temperature=torch.zeros(B, dtype=torch.float32,
                                                                 device=w["target"].device)))
    np.testing.assert_array_equal(got["accepted"], o["accepted"])
    np.testing.assert_array_equal(got["tokens"], o["tokens"])
    np.testing.assert_array_equal(got["status"].astype(np.uint32), o["status"])
    return o


def _tied(dev, seed, B, k, V, dtype=torch.bfloat16, sigma=1.0, step=None):
    """Logits N(0, sigma^2) in ``dtype``; with ``step`` they are rounded to
    multiples of it first, so many rows hold their maximum more than once and
    the lowest-index rule decides."""
    g = torch.Generator(device=dev).manual_seed(seed)
    target = torch.randn((B, k + 1, V), generator=g, device=dev) * sigma
    if step is not None:
        target = torch.round(target / step) * step
    target = target.to(dtype)
    first = torch.argmax(target[:, :k].float(), dim=-1).to(torch.int32)
    coin = torch.rand((B, k), generator=g, device=dev) < 0.7
    rnd = torch.randint(0, V, (B, k), generator=g, device=dev, dtype=torch.int32)
    tokens = torch.where(coin, first, rnd).to(torch.int32).contiguous()
    return dict(target=target.contiguous(), draft=None, tokens=tokens, verify_len=None,
                temperature=None, conf=None, seed=seed)


def test_noalloc_greedy_matches_oracle(cuda_device):
    build.build()
    # the greedy benchmark batch: B=256, k=5, V=151936 bf16
    o = _noalloc_vs_oracle(workloads.greedy(cuda_device, seed=2))
    assert (o["accepted"] < 5).any() and (o["accepted"] == 5).any()
    # many tied maxima; verify_len outside [0, k] is clamped
    w = _tied(cuda_device, 41, B=96, k=5, V=4096, step=0.5)
    vals = w["target"].float()
    tied_rows = (vals == vals.amax(dim=-1, keepdim=True)).sum(dim=-1) > 1
    assert tied_rows.float().mean().item() > 0.2
    w["verify_len"] = torch.randint(-2, 8, (96,), generator=torch.Generator(device=cuda_device)
                                    .manual_seed(42), device=cuda_device, dtype=torch.int32)
    _noalloc_vs_oracle(w)


def test_noalloc_failure_paths_match_oracle(cuda_device):
    build.build()
    for dtype in (torch.bfloat16, torch.float32):
        w = _tied(cuda_device, 43, B=12, k=3, V=4096, dtype=dtype, sigma=2.0)
        t, x = w["target"], w["tokens"]
        first = torch.argmax(t.float(), dim=-1).to(torch.int32)
        x[:, :] = first[:, :3]          # every drafted token agrees: the chain reads every row
        x[0, 1] = -3                    # token below the vocabulary
        x[1, 0] = 4096                  # token past the vocabulary
        t[2, 1, 77] = float("nan")      # NaN in a row the chain reads
        t[3, 3, 5] = float("inf")       # +inf in the bonus row
        t[4, 0, :] = float("-inf")      # a row of only masked logits
        x[5, 0] = (first[5, 0] + 1) % 4096  # rejected at position 0 ...
        t[5, 2, 9] = float("nan")       # ... so this NaN is never read
        o = _noalloc_vs_oracle(w)
        assert list(o["accepted"][:6]) == [-1, -1, -1, -1, -1, 0]
        assert (o["status"][:5] != 0).all() and (o["status"][5:] == 0).all()


def test_noalloc_zero_block_and_largest_fp32_vocabulary(cuda_device):
    build.build()
    g = torch.Generator(device=cuda_device).manual_seed(44)
    # k = 0: no drafted tokens at all; every request emits the arg-max of row 0
    t0 = torch.randn((7, 1, 2048), generator=g, device=cuda_device).to(torch.bfloat16)
    w0 = dict(target=t0, draft=None, tokens=None, verify_len=None, temperature=None, conf=None, seed=0)
    got = host(binding.greedy_noalloc(t0, None))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(got["accepted"], 0)
    np.testing.assert_array_equal(got["tokens"][:, 0], torch.argmax(t0[:, 0].float(), dim=-1).cpu().numpy())
    o = run_oracle(dict(w0, tokens=torch.zeros((7, 0), dtype=torch.int32, device=cuda_device),
                        temperature=torch.zeros(7, dtype=torch.float32, device=cuda_device)))
    np.testing.assert_array_equal(got["tokens"], o["tokens"])
    # fp32 at the largest vocabulary the array takes at B = 256, k = 8
    w = _tied(cuda_device, 45, B=256, k=8, V=131072, dtype=torch.float32, sigma=3.0)
    _noalloc_vs_oracle(w)
    with pytest.raises(binding.SpecVerifyError):
        binding.greedy_noalloc(torch.zeros((256, 9, 131080), dtype=torch.float32, device=cuda_device),
                               torch.zeros((256, 8), dtype=torch.int32, device=cuda_device))
