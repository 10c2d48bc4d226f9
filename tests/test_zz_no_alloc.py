"""spec_verify_greedy_noalloc -- greedy verification for callers that may not
allocate device memory (for example a serving engine that has already reserved
nearly all free GPU memory for its KV cache, or a plugin host that only lends a
stream and buffers).  Its working space is a fixed array inside the library.

Checked through the C ABI against spec_verify_greedy (which uses a context's
workspace) on two calls in a row with different inputs, so a stale array from
the first call would show up in the second; greedy results must match exactly.
This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

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
