"""The device's Philox4x32-10 draws against the oracle's independent
implementation (itself pinned to cuRAND's host generator on the CPU),
bit for bit, over more than 10^6 counters."""
import numpy as np
import pytest

import oracle
from speculative_decoding_verification_86_b200 import binding, build

pytestmark = pytest.mark.gpu


def test_device_draws_match_the_oracle_generator(cuda_device):
    build.build()
    v = binding.SpecVerifier(cuda_device, max_batch=8, max_k=8, max_vocab=1024)
    try:
        B, k = 120000, 4  # 1.2 M draws per (seed, step)
        for seed, step in ((0, 0), (0x123456789ABCDEF0, 7), (1, 0xFFFFFFFF)):
            got = v.draws(B, k, seed=seed, step=step).cpu().numpy()
            for d in (0, 1):
                np.testing.assert_array_equal(got[:, :, d], oracle.uniform_grid(seed, B, k + 1, d, step))
        got = v.draws(4, 2, seed=9, step=1, request_offset=1000).cpu().numpy()
        for i in range(4):
            for j in range(3):
                for d in range(2):
                    assert got[i, j, d] == oracle.uniform(9, 1000 + i, j, d, 1)
    finally:
        v.close()
