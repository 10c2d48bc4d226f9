"""CPU pins of the oracle's batch-wide verify budget.

The load-aware form of the confidence rule ("Speculative decoding becomes
standard: DSpark and multi-token drafters", section "What DSpark adds": how
many positions to verify follows the head's survival estimates and the load of
the batch) keeps, among every request's candidate positions, the `total` ones
with the largest prefix survival, ties to the lower request and then the lower
position.  The oracle writes that definition as a sort; these tests pin it to
what fixes it independently of any sort:

- brute force: with distinct survivals, the kept set is the unique way of
  spending the budget on leading runs that maximises the summed survival;
- a static threshold is the special case in which the budget equals the number
  of positions at or above it;
- the extremes (budget 0, budget >= candidates) and the tie order.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle


def _prefix(rng, B, kb):
    s = rng.uniform(0.05, 1.0, size=(B, kb))
    return np.cumprod(s, axis=1)


def _brute_force(P, cap, total):
    B = P.shape[0]
    want = min(total, int(cap.sum()))
    best, arg = None, None
    for L in itertools.product(*[range(c + 1) for c in cap]):
        if sum(L) != want:
            continue
        val = sum(P[i, :L[i]].sum() for i in range(B))
        if best is None or val > best + 1e-15:
            best, arg = val, L
        elif abs(val - best) <= 1e-15:
            raise AssertionError("brute force found two optima: inputs have ties")
    return np.array(arg, dtype=np.int32)


@pytest.mark.parametrize("seed", range(12))
def test_topn_is_the_max_survival_allocation(oracle_lib, seed):
    rng = np.random.default_rng(seed)
    B, kb = int(rng.integers(1, 5)), int(rng.integers(1, 5))
    P = _prefix(rng, B, kb)
    cap = rng.integers(0, kb + 1, size=B).astype(np.int32)
    for total in range(0, int(cap.sum()) + 2):
        got = oracle.budget_topn(P, cap, total)
        assert np.array_equal(got, _brute_force(P, cap, total)), (total, cap)


def test_topn_extremes_and_sum(oracle_lib):
    rng = np.random.default_rng(7)
    P = _prefix(rng, 50, 8)
    cap = rng.integers(0, 9, size=50).astype(np.int32)
    assert np.array_equal(oracle.budget_topn(P, cap, 0), np.zeros(50, np.int32))
    assert np.array_equal(oracle.budget_topn(P, cap, int(cap.sum())), cap)
    assert np.array_equal(oracle.budget_topn(P, cap, 10 ** 12), cap)
    for total in (1, 17, 100, int(cap.sum()) - 1):
        L = oracle.budget_topn(P, cap, total)
        assert L.sum() == min(total, cap.sum())
        assert np.all(L <= cap)
        # every kept survival is at least every dropped candidate's
        kept = [P[i, j] for i in range(50) for j in range(L[i])]
        dropped = [P[i, j] for i in range(50) for j in range(L[i], cap[i])]
        if kept and dropped:
            assert min(kept) >= max(dropped)


def test_static_threshold_is_a_special_case(oracle_lib):
    rng = np.random.default_rng(11)
    B, kb = 200, 8
    P = _prefix(rng, B, kb)
    cap = np.full(B, kb, dtype=np.int32)
    for tau in (0.9, 0.5, 0.3, 0.1, 0.01):
        lead = (P >= tau).astype(int).cumprod(axis=1).sum(axis=1)
        L = oracle.budget_topn(P, cap, int(lead.sum()))
        assert np.array_equal(L, lead)


def test_ties_go_to_lower_request_then_lower_position(oracle_lib):
    P = np.array([[0.5, 0.5, 0.25],
                  [0.5, 0.5, 0.5],
                  [0.75, 0.5, 0.5]])
    cap = np.array([3, 3, 3], dtype=np.int32)
    # order: (2,0) 0.75; then the 0.5s by (request, position):
    # (0,0) (0,1) (1,0) (1,1) (1,2) (2,1) (2,2); then (0,2) 0.25
    expect = {1: [0, 0, 1], 2: [1, 0, 1], 3: [2, 0, 1], 4: [2, 1, 1], 6: [2, 3, 1],
              7: [2, 3, 2], 8: [2, 3, 3], 9: [3, 3, 3]}
    for total, L in expect.items():
        assert oracle.budget_topn(P, cap, total).tolist() == L, total


def test_verify_lengths_apply_the_budget_after_the_per_request_limits(oracle_lib):
    """Through the whole oracle: L_i = top-N over the positions that survive
    verify_len and the per-request threshold; the threaded path (which fixes
    the lengths on the whole batch first) gives the same outputs."""
    g = torch.Generator().manual_seed(5)
    B, k, V, kb, H = 24, 6, 64, 6, 96
    h = torch.randn(B, kb, H, generator=g).to(torch.bfloat16)
    w = (torch.randn(H, generator=g) / math.sqrt(H) * 3).to(torch.bfloat16)
    hb = h.view(torch.int16).numpy().view(np.uint16)
    wb = w.view(torch.int16).numpy().view(np.uint16)
    bias, tau = 1.5, 0.05
    vlen = torch.randint(0, k + 2, (B,), generator=g).int().numpy()
    target = torch.randn(B, k + 1, V, generator=g).float().numpy()
    draft = (target[:, :k] + 0.5 * torch.randn(B, k, V, generator=g).float().numpy()).astype(np.float32)
    tokens = torch.randint(0, V, (B, k), generator=g).int().numpy()
    static, _, pref = oracle.conf_budget(hb, wb, bias, tau)
    cap = np.minimum(np.clip(vlen, 0, k), static).astype(np.int32)
    for total in (0, 1, 9, int(cap.sum()) // 2, int(cap.sum()), 1000):
        conf = dict(hidden=hb, w=wb, bias=bias, threshold=tau, total=total)
        res = oracle.verify(target, draft, tokens, dtype=oracle.DTYPE_F32, verify_len=vlen,
                            conf=conf, seed=9)
        want = cap if total <= 0 else oracle.budget_topn(pref, cap, total)
        assert np.array_equal(res["verify_len_used"], want), total
        res4 = oracle.verify(target, draft, tokens, dtype=oracle.DTYPE_F32, verify_len=vlen,
                             conf=conf, seed=9, threads=4)
        for key in ("accepted", "tokens", "verify_len_used", "status"):
            assert np.array_equal(res[key], res4[key]), key
        np.testing.assert_array_equal(res["p_x"], res4["p_x"])
