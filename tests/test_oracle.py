"""Pins for the fp64 CPU oracle, checked against things other than itself.

* Philox4x32-10 against cuRAND's host-side Philox generator (a library run
  on the CPU, no stored values), plus a uniformity chi-square.
* Row softmax against torch.softmax in fp64, greedy rows against torch.argmax
  (documented to return the first maximal index), the confidence budget
  against sigmoid(h @ w + b).cumprod in fp64.
* The exactness invariant of rejection sampling ("Speculative decoding becomes
  standard: DSpark and multi-token drafters", section "Why draft-and-verify does
  not change the output": the emitted tokens follow the target's law exactly)
  by exhaustive enumeration of draft tokens and of the oracle's
  own decision cells on tiny vocabularies, to 1e-12; the probability of
  reaching position j equals prod_{j'<j} sum_t min(p, q) (closed form).
* The same laws from 10^6 Philox-driven runs (chi-square, p > 1e-4).
"""
import ctypes
import ctypes.util
import itertools
import math

import numpy as np
import pytest
import torch

import oracle

F32, BF16 = oracle.DTYPE_F32, oracle.DTYPE_BF16


# ---------------------------------------------------------------- Philox ----

def _curand_stream(seed, offset_words, n_words):
    path = ctypes.util.find_library("curand") or "/usr/local/cuda/lib64/libcurand.so"
    try:
        cr = ctypes.CDLL(path)
    except OSError:
        pytest.skip("libcurand not available")
    gen = ctypes.c_void_p()
    PHILOX4_32_10 = 161
    if cr.curandCreateGeneratorHost(ctypes.byref(gen), PHILOX4_32_10) != 0:
        pytest.skip("cuRAND host generator unavailable")
    try:
        assert cr.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
        assert cr.curandSetGeneratorOffset(gen, ctypes.c_ulonglong(offset_words)) == 0
        buf = (ctypes.c_uint32 * n_words)()
        assert cr.curandGenerate(gen, buf, n_words) == 0
        return np.array(buf, dtype=np.uint32)
    finally:
        cr.curandDestroyGenerator(gen)


def _curand_block_counter(n):
    # cuRAND's host Philox4_32_10 generator (default ordering) spreads its output
    # over 65536 subsequences: block n is Philox(counter = (n >> 16 as a 64-bit
    # integer in words 0-1, n & 0xffff in word 2, 0), key = (seed low, seed high)).
    hi = n >> 16
    return [hi & 0xFFFFFFFF, (hi >> 32) & 0xFFFFFFFF, n & 0xFFFF, 0]


def _block_for_counter(c0, c1, c2):
    assert c2 < (1 << 16)
    return (((c1 << 32) + c0) << 16) + c2


@pytest.mark.parametrize("seed", [0, 1, 0xDEADBEEF, 0x123456789ABCDEF0])
def test_philox_matches_curand_host_generator(oracle_lib, seed):
    key = [seed & 0xFFFFFFFF, seed >> 32]
    starts = [0, 1, 65534, 65536, (1 << 32) + 7, _block_for_counter(9, 5, 0),
              _block_for_counter(0xFFFFFFFF, 16383, 65533)]
    for n0 in starts:
        words = _curand_stream(seed, 4 * n0, 12)
        for b in range(3):
            got = oracle.philox(_curand_block_counter(n0 + b), key)
            assert np.array_equal(got, words[4 * b:4 * b + 4]), (seed, n0 + b)


def test_uniform_uses_counter_layout_and_53_bits(oracle_lib):
    # U(seed, i, j, d, step) = 53-bit uniform from words 0 and 1 of
    # Philox(counter = (2j + d, i, step, 0), key = seed).
    seed = 0x5EED
    for i, j, d, step in [(0, 0, 0, 0), (0, 0, 1, 0), (3, 4, 0, 0), (255, 5, 1, 0),
                          (1023, 8, 1, 0), (16000, 7, 0, 3), (2, 1, 1, 65535)]:
        w = _curand_stream(seed, 4 * _block_for_counter(2 * j + d, i, step), 4)
        expect = ((int(w[0]) >> 5) * (1 << 26) + (int(w[1]) >> 6)) / float(1 << 53)
        assert oracle.uniform(seed, i, j, d, step) == expect


def test_uniform_range_and_chi_square(oracle_lib):
    from scipy import stats
    u = oracle.uniform_grid(seed=7, requests=125000, positions=4, draw=0).ravel()
    u2 = oracle.uniform_grid(seed=7, requests=125000, positions=4, draw=1).ravel()
    for x in (u, u2):
        assert x.min() >= 0.0 and x.max() < 1.0
        scaled = x * float(1 << 53)
        assert np.all(scaled == np.floor(scaled))
        counts, _ = np.histogram(x, bins=1000, range=(0.0, 1.0))
        assert stats.chisquare(counts).pvalue > 1e-4
    # the two draws of a position are different streams
    assert abs(np.corrcoef(u, u2)[0, 1]) < 5e-3


# ------------------------------------------------- row-level library pins ----

def _bf16_bits(x):
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _bf16_values(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()


@pytest.mark.parametrize("T", [1e-3, 0.7, 1.0, 2.5, 100.0])
def test_row_softmax_matches_torch_fp64(oracle_lib, T):
    rng = np.random.default_rng(11)
    for V in (1, 7, 1000, 4099):
        x32 = (rng.standard_normal(V) * 3).astype(np.float32)
        got = oracle.row_softmax(x32, F32, T)
        ref = torch.softmax(torch.from_numpy(x32).double() / T, dim=0).numpy()
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-300)
        xb = _bf16_bits(x32)
        got = oracle.row_softmax(xb, BF16, T)
        ref = torch.softmax(torch.from_numpy(_bf16_values(xb)) / T, dim=0).numpy()
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-300)


def test_row_softmax_masked_and_nonfinite(oracle_lib):
    x = np.array([0.5, -np.inf, 1.5, -np.inf], dtype=np.float32)
    got = oracle.row_softmax(x, F32, 1.0)
    ref = torch.softmax(torch.from_numpy(x).double(), dim=0).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-13)
    assert got[1] == 0.0 and got[3] == 0.0
    for bad in ([0.0, np.nan], [0.0, np.inf], [-np.inf, -np.inf]):
        with pytest.raises(ValueError):
            oracle.row_softmax(np.array(bad, dtype=np.float32), F32, 1.0)


def test_row_argmax_is_first_maximal_index(oracle_lib):
    rng = np.random.default_rng(5)
    for V in (1, 2, 17, 151936):
        xb = _bf16_bits((rng.standard_normal(V) * 3).astype(np.float32))
        vals = _bf16_values(xb)
        if V > 4:  # plant ties of the maximum at later indices
            m = vals.argmax()
            xb[(m + 3) % V] = xb[m]
            xb[(m + V // 2) % V] = xb[m]
        want = int(torch.argmax(torch.from_numpy(_bf16_values(xb))))
        assert want == int(np.argmax(_bf16_values(xb)))
        assert oracle.row_argmax(xb, BF16) == want
    # signed zeros compare equal: the lowest index wins
    x = np.array([-1.0, -0.0, 0.0, -2.0], dtype=np.float32)
    assert oracle.row_argmax(x, F32) == 1


def test_conf_budget_matches_torch_fp64(oracle_lib):
    g = torch.Generator().manual_seed(3)
    B, kb, H = 64, 8, 2560
    h = (torch.randn(B, kb, H, generator=g)).to(torch.bfloat16)
    w = (torch.randn(H, generator=g) / math.sqrt(H)).to(torch.bfloat16)
    bias, tau = 0.5, 0.3
    hb = h.view(torch.int16).numpy().view(np.uint16)
    wb = w.view(torch.int16).numpy().view(np.uint16)
    L, surv, pref = oracle.conf_budget(hb, wb, bias, tau)
    s_ref = torch.sigmoid(h.double() @ w.double() + bias)
    p_ref = torch.cumprod(s_ref, dim=1)
    np.testing.assert_allclose(surv, s_ref.numpy(), rtol=1e-12)
    np.testing.assert_allclose(pref, p_ref.numpy(), rtol=1e-12)
    lead = (p_ref >= tau).int().cumprod(dim=1).sum(dim=1).numpy()
    assert np.array_equal(L, lead)
    assert len(set(L.tolist())) > 1
    # thresholds at the extremes
    assert np.all(oracle.conf_budget(hb, wb, bias, 0.0)[0] == kb)
    assert np.all(oracle.conf_budget(hb, wb, bias, 1.5)[0] == 0)


def test_conf_budget_threshold_is_inclusive(oracle_lib):
    """A survival product equal to the threshold keeps its position (P_j >= tau).
    With h = 0 and b = 0 every s_j is sigmoid(0) = 1/2 exactly, so P_j = 2^-(j+1)
    exactly and tau = 2^-m keeps exactly m positions."""
    kb, H = 6, 16
    h = np.zeros((1, kb, H), dtype=np.uint16)   # bf16 +0
    w = np.full(H, 0x3F80, dtype=np.uint16)     # bf16 1.0 (any w gives w . 0 = 0)
    for m in range(1, kb + 1):
        L, surv, pref = oracle.conf_budget(h, w, 0.0, 2.0 ** -m)
        assert surv.tolist() == [[0.5] * kb]
        assert pref.tolist() == [[2.0 ** -(j + 1) for j in range(kb)]]
        assert L.tolist() == [m]


# ------------------------------------------------------- exact enumeration ----

def _softmax(x, T):
    T = float(np.float32(T))  # temperatures are stored as fp32
    z = x.astype(np.float64) / T
    e = np.exp(z - z.max())
    return e / e.sum()


def _enumerate_paths(p, q, L, V, k):
    """All decision paths of one request with their probabilities.

    p: [k+1, V] target probabilities, q: [k, V] drafter probabilities.  A path
    fixes the drafted tokens it reads and, for every draw it makes, the
    midpoint of the cell of [0, 1) that leads there.  Returns a list of
    (weight, tokens[k], u[k+1, 2], expected n, expected emitted tokens)."""
    paths = []

    def cells(weights):
        total = weights.sum()
        c = np.concatenate([[0.0], np.cumsum(weights)]) / total
        return [(t, weights[t] / total, 0.5 * (c[t] + c[t + 1]))
                for t in range(V) if weights[t] > 0]

    def rec(j, w, toks, u, emitted):
        if j == L:
            for t, prob, mid in cells(p[L]):
                uu = u.copy()
                uu[L, 1] = mid
                paths.append((w * prob, toks.copy(), uu, L, emitted + [t]))
            return
        for x in range(V):
            if q[j, x] == 0:
                continue
            a = min(1.0, p[j, x] / q[j, x])
            t2 = toks.copy()
            t2[j] = x
            if a > 0:
                uu = u.copy()
                uu[j, 0] = 0.5 * a
                rec(j + 1, w * q[j, x] * a, t2, uu, emitted + [x])
            if a < 1:
                resid = np.maximum(0.0, p[j] - q[j])
                for t, prob, mid in cells(resid):
                    uu = u.copy()
                    uu[j, 0] = 0.5 * (1.0 + a)
                    uu[j, 1] = mid
                    paths.append((w * q[j, x] * (1 - a) * prob, t2, uu, j, emitted + [t]))

    rec(0, 1.0, np.zeros(k, dtype=np.int32), np.full((k + 1, 2), 0.5), [])
    return paths


@pytest.mark.parametrize("V,k,L,T,seed", [
    (2, 1, 1, 1.0, 0), (5, 2, 2, 0.7, 1), (8, 3, 3, 1.0, 2), (6, 3, 2, 2.0, 3),
    (4, 3, 0, 1.0, 4), (7, 2, 1, 0.7, 5),
])
def test_exactness_invariant_by_enumeration(oracle_lib, V, k, L, T, seed):
    rng = np.random.default_rng(100 + seed)
    tgt = (rng.standard_normal((k + 1, V)) * 1.5).astype(np.float32)
    drf = (tgt[:k] + rng.standard_normal((k, V)) * 1.0).astype(np.float32)
    p = np.stack([_softmax(tgt[j], T) for j in range(k + 1)])
    q = np.stack([_softmax(drf[j], T) for j in range(k)])
    paths = _enumerate_paths(p, q, L, V, k)
    B = len(paths)
    weights = np.array([pp[0] for pp in paths])
    assert abs(weights.sum() - 1.0) < 1e-12
    res = oracle.verify(
        np.broadcast_to(tgt, (B, k + 1, V)).copy(), np.broadcast_to(drf, (B, k, V)).copy(),
        np.stack([pp[1] for pp in paths]), dtype=F32,
        verify_len=np.full(B, L, dtype=np.int32), temperature=np.full(B, T, dtype=np.float32),
        u_override=np.stack([pp[2] for pp in paths]))
    assert np.all(res["status"] == 0)
    # the oracle's decisions follow the cells the path was built from
    for b, (_, _, _, n, emitted) in enumerate(paths):
        assert res["accepted"][b] == n
        assert list(res["tokens"][b, :n + 1]) == emitted
        assert np.all(res["tokens"][b, n + 1:] == -1)
        for j in range(min(n + 1, L)):
            x = paths[b][1][j]
            assert abs(res["p_x"][b, j] - p[j, x]) <= 1e-14 + 1e-12 * p[j, x]
            assert abs(res["q_x"][b, j] - q[j, x]) <= 1e-14 + 1e-12 * q[j, x]
    # law of the emitted token at each reached position == target row (exactness)
    n_out = res["accepted"]
    alpha = np.minimum(p[:k], q).sum(axis=1)
    for j in range(L + 1):
        reach = n_out >= j
        p_reach = weights[reach].sum()
        assert abs(p_reach - np.prod(alpha[:j])) < 1e-12
        law = np.zeros(V)
        np.add.at(law, res["tokens"][reach, j], weights[reach])
        np.testing.assert_allclose(law / p_reach, p[j], atol=1e-12)


def test_greedy_chain_matches_argmax_rule(oracle_lib):
    rng = np.random.default_rng(9)
    B, k, V = 200, 4, 50
    tgt = _bf16_bits((rng.standard_normal((B, k + 1, V)) * 0.6).astype(np.float32))  # many ties
    vals = _bf16_values(tgt)
    first = np.argmax(vals, axis=-1)
    toks = np.where(rng.random((B, k)) < 0.7, first[:, :k], rng.integers(0, V, (B, k))).astype(np.int32)
    vlen = rng.integers(0, k + 1, B).astype(np.int32)
    res = oracle.verify(tgt, None, toks, dtype=BF16, verify_len=vlen,
                        temperature=np.zeros(B, dtype=np.float32))
    for i in range(B):
        n = 0
        while n < vlen[i] and toks[i, n] == first[i, n]:
            n += 1
        want = list(toks[i, :n]) + [first[i, n]]
        assert res["accepted"][i] == n
        assert list(res["tokens"][i, :n + 1]) == want
        assert np.all(res["p_x"][i] == -1.0)


# ------------------------------------------------------ statistical pins ----

def test_laws_from_philox_driven_runs(oracle_lib):
    from scipy import stats
    rng = np.random.default_rng(21)
    V, k = 6, 2
    tgt = (rng.standard_normal((k + 1, V)) * 1.2).astype(np.float32)
    drf = (0.5 * tgt[:k] + rng.standard_normal((k, V))).astype(np.float32)
    p = np.stack([_softmax(tgt[j], 1.0) for j in range(k + 1)])
    q = np.stack([_softmax(drf[j], 1.0) for j in range(k)])
    alpha = np.minimum(p[:k], q).sum(axis=1)
    n_hist = np.zeros(k + 1)
    tok0 = np.zeros(V)
    tok1 = np.zeros(V)
    total = 0
    for seed in range(5):
        B = 200000
        toks = np.stack([rng.choice(V, size=B, p=q[j]) for j in range(k)], axis=1).astype(np.int32)
        res = oracle.verify(np.broadcast_to(tgt, (B, k + 1, V)).copy(),
                            np.broadcast_to(drf, (B, k, V)).copy(), toks, dtype=F32, seed=seed,
                            threads=4)
        n = res["accepted"]
        n_hist += np.bincount(n, minlength=k + 1)
        tok0 += np.bincount(res["tokens"][:, 0], minlength=V)
        tok1 += np.bincount(res["tokens"][n >= 1, 1], minlength=V)
        total += B
    expect_n = np.array([1 - alpha[0], alpha[0] * (1 - alpha[1]), alpha[0] * alpha[1]])
    assert stats.chisquare(n_hist, expect_n * total).pvalue > 1e-4
    assert stats.chisquare(tok0, p[0] * total).pvalue > 1e-4
    assert stats.chisquare(tok1, p[1] * tok1.sum()).pvalue > 1e-4


def test_mean_accepted_length_closed_form(oracle_lib):
    # E[n] = sum_{j=1..L} prod_{j'<j} alpha_j' per request; over many requests the
    # sample mean lies within 4 standard errors.
    from speculative_decoding_verification_86_b200 import workloads
    w = workloads.stochastic("cpu", seed=1, B=256, k=5, V=16384, fixed_len=5)
    h = workloads.to_numpy_inputs(w)
    res = oracle.verify(h["target"], h["draft"], h["tokens"], dtype=BF16, verify_len=h["verify_len"],
                        seed=h["seed"], threads=8)
    tgt = _bf16_values(h["target"])
    drf = _bf16_values(h["draft"])
    zt = tgt[:, :5] - tgt[:, :5].max(-1, keepdims=True)
    zd = drf - drf.max(-1, keepdims=True)
    p = np.exp(zt) / np.exp(zt).sum(-1, keepdims=True)
    qq = np.exp(zd) / np.exp(zd).sum(-1, keepdims=True)
    alpha = np.minimum(p, qq).sum(-1)                       # [B, 5]
    surv = np.cumprod(alpha, axis=1)                        # P(n >= j+1)
    mean = surv.sum(1)
    second = np.zeros_like(mean)                            # E[n^2] = sum (2j-1) P(n>=j)
    for j in range(5):
        second += (2 * j + 1) * surv[:, j]
    var = (second - mean ** 2).sum()
    n = res["accepted"].astype(np.float64)
    assert abs(n.sum() - mean.sum()) < 4 * math.sqrt(var)


def test_q_equal_p_accepts_every_position(oracle_lib):
    rng = np.random.default_rng(4)
    B, k, V = 64, 5, 300
    tgt = _bf16_bits((rng.standard_normal((B, k + 1, V)) * 3).astype(np.float32))
    toks = rng.integers(0, V, (B, k)).astype(np.int32)
    vlen = rng.integers(0, k + 1, B).astype(np.int32)
    for T in (0.7, 1.0):
        res = oracle.verify(tgt, tgt[:, :k].copy(), toks, dtype=BF16, verify_len=vlen,
                            temperature=np.full(B, T, dtype=np.float32), seed=3)
        assert np.array_equal(res["accepted"], vlen)


# ------------------------------------------------------------ edge cases ----

def test_errors_are_found_lazily_in_chain_order(oracle_lib):
    V, k = 16, 3
    tgt = np.zeros((4, k + 1, V), dtype=np.float32)
    drf = np.zeros((4, k, V), dtype=np.float32)
    tgt[:, :, 3] = 5.0   # p puts most mass on token 3
    drf[:, :, 7] = 5.0   # q puts most mass on token 7 -> x = 7 is rejected at once
    toks = np.full((4, k), 7, dtype=np.int32)
    tgt[0, 0, 1] = np.nan            # request 0: NaN in a row the chain reads
    tgt[1, 2, 1] = np.nan            # request 1: NaN past the first rejection
    toks[2, 0] = V                   # request 2: out-of-range token
    u = np.full((4, k + 1, 2), 0.5)  # u = 0.5 rejects x = 7 at position 0
    res = oracle.verify(tgt, drf, toks, dtype=F32, u_override=u,
                        temperature=np.array([1, 1, 1, -1], dtype=np.float32))
    assert res["status"][0] == oracle.ERR_NONFINITE and res["accepted"][0] == -1
    assert res["status"][1] == 0 and res["accepted"][1] == 0
    assert res["status"][2] == oracle.ERR_BAD_TOKEN and res["accepted"][2] == -1
    assert res["status"][3] == oracle.ERR_BAD_TEMPERATURE
    assert np.all(res["tokens"][[0, 2, 3]] == -1)


def test_greedy_chain_fails_on_a_nonfinite_row(oracle_lib):
    """T = 0 reads target rows only; NaN or +inf in a row it reads fails the
    request, while -inf (a masked token) does not, and a bad value in a row
    past the first disagreement is never read."""
    V, k = 8, 2
    tgt = np.zeros((4, k + 1, V), dtype=np.float32)
    tgt[:, :, 5] = 1.0                   # arg-max 5 everywhere
    toks = np.full((4, k), 5, dtype=np.int32)
    tgt[0, 1, 2] = np.inf                # request 0: +inf in row 1, which the chain reads
    tgt[1, 0, 6] = np.nan                # request 1: NaN in row 0
    tgt[2, 0, 0] = -np.inf               # request 2: a masked token only
    toks[3, 0] = 4                       # request 3: disagrees at position 0 ...
    tgt[3, 1, 0] = np.inf                # ... so row 1's +inf is never read
    with pytest.raises(ValueError):
        oracle.row_argmax(np.array([0.0, np.inf, 1.0], dtype=np.float32), F32)
    res = oracle.verify(tgt, None, toks, dtype=F32, temperature=np.zeros(4, dtype=np.float32))
    assert res["status"].tolist() == [oracle.ERR_NONFINITE, oracle.ERR_NONFINITE, 0, 0]
    assert res["accepted"].tolist() == [-1, -1, 2, 0]
    assert res["tokens"][2].tolist() == [5, 5, 5] and res["tokens"][3].tolist() == [5, -1, -1]


def test_residual_floor_and_inverse_cdf_fallback(oracle_lib):
    # p and q differ by ~1e-14: rejection needs u within 1e-13 of 1 and the
    # residual mass is below the 1e-12 floor, so the token comes from p.
    # u' = 0.2 picks token 0 of p (uniform over 4); token 0 has no residual
    # weight (q_0 > p_0), so sampling the residual instead would give token 1.
    tgt = np.zeros((1, 2, 4), dtype=np.float32)
    drf = np.zeros((1, 1, 4), dtype=np.float32)
    drf[0, 0, 0] = np.float32(1e-13)
    u = np.array([[[1.0 - 2.0 ** -50, 0.2], [0.5, 0.5]]])
    res = oracle.verify(tgt, drf, np.array([[0]], dtype=np.int32), dtype=F32, u_override=u)
    assert res["accepted"][0] == 0 and res["tokens"][0, 0] == 0
    # u = 1 lies past every cell: the largest index with positive weight is taken
    tgt = np.array([[[0.0, 1.0, -np.inf, 2.0, -np.inf]]], dtype=np.float32)
    u = np.array([[[0.5, 1.0]]])
    res = oracle.verify(tgt, np.zeros((1, 0, 5), dtype=np.float32), np.zeros((1, 0), dtype=np.int32),
                        dtype=F32, u_override=u)
    assert res["accepted"][0] == 0 and res["tokens"][0, 0] == 3


def test_verify_len_is_clamped_to_the_block(oracle_lib):
    """L_i = verify_len_i clamped to [0, k] (a negative length verifies
    nothing); with L_i = 0 a request emits one token from target row 0 and
    accepts none."""
    rng = np.random.default_rng(17)
    B, k, V = 6, 3, 16
    target = rng.standard_normal((B, k + 1, V)).astype(np.float32)
    draft = rng.standard_normal((B, k, V)).astype(np.float32)
    tokens = rng.integers(0, V, (B, k)).astype(np.int32)
    vlen = np.array([-5, -1, 0, 2, 3, 9], dtype=np.int32)
    res = oracle.verify(target, draft, tokens, dtype=F32, verify_len=vlen, seed=4)
    assert res["verify_len_used"].tolist() == [0, 0, 0, 2, 3, 3]
    assert np.all(res["accepted"] <= res["verify_len_used"])
    for i in range(3):
        assert res["accepted"][i] == 0
        assert 0 <= res["tokens"][i, 0] < V and np.all(res["tokens"][i, 1:] == -1)


def test_empty_batch(oracle_lib):
    res = oracle.verify(np.zeros((0, 3, 8), dtype=np.float32), np.zeros((0, 2, 8), dtype=np.float32),
                        np.zeros((0, 2), dtype=np.int32), dtype=F32)
    assert res["accepted"].shape == (0,)


# ------------------------------------------------------ hand-worked cases ----

def test_hand_worked_golden_cases(oracle_lib):
    import golden_cases
    cases = golden_cases.load()
    assert len(cases) >= 8
    for c in cases:
        res = oracle.verify(c["target"], c["draft"], c["tokens"], dtype=F32,
                            verify_len=c["verify_len"], temperature=c["temperature"],
                            u_override=c["u"])
        assert res["status"][0] == 0, c["name"]
        assert res["accepted"][0] == c["n"], c["name"]
        assert res["tokens"][0].tolist() == c["out_tokens"].tolist(), c["name"]
