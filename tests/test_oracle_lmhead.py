"""Pins of the oracle's shared-head logits (l = h W^T from bf16 inputs)
against what fixes them independently: exact widening of known bf16 bit
patterns, a brute-force correctly rounded sum per logit, one-hot rows that
select a column of W, and integer grids whose product is an exact integer
matmul.  The last test plants mistakes in the oracle's shared-head functions
(in this process, by monkeypatch) and checks that a pin fails on each."""
import math

import numpy as np
import pytest

import oracle


def _bits(x):
    """bf16 bits of float32 values that are exactly representable in bf16."""
    a = np.asarray(x, dtype=np.float32)
    u = a.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0)
    return (u >> 16).astype(np.uint16)


def test_bf16_widening_known_patterns():
    bits = np.array([0x3F80, 0xC000, 0x3E80, 0x0001, 0x7F80, 0x4049], dtype=np.uint16)
    got = oracle.bf16_to_f64(bits)
    want = [1.0, -2.0, 0.25, 2.0 ** -133, math.inf, 3.140625]
    assert got.tolist() == want


def test_logits_brute_force():
    rng = np.random.default_rng(0)
    rows, H, V = 3, 7, 5  # non-square: a transposed operand cannot pass
    def trunc(a):  # float32 values cut to bf16 precision
        return (a.astype(np.float32).view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)

    h = _bits(trunc(rng.standard_normal((rows, H))))
    w = _bits(trunc(rng.standard_normal((V, H))))
    got = oracle.lmhead_logits(h, w)
    hf, wf = oracle.bf16_to_f64(h), oracle.bf16_to_f64(w)
    assert got.shape == (rows, V)
    for r in range(rows):
        for v in range(V):
            terms = [hf[r, c] * wf[v, c] for c in range(H)]
            want = math.fsum(terms)
            assert abs(got[r, v] - want) <= 1e-15 * sum(abs(t) for t in terms)


def test_one_hot_rows_select_a_column():
    rng = np.random.default_rng(1)
    H, V = 16, 40
    w = _bits((rng.integers(-100, 100, (V, H)) / 16.0).astype(np.float32))
    h = np.zeros((H, H), dtype=np.float32)
    np.fill_diagonal(h, 1.0)
    got = oracle.lmhead_logits(_bits(h), w)
    np.testing.assert_array_equal(got, oracle.bf16_to_f64(w).T)


def test_integer_grid_is_exact():
    rng = np.random.default_rng(2)
    rows, H, V = 9, 2560, 300
    hi = rng.integers(-3, 4, (rows, H))
    wi = rng.integers(-1, 2, (V, H))
    got = oracle.lmhead_logits(_bits((hi / 4.0).astype(np.float32)), _bits((wi / 8.0).astype(np.float32)))
    exact = (hi.astype(np.int64) @ wi.T.astype(np.int64)).astype(np.float64) / 32.0
    np.testing.assert_array_equal(got, exact)
    # the fp32 rounding the verification applies is exact on this grid
    np.testing.assert_array_equal(got.astype(np.float32).astype(np.float64), got)


def _grid_case(seed, B, k, H, V):
    rng = np.random.default_rng(seed)
    ht = rng.integers(-3, 4, (B, k + 1, H))
    hd = rng.integers(-3, 4, (B, k, H))
    w = rng.integers(-2, 3, (V, H))
    tokens = rng.integers(0, V, (B, k)).astype(np.int32)
    # exact logits by integer arithmetic: (h/4)(w/8)^T = (h w^T)/32
    lt = (np.einsum("bjh,vh->bjv", ht, w) / 32.0).astype(np.float32)
    ld = (np.einsum("bjh,vh->bjv", hd, w) / 32.0).astype(np.float32)
    to_bits = lambda a, s: _bits((a / s).astype(np.float32))
    return to_bits(ht, 4.0), to_bits(hd, 4.0), to_bits(w, 8.0), tokens, lt, ld


def test_verify_lmhead_is_verify_on_the_heads_logits():
    """The target rows come from hidden_target, the drafter rows from
    hidden_draft, and position j of request i from row (i, j): swapping the two
    models, transposing the head or misaligning a position changes the result."""
    ht, hd, w, tokens, lt, ld = _grid_case(3, B=6, k=3, H=24, V=50)
    temps = np.array([1.0, 0.0, 0.7, 1.0, 1.3, 0.0], dtype=np.float32)
    vlen = np.array([3, 2, 3, 0, 1, 3], dtype=np.int32)
    got = oracle.verify_lmhead(ht, hd, w, tokens, temperature=temps, verify_len=vlen, seed=11)
    want = oracle.verify(lt, ld, tokens, dtype=oracle.DTYPE_F32, temperature=temps,
                         verify_len=vlen, seed=11)
    for key in ("accepted", "tokens"):
        np.testing.assert_array_equal(got[key], want[key])
    np.testing.assert_array_equal(got["p_x"], want["p_x"])
    np.testing.assert_array_equal(got["q_x"], want["q_x"])
    # the pin is sensitive: drafter rows taken from the target's hidden states differ
    wrong = oracle.verify(lt, lt[:, :3].copy(), tokens, dtype=oracle.DTYPE_F32,
                          temperature=temps, verify_len=vlen, seed=11)
    assert not np.array_equal(wrong["q_x"], want["q_x"])
    zeros = np.zeros(6, dtype=np.float32)
    want_greedy = oracle.verify(lt, None, tokens, dtype=oracle.DTYPE_F32, temperature=zeros)
    greedy = oracle.verify_lmhead(ht, None, w, tokens, temperature=zeros)
    np.testing.assert_array_equal(greedy["tokens"], want_greedy["tokens"])
    np.testing.assert_array_equal(greedy["accepted"], want_greedy["accepted"])


# ------------------------------------------ the pins catch planted mistakes --

def _bf16_round(a):
    """float64 -> nearest bf16 value (round to nearest even), as float64."""
    u = np.asarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


_PINS = [test_bf16_widening_known_patterns, test_logits_brute_force, test_one_hot_rows_select_a_column,
         test_integer_grid_is_exact, test_verify_lmhead_is_verify_on_the_heads_logits]


def _mutants():
    good_widen, good_logits, good_verify = oracle.bf16_to_f64, oracle.lmhead_logits, oracle.verify
    return {
        "bf16 widened from the wrong half": ("bf16_to_f64", lambda b: (
            (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(15))
            .view(np.float32).astype(np.float64))),
        "logits accumulated in fp32": ("lmhead_logits", lambda h, w: (
            good_widen(h).astype(np.float32) @ good_widen(w).astype(np.float32).T).astype(np.float64)),
        "head not transposed": ("lmhead_logits", lambda h, w: good_widen(h) @ good_widen(w)),
        "logits rounded to bf16": ("lmhead_logits", lambda h, w: _bf16_round(good_logits(h, w))),
        "drafter rows from the target's hidden states": ("verify_lmhead", lambda ht, hd, w, tok, **kw: (
            good_verify(good_logits(ht, w).astype(np.float32),
                        None if hd is None else good_logits(ht[..., :hd.shape[1], :], w).astype(np.float32),
                        tok, dtype=oracle.DTYPE_F32, **kw))),
    }


@pytest.mark.parametrize("name", list(_mutants()))
def test_planted_mistakes_fail_a_pin(monkeypatch, name):
    attr, fn = _mutants()[name]
    monkeypatch.setattr(oracle, attr, fn)
    caught = 0
    for pin in _PINS:
        try:
            with np.errstate(all="ignore"):  # a mutant may overflow
                pin()
        except (AssertionError, ValueError):
            caught += 1
    assert caught > 0, name
