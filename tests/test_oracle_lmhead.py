"""Pins of the oracle's shared-head logits (l = h W^T from bf16 inputs)
against what fixes them independently: exact widening of known bf16 bit
patterns, a brute-force correctly rounded sum per logit, one-hot rows that
select a column of W, and integer grids whose product is an exact integer
matmul."""
import math

import numpy as np

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
