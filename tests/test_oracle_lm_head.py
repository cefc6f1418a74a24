"""Pins of the oracle's LM-head scores, greedy tokens and accept rule, each
checked against something other than the oracle itself.

The AR view's greedy token per block row (technical summary §2.3 items 2-3)
is the first index of the largest score of its output projection: logits[r, v]
= <hidden[r], w_head[v]>. Pins:
  - a pure-Python loop on tiny inputs whose values are small dyadic numbers
    (every product and sum exact), with its own first-maximum scan;
  - one-hot hidden rows: the scores are one column of w_head, exactly;
  - numpy's fp64 matmul (a library routine, not the oracle's loop) and the
    sums of absolute products;
  - exact linearity under a power-of-two scale;
  - ties resolved to the lowest index, NaN never chosen;
  - the accept rule on given tokens equals the pinned consensus oracle on
    logits whose argmax are those tokens, plus the rule's special cases.
"""
import math
import random

import numpy as np
import pytest

import oracle


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bits by truncation; the tests only feed exactly representable values
    or do not care which nearby bf16 value is used."""
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_pure_python_loop_on_dyadic_inputs():
    rng = random.Random(7)
    vals = [-2.0, -1.0, -0.5, 0.0, 0.5, 1.0, 2.0, 1.5]
    for trial in range(20):
        R, d, V = rng.randint(1, 3), rng.randint(1, 6), rng.randint(1, 9)
        h = [[rng.choice(vals) for _ in range(d)] for _ in range(R)]
        w = [[rng.choice(vals) for _ in range(d)] for _ in range(V)]
        got = oracle.lm_head_logits(to_bf16_bits(np.array(h)), to_bf16_bits(np.array(w)))
        for r in range(R):
            row = []
            for v in range(V):
                s = 0.0
                for k in reversed(range(d)):  # another order: exact anyway
                    s += h[r][k] * w[v][k]
                row.append(s)
                assert got[r, v] == s
            best, idx = -math.inf, 0
            for v, x in enumerate(row):
                if x > best:
                    best, idx = x, v
            assert oracle.greedy_tokens(got[r:r + 1])[0] == idx


def test_one_hot_hidden_reads_one_column():
    rng = np.random.default_rng(1)
    d, V = 48, 700
    w = to_bf16_bits(rng.standard_normal((V, d)))
    for k in (0, 17, d - 1):
        h = np.zeros((1, d), np.float32)
        h[0, k] = 1.0
        got = oracle.lm_head_logits(to_bf16_bits(h), w)
        np.testing.assert_array_equal(got[0], bits_to_f64(w[:, k]))
        assert oracle.greedy_tokens(got)[0] == int(np.argmax(bits_to_f64(w[:, k])))


def test_matches_numpy_fp64_matmul_and_abs_sums():
    rng = np.random.default_rng(2)
    R, d, V = 5, 256, 3001
    h = to_bf16_bits(rng.standard_normal((R, d)))
    w = to_bf16_bits(rng.standard_normal((V, d)) / 16)
    rows = np.array([4, 0, 2], np.int64)
    got, ab = oracle.lm_head_logits(h, w, rows=rows, with_absdot=True)
    H, W = bits_to_f64(h)[rows], bits_to_f64(w)
    ref = H @ W.T
    ref_ab = np.abs(H) @ np.abs(W).T
    assert np.all(np.abs(got - ref) <= 1e-12 * ref_ab)
    np.testing.assert_allclose(ab, ref_ab, rtol=1e-12)
    np.testing.assert_array_equal(oracle.greedy_tokens(got), np.argmax(ref, axis=1))


def test_power_of_two_scale_is_exact():
    rng = np.random.default_rng(3)
    h = rng.standard_normal((2, 64)).astype(np.float32)
    w = to_bf16_bits(rng.standard_normal((50, 64)))
    hb = to_bf16_bits(h)
    a = oracle.lm_head_logits(hb, w)
    b = oracle.lm_head_logits(to_bf16_bits(bits_to_f64(hb) * 4.0), w)
    np.testing.assert_array_equal(b, 4.0 * a)


def test_ties_take_the_lowest_index_and_nan_never_wins():
    d, V = 8, 12
    w = np.zeros((V, d), np.float32)
    w[:, 0] = np.linspace(-1, 0.5, V)
    w[9, 0] = 3.0
    w[2, 0] = 3.0  # the same maximum at a lower index
    h = np.zeros((1, d), np.float32)
    h[0, 0] = 1.0
    got = oracle.lm_head_logits(to_bf16_bits(h), to_bf16_bits(w))
    assert oracle.greedy_tokens(got)[0] == 2
    x = np.array([[np.nan, -0.0, 0.0, -1.0]])
    assert oracle.greedy_tokens(x)[0] == 1  # -0 == +0: the first of them
    assert oracle.greedy_tokens(np.full((1, 3), np.nan))[0] == 0


def test_accept_from_tokens_agrees_with_consensus():
    rng = np.random.default_rng(4)
    cu = np.array([0, 5, 5, 13, 16], np.int32)
    R, V = int(cu[-1]), 97
    for trial in range(30):
        logits = rng.standard_normal((R, V)).astype(np.float32)
        t = np.argmax(logits, axis=1).astype(np.int32)
        draft = np.where(rng.random(R) < 0.7, t, rng.integers(0, V, R)).astype(np.int32)
        acc, nxt, am = oracle.consensus(logits, draft, cu)
        np.testing.assert_array_equal(am, t)
        acc2, nxt2 = oracle.accept_from_tokens(t, draft, cu)
        np.testing.assert_array_equal(acc2, acc)
        np.testing.assert_array_equal(nxt2, nxt)


def test_accept_rule_special_cases():
    cu = np.array([0, 4, 8, 12, 12], np.int32)
    t = np.array([5, 6, 7, 8, 1, 2, 3, 4, 9, 9, 9, 9], np.int32)
    draft = t.copy()
    draft[4] = 0        # sequence 1: first draft wrong -> only the correction
    draft[10] = 0       # sequence 2: mismatch at j = 2 -> j + 1 rows
    acc, nxt = oracle.accept_from_tokens(t, draft, cu)
    np.testing.assert_array_equal(acc, [4, 1, 3, 0])   # all match -> K; K_b = 0 -> 0
    np.testing.assert_array_equal(nxt, [8, 1, 9, -1])


@pytest.mark.parametrize("bad", ["rows"])
def test_rejects_out_of_range_rows(bad):
    h = np.zeros((2, 4), np.uint16)
    w = np.zeros((3, 4), np.uint16)
    with pytest.raises(ValueError):
        oracle.lm_head_logits(h, w, rows=np.array([2]))
