"""Pins of the oracle's temperature > 0 consensus, independent of the oracle.

The rule (the pages name temperature settings but give no sampling rule; the
reading taken): the AR token of row r is the Gumbel-max sample
    t_r = argmax_v logits[r, v] / T - ln(-ln u_{r,v})
with u from Philox4x32-10 at counter (v // 4, r, offset lo, offset hi), key
(seed lo, seed hi), word v % 4, u = (top 24 bits + 1/2) / 2^24; drafts are
accepted left to right iff they equal t (technical summary §2.3 item 3).

Pinned by: the generator's published known-answer vectors; the counter layout
and uniform mapping recomputed here from those words on two-entry rows; the
Gumbel-max theorem (empirical frequencies against softmax(x / T), chi-square);
the T -> 0 limit (greedy argmax) and the T -> infinity limit (uniform); NaN
never sampled; the acceptance rule's special cases.
"""
import math

import numpy as np
import pytest

import oracle


def test_philox_known_answers():
    """Known-answer vectors published with Philox4x32-10 (Random123 test set)."""
    cases = [
        ([0, 0, 0, 0], [0, 0], [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8]),
        ([0xFFFFFFFF] * 4, [0xFFFFFFFF] * 2, [0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD]),
        ([0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344], [0xA4093822, 0x299F31D0],
         [0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1]),
    ]
    for ctr, key, want in cases:
        assert oracle.philox4x32_10(ctr, key).tolist() == want


def _u(r, v, seed, offset):
    """The uniform of (row r, entry v), recomputed from the generator's words."""
    w = oracle.philox4x32_10([v // 4, r, offset & 0xFFFFFFFF, offset >> 32],
                             [seed & 0xFFFFFFFF, seed >> 32])
    return ((int(w[v % 4]) >> 8) + 0.5) / 2 ** 24


def test_counter_layout_on_two_entry_rows():
    """Two equal logits: the sample is the entry with the larger uniform (the
    Gumbel transform is increasing in u), for entries in the same and in
    different Philox words, rows and offsets."""
    seed, offset = 0x1234_5678_9ABC_DEF0, (7 << 32) + 11
    R = 64
    for (v0, v1) in [(0, 1), (2, 3), (3, 4), (5, 9)]:
        V = v1 + 1
        x = np.full((R, V), -np.inf, np.float32)
        x[:, v0] = 0.0
        x[:, v1] = 0.0
        t, _ = oracle.sampled_tokens(x, 1.0, seed, offset)
        for r in range(R):
            want = v0 if _u(r, v0, seed, offset) > _u(r, v1, seed, offset) else v1
            assert t[r] == want, (v0, v1, r)


def _chi2_sf(stat, dof):
    """Upper tail of the chi-square distribution (series for the regularised
    lower incomplete gamma)."""
    a, x = dof / 2.0, stat / 2.0
    term = total = 1.0 / a
    n = 1
    while term > total * 1e-15 and n < 10000:
        term *= x / (a + n)
        total += term
        n += 1
    lower = math.exp(-x + a * math.log(x) - math.lgamma(a)) * total
    return max(0.0, 1.0 - lower)


@pytest.mark.parametrize("T", [0.5, 1.0, 2.5])
def test_gumbel_max_matches_softmax(T):
    """Gumbel-max theorem: over many rows with the same logits the sample
    frequencies follow softmax(x / T)."""
    x0 = np.array([1.5, 0.2, -0.7, 0.9, 0.0, -2.0, 1.1], np.float32)
    R = 60000
    x = np.tile(x0, (R, 1))
    t, _ = oracle.sampled_tokens(x, T, seed=2024, offset=3)
    counts = np.bincount(t, minlength=x0.size).astype(np.float64)
    p = np.exp(x0.astype(np.float64) / T)
    p /= p.sum()
    expect = R * p
    stat = float(((counts - expect) ** 2 / expect).sum())
    assert _chi2_sf(stat, x0.size - 1) > 1e-4, (counts, expect, stat)


def test_low_temperature_is_greedy():
    """T -> 0: the sample is the argmax (rows whose top two logits are close
    are excluded: there the noise / T can still decide)."""
    g = np.random.default_rng(5)
    x = g.standard_normal((300, 512)).astype(np.float32)
    t, _ = oracle.sampled_tokens(x, 1e-4, seed=9, offset=0)
    srt = np.sort(x.astype(np.float64), axis=1)
    clear = (srt[:, -1] - srt[:, -2]) > 1e-2
    assert clear.sum() > 250
    assert np.array_equal(t[clear], np.argmax(x, axis=1)[clear])


def test_high_temperature_is_uniform():
    g = np.random.default_rng(6)
    V, R = 16, 48000
    x = np.tile(g.standard_normal(V).astype(np.float32), (R, 1))
    t, _ = oracle.sampled_tokens(x, 1e7, seed=1, offset=2)
    counts = np.bincount(t, minlength=V).astype(np.float64)
    stat = float(((counts - R / V) ** 2 / (R / V)).sum())
    assert _chi2_sf(stat, V - 1) > 1e-4


def test_nan_and_minus_inf_never_sampled_and_offsets_differ():
    g = np.random.default_rng(7)
    x = g.standard_normal((200, 64)).astype(np.float32)
    x[:, ::3] = np.nan
    x[:, 1::3] = -np.inf
    t, _ = oracle.sampled_tokens(x, 1.3, seed=3, offset=0)
    assert np.all(t % 3 == 2)
    t2, _ = oracle.sampled_tokens(x, 1.3, seed=3, offset=1)
    assert np.mean(t != t2) > 0.5
    t3, _ = oracle.sampled_tokens(x, 1.3, seed=3, offset=0)
    assert np.array_equal(t, t3)


def test_acceptance_on_the_samples():
    """The acceptance rule is the greedy one applied to the sampled tokens:
    all drafts right -> K_b accepted; first wrong -> 1 and the first sample;
    in general the accept rule on the returned samples."""
    g = np.random.default_rng(8)
    K = [5, 1, 7, 3]
    cu = np.concatenate([[0], np.cumsum(K)]).astype(np.int32)
    R = int(cu[-1])
    x = g.standard_normal((R, 300)).astype(np.float32)
    t, _ = oracle.sampled_tokens(x, 0.8, seed=11, offset=4)
    acc, nxt, tt = oracle.consensus_sampled(x, t, cu, 0.8, 11, 4)
    assert np.array_equal(tt, t)
    assert acc.tolist() == K and nxt.tolist() == [int(t[cu[b + 1] - 1]) for b in range(4)]
    wrong = t.copy()
    wrong[cu[:-1]] = (t[cu[:-1]] + 1) % 300
    acc, nxt, _ = oracle.consensus_sampled(x, wrong, cu, 0.8, 11, 4)
    assert acc.tolist() == [1, 1, 1, 1] and nxt.tolist() == t[cu[:-1]].tolist()
    drafts = np.where(g.random(R) < 0.6, t, g.integers(0, 300, R)).astype(np.int32)
    acc, nxt, _ = oracle.consensus_sampled(x, drafts, cu, 0.8, 11, 4)
    a2, n2 = oracle.accept_from_tokens(t, drafts, cu)
    assert np.array_equal(acc, a2) and np.array_equal(nxt, n2)
