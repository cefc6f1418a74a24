"""Pins for the oracle's greedy consensus (Orthrus technical summary §2.3 item 3:
a drafted token is accepted iff it equals the frozen AR view's greedy token,
checked left to right; at the first divergence j the prefix up to j-1 is
committed together with the AR correction token)."""
import itertools
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "consensus_rule.txt")


def _greedy_first_max(row):
    """Greedy token as Python sees it: the first position of the maximum."""
    row = list(row)
    return row.index(max(row))


def _simulate_sequential(logit_rows, drafts):
    """Sequential greedy decoding fed with the block's rows one step at a time.

    Step i emits the AR view's greedy token t_i. Row i+1's logits were computed
    with draft d_i in the slot after row i, so they are only usable if d_i was
    the token the AR view actually emitted; otherwise decoding stops after t_i
    (the correction). Returns the emitted tokens."""
    emitted = []
    for i, row in enumerate(logit_rows):
        t = _greedy_first_max(row)
        emitted.append(t)
        if drafts[i] != t:
            break
    return emitted


def _pack(seqs):
    """seqs: list of (logit_rows, drafts) -> oracle arrays."""
    rows, drafts, cu = [], [], [0]
    for lr, dr in seqs:
        rows.extend(lr)
        drafts.extend(dr)
        cu.append(cu[-1] + len(lr))
    V = len(rows[0]) if rows else 1
    return (np.array(rows, np.float32).reshape(-1, V), np.array(drafts, np.int32),
            np.array(cu, np.int32))


def test_special_cases():
    rng = np.random.default_rng(0)
    K, V = 6, 10
    x = rng.standard_normal((K, V)).astype(np.float32)
    t = x.argmax(1).astype(np.int32)
    cu = np.array([0, K], np.int32)
    # every draft matches -> K accepted, next = t_{K-1}
    acc, nxt, am = oracle.consensus(x, t, cu)
    assert acc[0] == K and nxt[0] == t[K - 1]
    np.testing.assert_array_equal(am, t)
    # first draft mismatches -> only the correction, next = t_0
    d = t.copy()
    d[0] = (t[0] + 1) % V
    acc, nxt, _ = oracle.consensus(x, d, cu)
    assert acc[0] == 1 and nxt[0] == t[0]
    # mismatch at j -> j+1 committed, next = t_j
    for j in range(K):
        d = t.copy()
        d[j] = (t[j] + 1) % V
        acc, nxt, _ = oracle.consensus(x, d, cu)
        assert acc[0] == min(j + 1, K) and nxt[0] == t[j]
    # only the last draft mismatches -> all K rows committed
    d = t.copy()
    d[K - 1] = (t[K - 1] + 1) % V
    acc, _, _ = oracle.consensus(x, d, cu)
    assert acc[0] == K


def test_brute_force_v3_k3_against_sequential_greedy():
    """Every K=3 block over V=3 with integer logits in {0,1,2} (ties included) and
    every draft vector, as one batched oracle call, against step-by-step greedy."""
    row_choices = list(itertools.product((0.0, 1.0, 2.0), repeat=3))
    seqs = []
    for rows in itertools.product(row_choices, repeat=3):
        for drafts in itertools.product(range(3), repeat=3):
            seqs.append((list(rows), list(drafts)))
    x, d, cu = _pack(seqs)
    acc, nxt, am = oracle.consensus(x, d, cu)
    for b, (rows, drafts) in enumerate(seqs):
        em = _simulate_sequential(rows, drafts)
        assert acc[b] == len(em), (rows, drafts)
        assert nxt[b] == em[-1], (rows, drafts)
        for i in range(3):
            assert am[3 * b + i] == _greedy_first_max(rows[i])


def test_argmax_matches_numpy_first_occurrence():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((64, 2000)).astype(np.float32)
    # plant exact ties of the row maximum at a lower and a higher index
    for r in range(0, 64, 4):
        j = int(x[r].argmax())
        x[r, (j + 7) % 2000] = x[r, j]
        x[r + 1, max(0, j - 5)] = x[r + 1].max()
    cu = np.array([0, 64], np.int32)
    _, _, am = oracle.consensus(x, np.zeros(64, np.int32), cu)
    np.testing.assert_array_equal(am, np.argmax(x, axis=1))


def test_nan_signed_zero_and_infinities():
    nan, inf = np.float32("nan"), np.float32("inf")
    rows = np.array([
        [-0.0, 0.0, -1.0, -2.0],     # -0 == +0: first index wins
        [0.0, -0.0, -1.0, -2.0],
        [nan, 1.0, 1.0, 0.0],        # NaN ignored (treated as -inf)
        [nan, nan, nan, nan],        # all NaN -> index 0
        [-inf, -inf, -inf, -inf],    # all -inf -> index 0
        [1.0, inf, nan, inf],        # +inf wins, first occurrence
    ], np.float32)
    cu = np.array([0, 6], np.int32)
    _, _, am = oracle.consensus(rows, np.zeros(6, np.int32), cu)
    np.testing.assert_array_equal(am, [0, 0, 1, 0, 0, 1])


def test_ragged_and_empty_blocks():
    rng = np.random.default_rng(2)
    sizes = [3, 0, 1, 5, 0, 2]
    cu = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    R = int(cu[-1])
    x = rng.standard_normal((R, 50)).astype(np.float32)
    t = x.argmax(1)
    d = np.where(rng.random(R) < 0.6, t, (t + 1) % 50).astype(np.int32)
    acc, nxt, _ = oracle.consensus(x, d, cu)
    for b, k in enumerate(sizes):
        if k == 0:
            assert acc[b] == 0 and nxt[b] == -1
            continue
        r0 = cu[b]
        em = _simulate_sequential([list(x[r0 + i]) for i in range(k)], list(d[r0:r0 + k]))
        assert acc[b] == len(em) and nxt[b] == em[-1]


def _read_golden(path):
    cases, cur = [], None
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, _, val = line.partition(":")
            key, val = key.strip(), val.strip()
            if key == "case":
                cur = {"name": val, "rows": []}
                cases.append(cur)
            elif key == "row":
                cur["rows"].append([float(v) for v in val.split()])
            elif key in ("draft", "expect_argmax"):
                cur[key] = [int(v) for v in val.split()]
            elif key in ("expect_accept", "expect_next"):
                cur[key] = int(val)
    return cases


def test_golden_hand_worked_rule():
    cases = _read_golden(GOLDEN)
    assert len(cases) >= 4
    for c in cases:
        x = np.array(c["rows"], np.float32)
        cu = np.array([0, x.shape[0]], np.int32)
        acc, nxt, am = oracle.consensus(x, np.array(c["draft"], np.int32), cu)
        assert list(am) == c["expect_argmax"], c["name"]
        assert acc[0] == c["expect_accept"], c["name"]
        assert nxt[0] == c["expect_next"], c["name"]
