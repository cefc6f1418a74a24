"""The sampled-consensus kernel's noise evaluation, emulated in fp32 on the CPU.

The kernel ranks base-2 scores x * log2(e) / T - log2(a) with a = -log2 u and
u = (k + 1/2) / 2^24, k the top 24 bits of a Philox word; this equals the
Gumbel-max score x / T - ln(-ln u) divided by ln 2, less a constant common to
every entry, so the argmax is the same. a comes from the hardware base-2
logarithm for u < 15/16 and from the series (v + v^2/2 + ... + v^7/7) / ln 2
in v = 1 - u for u >= 15/16. These tests restate that evaluation step by step
in numpy float32 (fused multiply-adds rounded once; the hardware logarithm
modelled as exact, its ~2^-22 absolute error being a separate, smaller term)
and bound its error against fp64 over every series k and a sample of the
others: far below the 1e-3 score margin the GPU parity tests allow.
"""
import math

import numpy as np

LN2 = math.log(2.0)
F32 = np.float32
# the kernel's series coefficients 1 / (j ln 2), j = 1..7, as float literals
COEF = [F32(1.442695022e+00), F32(7.213475108e-01), F32(4.808983505e-01), F32(3.606737554e-01),
        F32(2.885390222e-01), F32(2.404491752e-01), F32(2.060992867e-01)]
TWO_M24 = F32(5.9604644775390625e-8)


def _fma(a, b, c):
    """fp32 fused multiply-add: the fp64 product of two fp32 values is exact,
    the sum is rounded to fp32 (double rounding through fp64 is below the
    bounds checked here)."""
    return (np.asarray(a, np.float64) * np.asarray(b, np.float64) + np.asarray(c, np.float64)).astype(F32)


def _noise_log2(k):
    """-log2(a) as the kernel evaluates it, for 24-bit integers k."""
    kf = k.astype(F32)
    v = ((F32(16777216.0) - kf) - F32(0.5)) * TWO_M24
    q = _fma(v, COEF[6], COEF[5])
    for c in (COEF[4], COEF[3], COEF[2], COEF[1], COEF[0]):
        q = _fma(v, q, c)
    a_series = (v * q).astype(F32)
    u = _fma(kf, TWO_M24, F32(2.98023223876953125e-8))
    a_log = (-np.log2(u.astype(np.float64))).astype(F32)
    a = np.where(k >= (15 << 20), a_series, a_log)
    return -np.log2(a.astype(np.float64))


def _exact(k):
    u = (k.astype(np.float64) + 0.5) / 2.0 ** 24
    return -np.log2(-np.log(u) / LN2)


def test_coefficients_are_one_over_j_ln2():
    for j, c in enumerate(COEF, 1):
        assert abs(float(c) - 1.0 / (j * LN2)) <= 2 ** -24 * float(c)


def test_v_and_u_are_exact_where_used():
    k = np.arange(15 << 20, 1 << 24, 4099, dtype=np.int64)
    v = ((F32(16777216.0) - k.astype(F32)) - F32(0.5)) * TWO_M24
    assert np.array_equal(v.astype(np.float64), (2.0 ** 24 - k - 0.5) / 2.0 ** 24)
    k2 = np.arange(0, 1 << 23, 997, dtype=np.int64)  # below 2^23, k + 1/2 fits in fp32
    u = _fma(k2.astype(F32), TWO_M24, F32(2.98023223876953125e-8))
    assert np.array_equal(u.astype(np.float64), (k2 + 0.5) / 2.0 ** 24)


def test_series_branch_every_k():
    k = np.arange(15 << 20, 1 << 24, dtype=np.int64)
    err = np.abs(_noise_log2(k) - _exact(k))
    assert err.max() < 5e-7, err.max()


def test_log_branch_sampled_k():
    rng = np.random.default_rng(0)
    k = np.concatenate([rng.integers(0, 15 << 20, 1_000_000), np.arange(0, 4096),
                        np.arange((15 << 20) - 4096, 15 << 20)]).astype(np.int64)
    err = np.abs(_noise_log2(k) - _exact(k))
    assert err.max() < 2e-6, err.max()
    # the hardware logarithm's ~2^-22 absolute error becomes a relative error
    # of a of at most 2^-22 / log2(16/15) at the branch point
    assert 2 ** -22 / math.log2(16 / 15) < 3e-6


def test_base2_scores_rank_like_the_gumbel_scores():
    """Dividing x / T - ln(-ln u) by ln 2 and dropping log2(ln 2) gives the
    kernel's x log2(e) / T - log2(-log2 u): same ordering on random rows."""
    rng = np.random.default_rng(1)
    for T in (0.3, 1.0, 2.5):
        x = rng.standard_normal((200, 64))
        k = rng.integers(0, 1 << 24, (200, 64))
        u = (k + 0.5) / 2.0 ** 24
        s = x / T - np.log(-np.log(u))
        r = x * (1.0 / (T * LN2)) - np.log2(-np.log2(u))
        assert np.allclose(r, s / LN2 + math.log2(LN2), atol=1e-12)
        assert np.array_equal(np.argmax(r, axis=1), np.argmax(s, axis=1))


def test_kernel_source_uses_these_constants():
    """The coefficients and scale factors above are the ones in the kernel's
    noise_log2 (read from the CUDA source, so the two cannot drift apart)."""
    import os
    import re
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = open(os.path.join(root, "diffusion_draft_ar_b200", "csrc", "consensus.cuh")).read()
    body = src[src.index("float noise_log2(uint32_t word)"):]
    body = body[:body.index("\n}\n")]
    lits = {F32(float(m.rstrip("f"))) for m in re.findall(r"\d+\.\d*(?:e[+-]?\d+)?f", body)}
    for c in COEF + [TWO_M24, F32(2.98023223876953125e-8), F32(16777216.0), F32(0.5)]:
        assert c in lits, c
    assert "15u << 20" in body
