"""Fused LM head + greedy consensus (``orthrus_lm_head_consensus``) against the
oracle's fp64 scores.

What is unique and what is not: the GPU sums bf16 products in fp32 on the
tensor cores in an order of its own, so its greedy token is one of the indices
whose exact score is within the fp32 accumulation bound of the maximum. For
every checked row the oracle gives the exact scores s_v and the sums of
absolute products a_v; with gamma = d*u/(1 - d*u), u = 2^-23 (no assumption on
the accumulator's rounding mode), the GPU's token j must satisfy
s_j >= s_max - gamma * (a_max + a_j). Where that set holds one index (nearly
always), the token must be exactly the oracle's. Accept lengths and next
tokens then follow from the tokens by the exact rule (oracle.accept_from_tokens).

With small-integer inputs every partial sum is exact in fp32, so the GPU must
reproduce the oracle bit for bit, including the many exact ties (lowest index).
"""
import numpy as np
import pytest
import torch

import oracle
from tests._gpu import gpu, lib, needs_cuda

pytestmark = [gpu, needs_cuda]

U_ACC = 2.0 ** -23


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def make_case(R, d, V, seed, cu=None, integer=False, p_match=0.8):
    g = torch.Generator(device="cpu").manual_seed(seed)
    if integer:
        hidden = torch.randint(-1, 2, (R, d), generator=g).to(torch.bfloat16)
        w = torch.randint(-2, 3, (V, d), generator=g).to(torch.bfloat16)
    else:
        hidden = torch.randn((R, d), generator=g).to(torch.bfloat16)
        w = (torch.randn((V, d), generator=g) / d ** 0.5).to(torch.bfloat16)
    if cu is None:
        cu = torch.arange(0, R + 1, 32 if R % 32 == 0 else R, dtype=torch.int32)
        if cu[-1] != R:
            cu = torch.tensor([0, R], dtype=torch.int32)
    cu = torch.as_tensor(cu, dtype=torch.int32)
    # drafts: a seeded stand-in for the diffusion view's proposals, built from
    # torch's own fp32 scores (input plumbing, not the kernel under test)
    ref = (hidden.float() @ w.float().T).argmax(dim=1).to(torch.int32)
    coins = torch.rand((R,), generator=g)
    alt = torch.randint(0, V, (R,), generator=g, dtype=torch.int32)
    drafts = torch.where(coins < p_match, ref, alt).to(torch.int32)
    return hidden, w, cu, drafts


def run_gpu(hidden, w, cu, drafts, max_block, prefix_lens=None):
    O = lib()
    B = cu.numel() - 1
    R = hidden.shape[0]
    dev = "cuda"
    h, wd, cud, dr = hidden.to(dev), w.to(dev), cu.to(dev), drafts.to(dev)
    acc = torch.full((B,), -7, dtype=torch.int32, device=dev)
    nxt = torch.full((B,), -7, dtype=torch.int32, device=dev)
    am = torch.full((R,), -7, dtype=torch.int32, device=dev)
    ws = torch.empty(O.lm_head_workspace_size(R), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    lens = None if prefix_lens is None else prefix_lens.to(dev)
    O.lm_head_consensus(h, wd, dr, cud, B, max_block, acc, nxt, ws, row_argmax=am,
                        prefix_lens=lens, error_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    out = dict(acc=acc.cpu().numpy(), nxt=nxt.cpu().numpy(), am=am.cpu().numpy())
    if lens is not None:
        out["lens"] = lens.cpu().numpy()
    return out


def resolve_tokens(hidden, w, rows, gpu_t):
    """Oracle tokens for `rows`; where the fp32 bound admits several indices the
    GPU's choice is checked to be one of them and taken. Returns (tokens, ambiguous)."""
    d = hidden.shape[1]
    gamma = d * U_ACC / (1 - d * U_ACC)
    s, a = oracle.lm_head_logits(bits(hidden), bits(w), rows=rows, with_absdot=True)
    t0 = oracle.greedy_tokens(s)
    out = t0.copy()
    ambiguous = 0
    for i in range(len(rows)):
        j = int(gpu_t[i])
        assert 0 <= j < w.shape[0], (rows[i], j)
        m = t0[i]
        valid = s[i] >= s[i, m] - gamma * (a[i, m] + a[i])
        if valid.sum() > 1:
            ambiguous += 1
            assert valid[j], (rows[i], j, s[i, j], s[i, m])
            out[i] = j
        else:
            assert j == m, (rows[i], j, m, s[i, j], s[i, m])
    return out, ambiguous


CASES = [
    # (R, d, V, cu, max_block)
    (8, 64, 512, [0, 8], 8),                                  # tiny: one 128-row block
    (80, 128, 1000, [0, 8, 24, 56, 64, 80], 32),              # ragged blocks, V tail
    (300, 256, 3001, [0, 32, 64, 96, 128, 160, 192, 224, 256, 288, 300], 32),  # two blocks/tile
    (32, 2048, 151936, [0, 32], 32),                          # Qwen3-1.7B verify rows
]


@pytest.mark.parametrize("R,d,V,cu,K", CASES, ids=[f"R{c[0]}-d{c[1]}-V{c[2]}" for c in CASES])
def test_lm_head_consensus_all_rows(R, d, V, cu, K):
    hidden, w, cu_t, drafts = make_case(R, d, V, seed=R + V, cu=cu)
    got = run_gpu(hidden, w, cu_t, drafts, K)
    t, amb = resolve_tokens(hidden, w, np.arange(R, dtype=np.int64), got["am"])
    # the bound admits a second index when the top two scores lie within it
    # (about 7% of rows at V = 151936, d = 2048); those rows are checked valid
    assert amb <= R // 4 + 2
    np.testing.assert_array_equal(got["am"], t)
    acc, nxt = oracle.accept_from_tokens(t, drafts.numpy(), cu_t.numpy())
    np.testing.assert_array_equal(got["acc"], acc)
    np.testing.assert_array_equal(got["nxt"], nxt)


@pytest.mark.parametrize("R,d,V", [(8, 64, 512), (300, 256, 3001), (512, 512, 20000)])
def test_integer_inputs_bit_exact_with_ties(R, d, V):
    """Small-integer hidden states and weights: every score is an exact
    integer in fp32, many rows hold tied maxima, and the GPU's tokens must be the
    oracle's first maxima exactly."""
    hidden, w, cu_t, drafts = make_case(R, d, V, seed=3, integer=True)
    got = run_gpu(hidden, w, cu_t, drafts, int((cu_t[1:] - cu_t[:-1]).max()))
    s = oracle.lm_head_logits(bits(hidden), bits(w))
    t = oracle.greedy_tokens(s)
    ties = int(sum((s[i] == s[i, t[i]]).sum() > 1 for i in range(R)))
    assert ties > 0
    np.testing.assert_array_equal(got["am"], t)
    acc, nxt = oracle.accept_from_tokens(t, drafts.numpy(), cu_t.numpy())
    np.testing.assert_array_equal(got["acc"], acc)
    np.testing.assert_array_equal(got["nxt"], nxt)


def test_degenerate_zero_scores_and_single_entry_vocab():
    # all scores 0: every row's token is 0
    hidden = torch.zeros((40, 64), dtype=torch.bfloat16)
    w = torch.randn((777, 64)).to(torch.bfloat16)
    cu = torch.tensor([0, 8, 40], dtype=torch.int32)
    drafts = torch.zeros(40, dtype=torch.int32)
    drafts[20] = 5
    got = run_gpu(hidden, w, cu, drafts, 32)
    assert (got["am"] == 0).all()
    np.testing.assert_array_equal(got["acc"], [8, 13])
    np.testing.assert_array_equal(got["nxt"], [0, 0])
    # V = 1
    got = run_gpu(torch.randn((16, 128)).to(torch.bfloat16), torch.randn((1, 128)).to(torch.bfloat16),
                  torch.tensor([0, 16], dtype=torch.int32), torch.zeros(16, dtype=torch.int32), 16)
    assert (got["am"] == 0).all() and got["acc"][0] == 16


def test_nan_weight_row_never_wins():
    hidden, w, cu, drafts = make_case(64, 128, 5000, seed=11)
    w[1234] = float("nan")
    got = run_gpu(hidden, w, cu, drafts, 32)
    assert (got["am"] != 1234).all()
    t, _ = resolve_tokens(hidden, w, np.arange(64, dtype=np.int64), got["am"])
    np.testing.assert_array_equal(got["am"], t)


def test_commit_advances_prefix_lens():
    hidden, w, cu, drafts = make_case(96, 256, 4096, seed=5, cu=[0, 32, 64, 96])
    lens = torch.tensor([100, 4096, 7], dtype=torch.int32)
    got = run_gpu(hidden, w, cu, drafts, 32, prefix_lens=lens)
    np.testing.assert_array_equal(got["lens"], lens.numpy() + got["acc"])
    t, _ = resolve_tokens(hidden, w, np.arange(96, dtype=np.int64), got["am"])
    acc, _ = oracle.accept_from_tokens(t, drafts.numpy(), cu.numpy())
    np.testing.assert_array_equal(got["acc"], acc)


def test_qwen3_8b_verify_rows_sampled():
    """The Qwen3-8B verify step: 16 sequences x 32 rows, d_model 4096, V 151936.
    Two whole sequences (rows 0-31 and 480-511, the first and last row tiles)
    plus rows around the 128/256-row block edges are checked against fp64;
    accept lengths and next tokens of the two whole sequences exactly."""
    R, d, V = 512, 4096, 151936
    cu = torch.arange(0, R + 1, 32, dtype=torch.int32)
    hidden, w, cu, drafts = make_case(R, d, V, seed=8, cu=cu)
    got = run_gpu(hidden, w, cu, drafts, 32)
    rows = np.array(list(range(0, 32)) + [127, 128, 255, 256, 383, 384] + list(range(480, 512)),
                    dtype=np.int64)
    t, amb = resolve_tokens(hidden, w, rows, got["am"][rows])
    assert amb <= len(rows) // 4 + 2
    for b, sl in ((0, slice(0, 32)), (15, slice(38, 70))):
        tb = t[sl]
        acc, nxt = oracle.accept_from_tokens(tb, drafts.numpy()[32 * b:32 * b + 32],
                                             np.array([0, 32], np.int32))
        assert got["acc"][b] == acc[0] and got["nxt"][b] == nxt[0]


@pytest.mark.parametrize("R,d,V", [(1, 64, 257), (7, 192, 17), (129, 64, 1000), (255, 128, 513),
                                   (257, 64, 300), (130, 192, 4097)])
def test_edge_tilings_integer_exact(R, d, V):
    """Ragged tilings on exact (integer) scores: one row; a second 128-row block
    holding a single row (R = 129); row and vocabulary tails of one element
    (R = 257, V = 257, 4097); d_model of three K steps. Every token, accept
    length and next token must equal the oracle's."""
    hidden, w, _, drafts = make_case(R, d, V, seed=R * 7 + V, integer=True)
    cuts = sorted({0, R, *[min(R, x) for x in (1, R // 3, R // 2)]})
    cu = torch.tensor(cuts, dtype=torch.int32)
    K = int((cu[1:] - cu[:-1]).max())
    got = run_gpu(hidden, w, cu, drafts, K)
    t = oracle.greedy_tokens(oracle.lm_head_logits(bits(hidden), bits(w)))
    np.testing.assert_array_equal(got["am"], t)
    acc, nxt = oracle.accept_from_tokens(t, drafts.numpy(), cu.numpy())
    np.testing.assert_array_equal(got["acc"], acc)
    np.testing.assert_array_equal(got["nxt"], nxt)
