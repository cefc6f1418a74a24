"""Temperature > 0 consensus on the GPU against the fp64 oracle.

Both sides draw the same noise: Philox4x32-10 at counter (v / 4, row, offset),
key = seed, implemented on each side from the generator's published
definition; the oracle scores in fp64, the kernel in fp32. The sampled tokens
must be the oracle's wherever the oracle's winning margin exceeds the fp32
evaluation error (1e-3 here, far above it: a few 1e-6); the accept lengths
and next tokens must equal the oracle's acceptance rule on the kernel's
tokens, bit for bit (and the oracle's own outputs where every token agrees)."""
import numpy as np
import pytest
import torch

import oracle
from diffusion_draft_ar_b200 import workloads as W
from tests._gpu import gpu, lib, needs_cuda

pytestmark = [gpu, needs_cuda]
EPS = 1e-3


def _run(O, logits, drafts, cu, B, K, T, seed, offset, lens=None):
    dev = "cuda"
    acc = torch.full((B,), -7, dtype=torch.int32, device=dev)
    nxt = torch.full((B,), -7, dtype=torch.int32, device=dev)
    tok = torch.full((drafts.numel(),), -7, dtype=torch.int32, device=dev)
    ws = torch.empty(O.consensus_workspace_size(B, K, logits.shape[1]), dtype=torch.uint8,
                     device=dev)
    O.consensus_sampled(logits, drafts, cu, B, K, T, seed, offset, acc, nxt, ws, row_token=tok,
                        prefix_lens=lens)
    torch.cuda.synchronize()
    return acc.cpu().numpy(), nxt.cpu().numpy(), tok.cpu().numpy()


def _check(logits_np, drafts_np, cu_np, got, T, seed, offset, what):
    acc, nxt, tok = got
    t_o, margin = oracle.sampled_tokens(logits_np, T, seed, offset)
    diff = tok != t_o
    # a different token is allowed only on a near-tie of the exact scores
    assert np.all(margin[diff] <= EPS), (what, np.flatnonzero(diff)[:8], margin[diff][:8])
    assert diff.sum() <= max(1, len(tok) // 1000), (what, diff.sum())
    a2, n2 = oracle.accept_from_tokens(tok, drafts_np, cu_np)
    np.testing.assert_array_equal(acc, a2)
    np.testing.assert_array_equal(nxt, n2)
    if not diff.any():
        a3, n3, t3 = oracle.consensus_sampled(logits_np, drafts_np, cu_np, T, seed, offset)
        np.testing.assert_array_equal(acc, a3)
        np.testing.assert_array_equal(nxt, n3)
        np.testing.assert_array_equal(tok, t3)
    return t_o


def _drafts_from(t_o, coins, alt, p):
    return np.where(coins < p, t_o, alt).astype(np.int32)


@pytest.mark.parametrize("name,T,seed,offset", [
    ("tiny", 0.7, 1, 0), ("tiny", 1.6, 2, 5),
    ("qwen3_1p7b", 1.0, 3, 0), ("qwen3_1p7b", 0.6, 4, 1 << 33),
    ("qwen3_8b", 1.0, 5, 7), ("ragged", 0.8, 6, 2),
])
def test_sampled_consensus_matches_oracle(name, T, seed, offset):
    O = lib()
    wi = W.WorkloadInputs(W.WORKLOADS[name], seed=seed, with_cache=False, rounds=1, device="cuda")
    m, r = wi.meta, wi.rounds[0]
    logits_np = r.logits.cpu().numpy()
    cu_np = m.cu_block.numpy()
    t_o, _ = oracle.sampled_tokens(logits_np, T, seed, offset)
    drafts_np = _drafts_from(t_o, r.coins.cpu().numpy(), r.alt.cpu().numpy(),
                             wi.row_p_match().numpy())
    got = _run(O, r.logits, torch.from_numpy(drafts_np).cuda(), m.cu_block.cuda(), m.B,
               wi.w.max_block, T, seed, offset)
    _check(logits_np, drafts_np, cu_np, got, T, seed, offset, name)
    # the drafts were built from the samples, so on a batch most sequences
    # accept several
    if m.B >= 16:
        assert got[0].mean() > 1.5


def test_sampled_consensus_commit_unaligned_rows_and_special_values():
    """Rows not 16-byte aligned (ld = V + 1), NaN and -inf columns, a vocabulary
    that is not a multiple of 4, and the commit of the lengths."""
    O = lib()
    g = np.random.default_rng(3)
    K = [4, 1, 9, 6]
    cu_np = np.concatenate([[0], np.cumsum(K)]).astype(np.int32)
    R, V = int(cu_np[-1]), 20001
    base = g.standard_normal((R, V + 1)).astype(np.float32) * 2
    base[:, 5::7] = np.nan
    base[:, 3::11] = -np.inf
    dev_full = torch.from_numpy(base).cuda()
    logits = dev_full[:, :V]                       # row stride V + 1: rows not 16-byte aligned
    logits_np = np.ascontiguousarray(base[:, :V])
    T, seed, offset = 1.3, 99, 12
    t_o, _ = oracle.sampled_tokens(logits_np, T, seed, offset)
    drafts_np = np.where(g.random(R) < 0.7, t_o, g.integers(0, V, R)).astype(np.int32)
    lens0 = np.array([100, 7, 0, 55], np.int32)
    lens = torch.from_numpy(lens0.copy()).cuda()
    got = _run(O, logits, torch.from_numpy(drafts_np).cuda(), torch.from_numpy(cu_np).cuda(),
               len(K), max(K), T, seed, offset, lens=lens)
    _check(logits_np, drafts_np, cu_np, got, T, seed, offset, "unaligned")
    np.testing.assert_array_equal(lens.cpu().numpy(), lens0 + got[0])
    assert not np.isnan(logits_np[np.arange(R), got[2]]).any()
    assert np.isfinite(logits_np[np.arange(R), got[2]]).all()


def test_all_drafts_right_and_first_wrong():
    O = lib()
    g = np.random.default_rng(4)
    K, B, V = 8, 5, 4096
    cu_np = np.arange(0, (B + 1) * K, K, dtype=np.int32)
    logits_np = g.standard_normal((B * K, V)).astype(np.float32)
    logits = torch.from_numpy(logits_np).cuda()
    T, seed, offset = 0.9, 7, 3
    t_o, _ = oracle.sampled_tokens(logits_np, T, seed, offset)
    cu = torch.from_numpy(cu_np).cuda()
    acc, nxt, tok = _run(O, logits, torch.from_numpy(t_o).cuda(), cu, B, K, T, seed, offset)
    assert acc.tolist() == [K] * B and nxt.tolist() == t_o[K - 1::K].tolist()
    wrong = t_o.copy()
    wrong[::K] = (t_o[::K] + 1) % V
    acc, nxt, _ = _run(O, logits, torch.from_numpy(wrong).cuda(), cu, B, K, T, seed, offset)
    assert acc.tolist() == [1] * B and nxt.tolist() == t_o[::K].tolist()
