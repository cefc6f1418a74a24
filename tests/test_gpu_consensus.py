"""Greedy consensus on the GPU against the oracle: bit-exact accept lengths,
correction tokens and per-row greedy tokens."""
import numpy as np
import pytest
import torch

import oracle
from diffusion_draft_ar_b200 import workloads as W
from tests._gpu import gpu, lib, needs_cuda

pytestmark = [gpu, needs_cuda]


def run_gpu(logits: torch.Tensor, drafts: torch.Tensor, cu_block, B: int, max_block: int,
            with_argmax: bool = True):
    O = lib()
    dev = "cuda"
    x = logits.to(dev)
    d = drafts.to(dev)
    cu = cu_block.to(dev) if cu_block is not None else None
    acc = torch.full((B,), -7, dtype=torch.int32, device=dev)
    nxt = torch.full((B,), -7, dtype=torch.int32, device=dev)
    R = d.shape[0]
    am = torch.full((R,), -7, dtype=torch.int32, device=dev) if with_argmax else None
    ws = torch.empty(O.consensus_workspace_size(B, max_block, x.shape[1]), dtype=torch.uint8,
                     device=dev)
    O.consensus(x, d, cu, B, max_block, acc, nxt, ws, row_argmax=am)
    torch.cuda.synchronize()
    return acc.cpu().numpy(), nxt.cpu().numpy(), (am.cpu().numpy() if with_argmax else None)


def check(logits, drafts, cu_block, B, max_block, with_argmax=True):
    x = logits.cpu().numpy() if isinstance(logits, torch.Tensor) else logits
    cu = cu_block if cu_block is not None else torch.arange(0, B * max_block + 1, max_block,
                                                           dtype=torch.int32)
    ra, rn, rm = oracle.consensus(x, drafts.cpu().numpy(), cu.cpu().numpy())
    ga, gn, gm = run_gpu(torch.as_tensor(x), drafts, cu_block, B, max_block, with_argmax)
    np.testing.assert_array_equal(ga, ra)
    np.testing.assert_array_equal(gn, rn)
    if with_argmax:
        np.testing.assert_array_equal(gm, rm)
    return ra


def workload_case(name, seed=0):
    wi = W.WorkloadInputs(W.WORKLOADS[name], seed=seed, with_cache=False)
    r = wi.rounds[0]
    _, _, t = oracle.consensus(r.logits.numpy(), np.zeros(wi.meta.R, np.int32),
                               wi.meta.cu_block.numpy())
    drafts = wi.drafts(0, torch.from_numpy(t))
    return wi, r.logits, drafts


@pytest.mark.parametrize("name", ["tiny", "qwen3_1p7b", "qwen3_8b", "ragged"])
def test_workloads_bit_exact(name):
    wi, logits, drafts = workload_case(name)
    acc = check(logits, drafts, wi.meta.cu_block, wi.meta.B, wi.w.max_block)
    assert acc.min() >= 1


def test_without_row_argmax_and_uniform_blocks():
    wi, logits, drafts = workload_case("qwen3_1p7b", seed=3)
    check(logits, drafts, None, 1, 32, with_argmax=False)


def test_special_values():
    V = 1000
    rows = np.random.default_rng(0).standard_normal((12, V)).astype(np.float32)
    nan, inf = np.float32("nan"), np.float32("inf")
    rows[0, :] = nan                                   # all NaN -> 0
    rows[1, :] = -inf                                  # all -inf -> 0
    rows[2, 500] = inf; rows[2, 700] = inf             # first +inf
    rows[3, :] = 0.0; rows[3, 10] = -0.0               # zeros tie -> index 0
    rows[4, :] = -1.0; rows[4, 999] = -0.0; rows[4, 3] = 0.0   # -0 == +0 -> 3
    rows[5, ::2] = nan                                  # NaNs interleaved
    m = rows[6].max(); rows[6, 999] = m; rows[6, 998] = m       # tie at the tail
    rows[7, 0] = 100.0; rows[7, 17] = 100.0             # tie at the head
    rows[8, :] = 5.0                                     # all equal -> 0
    rows[9, 16383 % V] = 50.0
    cu = torch.tensor([0, 4, 8, 12], dtype=torch.int32)
    drafts = torch.zeros(12, dtype=torch.int32)
    check(rows, drafts, cu, 3, 4)


@pytest.mark.parametrize("V,ld", [(1003, 1003), (1003, 1005), (151936, 151937), (16385, 16385),
                                  (5, 8), (1, 1)])
def test_odd_vocab_and_unaligned_rows(V, ld):
    """Rows that start off a 16-byte boundary and vocabularies that are not a
    multiple of 4 or of the chunk size."""
    g = np.random.default_rng(V + ld)
    R = 24
    buf = g.standard_normal((R, ld)).astype(np.float32)
    # repeat the row maximum at a later index to check tie handling across chunks
    for r in range(R):
        j = int(buf[r, :V].argmax())
        buf[r, max(0, V - 1 - (r % 3))] = buf[r, j]
    t = buf[:, :V].argmax(1)
    drafts = torch.from_numpy(np.where(g.random(R) < 0.8, t, (t + 1) % V).astype(np.int32))
    cu = torch.tensor([0, 5, 5, 12, 24], dtype=torch.int32)
    O = lib()
    x = torch.from_numpy(buf).cuda()
    view = x[:, :V]
    assert view.stride(0) == ld
    acc = torch.zeros(4, dtype=torch.int32, device="cuda")
    nxt = torch.zeros(4, dtype=torch.int32, device="cuda")
    am = torch.zeros(R, dtype=torch.int32, device="cuda")
    ws = torch.empty(O.consensus_workspace_size(4, 12, V), dtype=torch.uint8, device="cuda")
    O.consensus(view, drafts.cuda(), cu.cuda(), 4, 12, acc, nxt, ws, row_argmax=am)
    ra, rn, rm = oracle.consensus(np.ascontiguousarray(buf[:, :V]), drafts.numpy(), cu.numpy())
    np.testing.assert_array_equal(am.cpu().numpy(), rm)
    np.testing.assert_array_equal(acc.cpu().numpy(), ra)
    np.testing.assert_array_equal(nxt.cpu().numpy(), rn)


def test_accept_rule_cases():
    """All match -> K; first mismatch -> 1; mismatch at j -> j+1; block of 64 rows."""
    g = np.random.default_rng(5)
    K, V = 64, 777
    x = g.standard_normal((4 * K, V)).astype(np.float32)
    t = x.argmax(1).astype(np.int32)
    d = t.copy()
    d[K + 0] = (t[K] + 1) % V            # sequence 1: first draft wrong
    d[2 * K + 40] = (t[2 * K + 40] + 1) % V  # sequence 2: wrong at 40 (second warp chunk)
    d[3 * K + 63] = (t[3 * K + 63] + 1) % V  # sequence 3: only the last is wrong
    cu = torch.arange(0, 4 * K + 1, K, dtype=torch.int32)
    acc = check(x, torch.from_numpy(d), cu, 4, K)
    assert list(acc) == [K, 1, 41, K]


def test_empty_batch():
    O = lib()
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    z = torch.empty(0, dtype=torch.int32, device="cuda")
    O.consensus(torch.zeros((0, 8), device="cuda"), z, torch.zeros(1, dtype=torch.int32,
                device="cuda"), 0, 4, z, z, ws)
