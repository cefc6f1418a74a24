"""orthrus_consensus_noalloc: the consensus entry point for callers that cannot
allocate device memory when they call in (an engine that reserves all of HBM
up front and gives plug-ins no scratch, or a decode path that must not pay for
cudaMalloc's implicit synchronisation). Its scratch is a fixed array inside the
library, shared by every call on a device.

Checked through the C ABI against the workspace-taking orthrus_consensus and
against the oracle, bit for bit (the tolerance every consensus test uses), on
two calls in a row with different inputs: the larger request first, then a
smaller one that reads array slots the first call wrote, so the second call
cannot pass on what the first left behind. (The size limit is checked on the
host, without a GPU, in test_abi.py.) This file is named to be collected last."""
import numpy as np
import torch

import oracle
from diffusion_draft_ar_b200 import workloads as W
from tests._gpu import gpu, lib, needs_cuda

pytestmark = [gpu, needs_cuda]


def _inputs(name, seed):
    wi = W.WorkloadInputs(W.WORKLOADS[name], seed=seed, with_cache=False, device="cuda")
    r = wi.rounds[0]
    targets = torch.argmax(r.logits, dim=1).to(torch.int32)
    return wi, r.logits, wi.drafts(0, targets)


def _with_workspace(O, logits, drafts, cu, B, K):
    acc = torch.full((B,), -5, dtype=torch.int32, device="cuda")
    nxt = torch.full((B,), -5, dtype=torch.int32, device="cuda")
    am = torch.full((drafts.numel(),), -5, dtype=torch.int32, device="cuda")
    ws = torch.empty(O.consensus_workspace_size(B, K, logits.shape[1]), dtype=torch.uint8,
                     device="cuda")
    O.consensus(logits, drafts, cu, B, K, acc, nxt, ws, row_argmax=am)
    return acc, nxt, am


def _without_workspace(O, logits, drafts, cu, B, K):
    acc = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    nxt = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    am = torch.full((drafts.numel(),), -9, dtype=torch.int32, device="cuda")
    O.consensus_noalloc(logits, drafts, cu, B, K, acc, nxt, row_argmax=am)
    return acc, nxt, am


def test_noalloc_matches_workspace_entry_point_and_oracle_twice_in_a_row():
    O = lib()
    # larger request first (ragged: 64 sequences, ~1200 rows), then a smaller one
    # (Qwen3-8B: 512 rows) whose keys occupy slots the first call wrote
    cases = [_inputs("ragged", 1), _inputs("qwen3_8b", 0)]
    assert cases[0][1].shape[0] > cases[1][1].shape[0]
    for wi, logits, drafts in cases:
        cu = wi.meta.cu_block.cuda()
        ref = _with_workspace(O, logits, drafts, cu, wi.meta.B, wi.w.max_block)
        got = _without_workspace(O, logits, drafts, cu, wi.meta.B, wi.w.max_block)
        torch.cuda.synchronize()
        for a, b in zip(got, ref):
            assert torch.equal(a, b)
        acc_o, nxt_o, am_o = oracle.consensus(logits.cpu().numpy(), drafts.cpu().numpy(),
                                              wi.meta.cu_block.numpy())
        np.testing.assert_array_equal(got[0].cpu().numpy(), acc_o)
        np.testing.assert_array_equal(got[1].cpu().numpy(), nxt_o)
        np.testing.assert_array_equal(got[2].cpu().numpy(), am_o)
        assert int(got[0].min()) >= 1
