"""orthrus_consensus_noalloc: the consensus entry point for callers that cannot
allocate device memory when they call in (an engine that reserves all of HBM
up front and gives plug-ins no scratch, or a decode path that must not pay for
cudaMalloc's implicit synchronisation). Its scratch is a fixed array inside the
library, shared by every call on a device.

Checked through the C ABI against the workspace-taking orthrus_consensus, bit
for bit (the tolerance every consensus test uses), on two calls in a row with
different inputs, so a second call cannot pass on what the first left behind.
This file is named to be collected last."""
import ctypes

import numpy as np
import pytest
import torch

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


def test_noalloc_matches_workspace_entry_point_twice_in_a_row():
    O = lib()
    cases = [_inputs("qwen3_8b", 0), _inputs("ragged", 1)]
    for wi, logits, drafts in cases:   # two calls in a row, different shapes and data
        cu = wi.meta.cu_block.cuda()
        ref = _with_workspace(O, logits, drafts, cu, wi.meta.B, wi.w.max_block)
        got = _without_workspace(O, logits, drafts, cu, wi.meta.B, wi.w.max_block)
        torch.cuda.synchronize()
        for a, b in zip(got, ref):
            assert torch.equal(a, b)
        assert int(got[0].min()) >= 1


def test_noalloc_rejects_requests_beyond_its_array():
    O = lib()
    V = 151936
    B, K = 300, 32      # 9600 rows x 10 chunks = 96000 keys > 65536
    st = O.lib.orthrus_consensus_noalloc(ctypes.c_void_p(16), V, V, ctypes.c_void_p(16), None,
                                         B, K, ctypes.c_void_p(16), ctypes.c_void_p(16), None,
                                         None)
    assert st == O.ERR_UNSUPPORTED
    assert b"scratch" in O.lib.orthrus_last_error()
