"""Eight chained Orthrus rounds on the ragged serving batch (64 sequences, prefix
lengths 512..32768, per-sequence blocks of 8/16/32, random page table), GPU
against the oracle, as the decoding loop of the technical summary §2.3 runs them:
DIFFUSION attention -> VERIFY attention -> consensus -> append, with each
round's lengths coming from the previous round's append on the device.

Checked every round: consensus outputs bit-exact, lengths bit-exact, attention
outputs of both views within tolerance (every output in the first and the last
round, sampled (row, head) pairs in between); after the last round the whole K
and V caches bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from diffusion_draft_ar_b200 import workloads as W
from tests._gpu import assert_attn_close, gpu, lib, needs_cuda, sample_pairs
from tests._helpers import VIEW_ID

pytestmark = [gpu, needs_cuda]


def test_ragged_eight_rounds_chain():
    O = lib()
    w = W.WORKLOADS["ragged"]
    wi = W.WorkloadInputs(w, device="cuda", seed=0)
    m = wi.meta
    dev = "cuda"
    # device state
    kc, vc = wi.k_cache, wi.v_cache
    lens = m.prefix_lens.to(dev)
    cu, table = m.cu_block.to(dev), m.page_table.to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    # oracle state
    kc_o, vc_o = W.bf16_bits(kc).copy(), W.bf16_bits(vc).copy()
    lens_o = m.prefix_lens.numpy().copy()
    cu_np, table_np = m.cu_block.numpy(), m.page_table.numpy()
    ws_attn = None
    ws_cons = torch.empty(O.consensus_workspace_size(m.B, w.max_block, w.vocab), dtype=torch.uint8,
                          device=dev)
    acc = torch.empty(m.B, dtype=torch.int32, device=dev)
    nxt = torch.empty(m.B, dtype=torch.int32, device=dev)
    am = torch.empty(m.R, dtype=torch.int32, device=dev)
    total_accepted = 0
    for rnd in range(w.rounds):
        r = wi.rounds[rnd]
        # --- attention, both views, against the oracle on the current state: every
        # output in the first and the last round, sampled outputs in between
        full = rnd in (0, w.rounds - 1)
        for view in W.VIEW_NAMES:
            out = torch.empty_like(r.q[view])
            p = O.attn_params(view, r.q[view], kc, vc, r.k_block[view], r.v_block[view], lens, cu,
                              table, out, w.max_block)
            n = O.block_attn_workspace_size(p)
            if ws_attn is None or ws_attn.numel() < n:
                ws_attn = torch.empty(n, dtype=torch.uint8, device=dev)
            O.block_attn(view, r.q[view], kc, vc, r.k_block[view], r.v_block[view], lens, cu, table,
                         out, ws_attn, w.max_block, error_flag=err)
            args = (VIEW_ID[view], W.bf16_bits(r.q[view]), kc_o, vc_o,
                    W.bf16_bits(r.k_block[view]), W.bf16_bits(r.v_block[view]), lens_o, cu_np,
                    table_np)
            if full:
                assert_attn_close(out, oracle.block_attn(*args), f"round {rnd} {view} (all)")
            else:
                rows, heads = sample_pairs(m, w.Hq, 48, seed=100 * rnd + VIEW_ID[view])
                ref = oracle.block_attn(*args, sel=(rows, heads))
                got = out[torch.from_numpy(rows).to(dev), torch.from_numpy(heads).long().to(dev)]
                assert_attn_close(got, ref, f"round {rnd} {view} (sampled)")
        # --- consensus: drafts built from the oracle's greedy tokens of this round
        logits_np = r.logits.cpu().numpy()
        _, _, t = oracle.consensus(logits_np, np.zeros(m.R, np.int32), cu_np)
        drafts = wi.drafts(rnd, torch.from_numpy(t).to(dev))
        acc_o, nxt_o, am_o = oracle.consensus(logits_np, drafts.cpu().numpy(), cu_np)
        O.consensus(r.logits, drafts, cu, m.B, w.max_block, acc, nxt, ws_cons, row_argmax=am)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
        np.testing.assert_array_equal(nxt.cpu().numpy(), nxt_o)
        np.testing.assert_array_equal(am.cpu().numpy(), am_o)
        # --- commit: append the VERIFY rows, lengths advance on the device
        O.kv_append(r.k_block["verify"], r.v_block["verify"], cu, w.max_block, acc, lens, table,
                    kc, vc, update_lens=True, error_flag=err)
        assert oracle.kv_append(W.bf16_bits(r.k_block["verify"]), W.bf16_bits(r.v_block["verify"]),
                                cu_np, acc_o, lens_o, table_np, kc_o, vc_o) == 0
        torch.cuda.synchronize()
        np.testing.assert_array_equal(lens.cpu().numpy(), lens_o)
        total_accepted += int(acc_o.sum())
    assert int(err.item()) == 0
    assert np.array_equal(W.bf16_bits(kc), kc_o)
    assert np.array_equal(W.bf16_bits(vc), vc_o)
    # p_b ~ U[0.5, 0.95] and K_b in {8, 16, 32}: several tokens per sequence per round
    assert total_accepted / (w.rounds * m.B) > 2.0
