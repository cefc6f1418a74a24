"""Write-then-truncate VERIFY against the oracle.

The technical summary §2.3 item 3 commits a round by writing the AR view's KV
for the whole block and truncating the cache to the accepted prefix. On the
GPU that is ``orthrus_block_attn_verify_write`` (the VERIFY attention launch
also stores every block row's K/V past the prefix) followed by
``orthrus_consensus_commit`` (the lengths advance by the accepted counts).

Its oracle is the plain definition spelled with the pinned oracle calls: the
cache after the attention call equals ``oracle.kv_append`` of ALL K_b rows with
the lengths left alone, and the lengths after the commit equal L_b + n_b with
n_b from ``oracle.consensus``. Checked here:
  - attention outputs bit-identical to ``orthrus_block_attn`` (same kernel and
    schedule, the writer warp only adds stores), in every schedule mode;
  - the whole K and V caches bit-exact against the oracle's full-block write
    (so no other byte is touched), lengths unchanged by the attention call;
  - consensus outputs and committed lengths bit-exact;
  - chained ragged rounds: lengths every round and, at the end, every cache
    slot below each final length bit-exact against the oracle chain that
    appends only the accepted rows (slots past the length are free);
  - a page table too short for the block flags BAD_LENGTH and writes nothing
    past it.
"""
import numpy as np
import pytest
import torch

import oracle
from diffusion_draft_ar_b200 import workloads as W
from tests._gpu import gpu, lib, needs_cuda

pytestmark = [gpu, needs_cuda]

CASES = [
    ("tiny", {}),
    ("qwen3_1p7b", {}),
    ("qwen3_8b", {}),                            # one CTA per unit
    ("qwen3_8b", {"max_ctas": 148}),             # balanced ranges + combine
    ("qwen3_8b", {"max_ctas": 37}),              # several units per CTA
    ("qwen3_8b", {"kv_split_tokens": 2048}),     # fixed chunks + combine
    ("longctx", {"kv_split_tokens": 2048}),
]


def _attn(O, fn, r, kc, vc, lens, cu, table, w, err, **kw):
    q, kb, vb = r.q["verify"], r.k_block["verify"], r.v_block["verify"]
    out = torch.full_like(q, float("nan"))
    p = O.attn_params("verify", q, kc, vc, kb, vb, lens, cu, table, out, w.max_block, **kw)
    ws = torch.empty(O.block_attn_workspace_size(p), dtype=torch.uint8, device="cuda")
    if fn == "plain":
        O.block_attn("verify", q, kc, vc, kb, vb, lens, cu, table, out, ws, w.max_block,
                     error_flag=err, **kw)
    else:
        O.block_attn_verify_write(q, kc, vc, kb, vb, lens, cu, table, out, ws, w.max_block,
                                  error_flag=err, **kw)
    return out


@pytest.mark.parametrize("name,kw", CASES, ids=[f"{n}-{'-'.join(f'{k}{v}' for k, v in kw.items()) or 'default'}"
                                                for n, kw in CASES])
def test_verify_write_matches_oracle(name, kw):
    O = lib()
    w = W.WORKLOADS[name]
    wi = W.WorkloadInputs(w, device="cuda", seed=0, rounds=1)
    m = wi.meta
    r = wi.rounds[0]
    lens, cu, table = m.prefix_lens.cuda(), m.cu_block.cuda(), m.page_table.cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kc0_bits, vc0_bits = W.bf16_bits(wi.k_cache), W.bf16_bits(wi.v_cache)

    ref_out = _attn(O, "plain", r, wi.k_cache, wi.v_cache, lens, cu, table, w, err, **kw)
    kc, vc = wi.k_cache.clone(), wi.v_cache.clone()
    out = _attn(O, "write", r, kc, vc, lens, cu, table, w, err, **kw)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))
    np.testing.assert_array_equal(lens.cpu().numpy(), m.prefix_lens.numpy())

    # oracle: every block row written past its prefix, lengths unchanged
    kc_o, vc_o = kc0_bits.copy(), vc0_bits.copy()
    lens_o = m.prefix_lens.numpy().copy()
    all_rows = m.block_lens.numpy().astype(np.int32)
    assert oracle.kv_append(W.bf16_bits(r.k_block["verify"]), W.bf16_bits(r.v_block["verify"]),
                            m.cu_block.numpy(), all_rows, lens_o, m.page_table.numpy(),
                            kc_o, vc_o, update_lens=False) == 0
    assert np.array_equal(W.bf16_bits(kc), kc_o)
    assert np.array_equal(W.bf16_bits(vc), vc_o)

    if w.vocab is None:
        return
    # commit: consensus advances the lengths by the accepted counts
    logits_np = r.logits.cpu().numpy()
    cu_np = m.cu_block.numpy()
    _, _, t = oracle.consensus(logits_np, np.zeros(m.R, np.int32), cu_np)
    drafts = wi.drafts(0, torch.from_numpy(t).cuda())
    acc_o, nxt_o, _ = oracle.consensus(logits_np, drafts.cpu().numpy(), cu_np)
    acc = torch.empty(m.B, dtype=torch.int32, device="cuda")
    nxt = torch.empty_like(acc)
    ws = torch.empty(O.consensus_workspace_size(m.B, w.max_block, w.vocab), dtype=torch.uint8,
                     device="cuda")
    O.consensus(r.logits, drafts, cu, m.B, w.max_block, acc, nxt, ws, prefix_lens=lens)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
    np.testing.assert_array_equal(nxt.cpu().numpy(), nxt_o)
    np.testing.assert_array_equal(lens.cpu().numpy(), m.prefix_lens.numpy() + acc_o)


def _free_slot_mask(lens: np.ndarray, table: np.ndarray, pages_per_seq: np.ndarray,
                    num_pages: int, P: int) -> torch.Tensor:
    """[num_pages, P] bool: slots at or past their sequence's length (no content
    is owed there). Every page belongs to one sequence in these workloads."""
    mask = torch.zeros(num_pages, P, dtype=torch.bool)
    for b in range(lens.shape[0]):
        for pidx in range(int(lens[b]) // P, int(pages_per_seq[b])):
            start = max(int(lens[b]) - pidx * P, 0)
            mask[int(table[b, pidx]), start:] = True
    return mask


def test_ragged_chain_write_then_truncate():
    """Four chained ragged rounds (64 sequences, L_b in 512..32768, K_b in
    {8, 16, 32}) through DIFFUSION attention -> verify_write -> consensus_commit,
    against the oracle chain that appends only the accepted rows."""
    O = lib()
    w = W.WORKLOADS["ragged"]
    rounds = 4
    wi = W.WorkloadInputs(w, device="cuda", seed=0, rounds=rounds)
    m = wi.meta
    dev = "cuda"
    kc, vc = wi.k_cache, wi.v_cache
    lens, cu, table = m.prefix_lens.to(dev), m.cu_block.to(dev), m.page_table.to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    kc_o, vc_o = W.bf16_bits(kc).copy(), W.bf16_bits(vc).copy()
    lens_o = m.prefix_lens.numpy().copy()
    cu_np, table_np = m.cu_block.numpy(), m.page_table.numpy()
    ws_cons = torch.empty(O.consensus_workspace_size(m.B, w.max_block, w.vocab), dtype=torch.uint8,
                          device=dev)
    acc = torch.empty(m.B, dtype=torch.int32, device=dev)
    nxt = torch.empty(m.B, dtype=torch.int32, device=dev)
    for rnd in range(rounds):
        r = wi.rounds[rnd]
        q, kb, vb = r.q["diffusion"], r.k_block["diffusion"], r.v_block["diffusion"]
        out_d = torch.empty_like(q)
        p = O.attn_params("diffusion", q, kc, vc, kb, vb, lens, cu, table, out_d, w.max_block)
        ws = torch.empty(O.block_attn_workspace_size(p), dtype=torch.uint8, device=dev)
        O.block_attn("diffusion", q, kc, vc, kb, vb, lens, cu, table, out_d, ws, w.max_block,
                     error_flag=err)
        _attn(O, "write", r, kc, vc, lens, cu, table, w, err)
        logits_np = r.logits.cpu().numpy()
        _, _, t = oracle.consensus(logits_np, np.zeros(m.R, np.int32), cu_np)
        drafts = wi.drafts(rnd, torch.from_numpy(t).to(dev))
        acc_o, nxt_o, _ = oracle.consensus(logits_np, drafts.cpu().numpy(), cu_np)
        O.consensus(r.logits, drafts, cu, m.B, w.max_block, acc, nxt, ws_cons, prefix_lens=lens)
        assert oracle.kv_append(W.bf16_bits(r.k_block["verify"]), W.bf16_bits(r.v_block["verify"]),
                                cu_np, acc_o, lens_o, table_np, kc_o, vc_o) == 0
        torch.cuda.synchronize()
        np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
        np.testing.assert_array_equal(nxt.cpu().numpy(), nxt_o)
        np.testing.assert_array_equal(lens.cpu().numpy(), lens_o)
    assert int(err.item()) == 0
    free = _free_slot_mask(lens_o, table_np, m.pages_per_seq.numpy(), m.num_pages, w.page_size)
    free = free.to(dev)[:, None, :, None]  # [pages, 1, P, 1] over [pages, Hkv, P, D]
    for got, want in ((kc, kc_o), (vc, vc_o)):
        g = got.view(torch.int16).masked_fill(free, 0)
        e = torch.from_numpy(want.view(np.int16)).to(dev).masked_fill(free, 0)
        assert torch.equal(g, e)
        del e


def test_short_table_flags_and_skips():
    """qwen3_1p7b with the page table cut to the prefix's pages: the block rows
    have no page, so the writer flags BAD_LENGTH and writes no cache byte; the
    attention outputs are still those of the plain VERIFY call."""
    O = lib()
    w = W.WORKLOADS["qwen3_1p7b"]
    wi = W.WorkloadInputs(w, device="cuda", seed=0, rounds=1)
    m = wi.meta
    r = wi.rounds[0]
    L = int(m.prefix_lens[0])
    table = m.page_table[:, : L // w.page_size].contiguous().cuda()
    lens, cu = m.prefix_lens.cuda(), m.cu_block.cuda()
    err0 = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref = _attn(O, "plain", r, wi.k_cache, wi.v_cache, lens, cu, table, w, err0)
    kc, vc = wi.k_cache.clone(), wi.v_cache.clone()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _attn(O, "write", r, kc, vc, lens, cu, table, w, err)
    torch.cuda.synchronize()
    assert int(err0.item()) == 0
    assert int(err.item()) == 0x2  # ORTHRUS_FLAG_BAD_LENGTH only
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    assert torch.equal(kc.view(torch.int16), wi.k_cache.view(torch.int16))
    assert torch.equal(vc.view(torch.int16), wi.v_cache.view(torch.int16))
