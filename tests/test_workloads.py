"""The seeded input generators: determinism, shapes, page tables, draft statistics."""
import numpy as np
import pytest
import torch

import oracle
from diffusion_draft_ar_b200 import workloads as W


def test_meta_of_every_workload():
    for name, w in W.WORKLOADS.items():
        m = W.make_meta(w, seed=0)
        assert m.B == w.B
        assert int(m.cu_block[0]) == 0 and (m.cu_block[1:] >= m.cu_block[:-1]).all()
        used = m.page_table[m.page_table >= 0]
        # every physical page is owned by exactly one (sequence, slot)
        assert used.numel() == m.num_pages
        assert torch.equal(torch.sort(used.long()).values, torch.arange(m.num_pages))
        # each sequence has room for its prefix plus the append headroom
        need = -(-(m.prefix_lens.long() + w.headroom) // w.page_size)
        assert torch.equal(need.to(torch.int32), (m.page_table >= 0).sum(1).to(torch.int32))
        if w.prefix_range:
            lo, hi = w.prefix_range
            assert int(m.prefix_lens.min()) >= lo and int(m.prefix_lens.max()) <= hi
        assert set(m.block_lens.tolist()) <= set(w.block_choices or (w.block,))
    m = W.make_meta(W.WORKLOADS["qwen3_8b"])
    assert m.num_pages == 16 * 129 and m.R == 512


def test_determinism_and_shapes():
    w = W.WORKLOADS["tiny"]
    a = W.WorkloadInputs(w, seed=0)
    b = W.WorkloadInputs(w, seed=0)
    c = W.WorkloadInputs(w, seed=1)
    assert torch.equal(a.k_cache.view(torch.int16), b.k_cache.view(torch.int16))
    assert torch.equal(a.rounds[0].logits, b.rounds[0].logits)
    assert not torch.equal(a.rounds[0].logits, c.rounds[0].logits)
    r = a.rounds[0]
    assert r.q["diffusion"].shape == (8, 4, 64) and r.k_block["verify"].shape == (8, 1, 64)
    assert a.k_cache.shape == (5, 1, 64, 64) and r.logits.shape == (8, 512)
    assert not torch.equal(r.q["diffusion"], r.q["verify"])


def test_bf16_draws_are_rounded_normals():
    g = torch.Generator().manual_seed(0)
    x = W.randn_bf16((1 << 16,), g, "cpu", std=2.0).float()
    assert abs(float(x.mean())) < 0.05 and abs(float(x.std()) - 2.0) < 0.05


def test_draft_rule_selects_targets_with_probability_p():
    n = 200000
    g = torch.Generator().manual_seed(3)
    coins = torch.rand(n, generator=g)
    alt = torch.randint(0, 7, (n,), generator=g).to(torch.int32)
    tgt = torch.full((n,), 9, dtype=torch.int32)
    d = W.drafts_from_targets(tgt, coins, alt, 0.8)
    assert abs(float((d == 9).float().mean()) - 0.8) < 0.005


@pytest.mark.parametrize("p,K", [(0.7, 8), (0.8, 32)])
def test_mean_accept_length_matches_geometric(p, K):
    """With i.i.d. matches of probability p the committed length min(m+1, K) has
    mean (1 - p^K) / (1 - p): a check on the generator, with the oracle deciding
    acceptance from the data."""
    w = W.Workload("stat", B=4000, Hq=1, Hkv=1, D=8, prefix_len=0, block=K, vocab=64,
                   p_match=p, headroom=0)
    wi = W.WorkloadInputs(w, seed=5, with_cache=False)
    r = wi.rounds[0]
    logits = r.logits.numpy()
    cu = wi.meta.cu_block.numpy()
    _, _, am = oracle.consensus(logits, np.zeros(wi.meta.R, np.int32), cu)
    drafts = wi.drafts(0, torch.from_numpy(am)).numpy()
    acc, _, _ = oracle.consensus(logits, drafts, cu)
    # alt may hit the target by chance (1/V): effective p = p + (1-p)/V
    pe = p + (1 - p) / 64
    want = (1 - pe ** K) / (1 - pe)
    assert abs(float(acc.mean()) - want) < 0.05 * want
