"""Block attention on the GPU (tcgen05 + TMA kernel) against the fp64 oracle.

Tolerance: max |err| <= 2e-2 and relative RMS <= 1e-2 over the compared outputs
(bf16 inputs, fp32 accumulation, bf16 output)."""
import numpy as np
import pytest
import torch

import oracle
from diffusion_draft_ar_b200 import workloads as W
from tests._gpu import DevAttn, assert_attn_close, gpu, lib, needs_cuda
from tests._helpers import oracle_attn_args, small_workload

pytestmark = [gpu, needs_cuda]
VIEWS = ["diffusion", "verify"]


def _full_parity(wi, view, **kw):
    d = DevAttn(wi)
    out = d.run(view, **kw)
    ref = oracle.block_attn(*oracle_attn_args(wi, view))
    assert int(d.err.item()) == 0
    return assert_attn_close(out, ref, f"{wi.w.name}/{view}/{kw}")


@pytest.mark.parametrize("view", VIEWS)
def test_tiny_full(view):
    """Tiny: L=256, K=8, 4/1 heads, D=64, contiguous cache."""
    _full_parity(W.WorkloadInputs(W.WORKLOADS["tiny"], seed=0), view)


@pytest.mark.parametrize("view", VIEWS)
def test_qwen3_1p7b_full(view):
    """Qwen3-1.7B-shaped layer: L=4096, K=32, 16/8 heads, D=128, every output checked."""
    _full_parity(W.WorkloadInputs(W.WORKLOADS["qwen3_1p7b"], seed=0), view)


def _ragged(D=128, Hq=8, Hkv=2, choices=(1, 5, 17, 32), lo=0, hi=300, B=6, seed=1, paged=True):
    w = small_workload(name="ragged_small", B=B, Hq=Hq, Hkv=Hkv, D=D, page_size=64,
                       prefix_len=None, prefix_range=(lo, hi), block=None, block_choices=choices,
                       paged=paged, headroom=64)
    return W.WorkloadInputs(w, seed=seed)


@pytest.mark.parametrize("view", VIEWS)
@pytest.mark.parametrize("max_ctas", [0, 1, 3, 7, 50])
def test_ragged_balanced_split(view, max_ctas):
    """Ragged prefixes (partial last pages) and block sizes; 1..148 CTAs so units are
    cut at arbitrary tile boundaries and merged by the combine kernel."""
    _full_parity(_ragged(), view, max_ctas=max_ctas)


@pytest.mark.parametrize("view", VIEWS)
@pytest.mark.parametrize("split", [64, 128, 192])
def test_ragged_fixed_chunks(view, split):
    _full_parity(_ragged(seed=2), view, kv_split=split)


@pytest.mark.parametrize("view", VIEWS)
@pytest.mark.parametrize("split,max_ctas", [(64, 1), (128, 2), (192, 5), (64, 7)])
def test_ragged_fixed_chunks_few_walkers(view, split, max_ctas):
    """Fixed chunks walked by fewer CTAs than chunk slots: CTA c takes slots c,
    c + grid, ... across units and sequences of different lengths, skipping
    the slots past a unit's last chunk; every chunk is merged as one partial."""
    _full_parity(_ragged(seed=2), view, kv_split=split, max_ctas=max_ctas)


@pytest.mark.parametrize("view", VIEWS)
def test_edge_prefix_lengths(view):
    """L in {0, 1, 63, 64, 65, 127, 128} with K in {1, 32}."""
    w = small_workload(name="edges", B=7, Hq=8, Hkv=2, D=128, page_size=64, prefix_len=None,
                       prefix_range=(0, 1), block=None, block_choices=(1, 32), paged=True,
                       headroom=200)
    wi = W.WorkloadInputs(w, seed=3)
    wi.meta.prefix_lens[:] = torch.tensor([0, 1, 63, 64, 65, 127, 128], dtype=torch.int32)
    for ms in (0, 2):
        _full_parity(wi, view, max_ctas=ms)


@pytest.mark.parametrize("view", VIEWS)
@pytest.mark.parametrize("D,Hq,Hkv,K", [(64, 8, 1, 16), (64, 2, 2, 64), (128, 1, 1, 64),
                                         (128, 16, 4, 32)])
def test_head_shapes(view, D, Hq, Hkv, K):
    """GQA groups of 1..8 query heads, G*K from 64 to 128, D 64 and 128."""
    w = small_workload(name="heads", B=3, Hq=Hq, Hkv=Hkv, D=D, page_size=64, prefix_len=None,
                       prefix_range=(30, 400), block=K, paged=True, headroom=64)
    _full_parity(W.WorkloadInputs(w, seed=4), view, max_ctas=5)


@pytest.mark.parametrize("view", VIEWS)
def test_large_pages_and_uniform_blocks(view):
    """128-token pages; cu_block omitted (every block has max_block rows)."""
    w = small_workload(name="p128", B=3, Hq=8, Hkv=2, D=128, page_size=128, prefix_len=None,
                       prefix_range=(100, 700), block=16, paged=True, headroom=64)
    wi = W.WorkloadInputs(w, seed=5)
    d = DevAttn(wi)
    out = d.run(view, cu_block=None, max_ctas=4)
    ref = oracle.block_attn(*oracle_attn_args(wi, view))
    assert_attn_close(out, ref, "p128")


@pytest.mark.parametrize("view", VIEWS)
def test_stale_nan_slots_do_not_leak(view):
    """Cache slots at or past each prefix length hold NaN bit patterns; the output
    must not see them (masked scores and cleared value rows)."""
    wi = _ragged(seed=6)
    m = wi.meta
    for b in range(m.B):
        L = int(m.prefix_lens[b])
        for pidx in range(int(m.pages_per_seq[b])):
            lo = max(0, L - 64 * pidx)
            if lo < 64:
                page = int(m.page_table[b, pidx])
                W.sentinel_fill_(wi.k_cache[page, :, lo:])
                W.sentinel_fill_(wi.v_cache[page, :, lo:])
    _full_parity(wi, view, max_ctas=3)


@pytest.mark.parametrize("view", VIEWS)
def test_empty_blocks(view):
    """Sequences with K_b = 0 contribute no rows and no work."""
    seed = next(s for s in range(100)
                if (W.make_meta(_ragged(choices=(0, 4, 9), seed=s).w, s).block_lens == 0).any())
    wi = _ragged(choices=(0, 4, 9), seed=seed)
    assert (wi.meta.block_lens == 0).any() and wi.meta.R > 0
    _full_parity(wi, view, max_ctas=4)


def test_bad_page_is_flagged_not_faulted():
    wi = _ragged(seed=8)
    d = DevAttn(wi)
    d.page_table[0, 0] = 10 ** 6
    d.run("verify", max_ctas=3)
    assert int(d.err.item()) & lib().FLAG_BAD_PAGE


def test_prefix_beyond_page_table_is_flagged():
    wi = _ragged(seed=9)
    d = DevAttn(wi)
    d.prefix_lens[1] = wi.meta.max_pages * 64 + 1
    d.run("diffusion")
    assert int(d.err.item()) & lib().FLAG_BAD_LENGTH


@pytest.mark.parametrize("view", VIEWS)
def test_few_long_units_proportional_chunks(view):
    """Few units of very different lengths (prefixes of 0, 3000 and 40000 tokens,
    2 KV heads): the default schedule gives every unit SMs in proportion to its
    tiles, cut into near-equal chunks, and merges them; every output checked,
    and the same outputs with an explicit balanced split."""
    w = small_workload(name="few_long", B=3, Hq=8, Hkv=2, D=128, page_size=64, prefix_len=None,
                       prefix_range=(40000, 40000), block=None, block_choices=(32,), paged=True,
                       headroom=64)
    wi = W.WorkloadInputs(w, seed=4)
    wi.meta.prefix_lens[:] = torch.tensor([0, 3000, 40000], dtype=torch.int32)
    _full_parity(wi, view)
    _full_parity(wi, view, max_ctas=148)


@pytest.mark.parametrize("view", VIEWS)
def test_qwen3_8b_full(view):
    """Qwen3-8B-shaped layer (16 x L=8192, K=32, 32/8 heads, random pages) in the
    launch configuration the bench times; every one of the 512 x 32 x 128 outputs
    against the oracle."""
    wi = W.WorkloadInputs(W.WORKLOADS["qwen3_8b"], seed=0, device="cuda")
    _full_parity(wi, view)


@pytest.mark.parametrize("split", [2048, 0])
def test_longctx_full(split):
    """L = 131072, VERIFY view, split over 2048-token chunks (and the library's
    proportional chunks); every output against the oracle."""
    wi = W.WorkloadInputs(W.WORKLOADS["longctx"], seed=0, device="cuda")
    _full_parity(wi, "verify", kv_split=split)


def _bias_block_keys(wi, score: float = 8.0, seed: int = 21):
    """Every query of both views is the same direction u (|q| = 4) and every block
    key is a multiple of u whose score is `score` + N(0, 1), so each block key
    outweighs a prefix key (score ~ N(0, 0.35^2) at D = 128) by about e^8: a wrong
    in-block mask moves outputs by O(1) even behind an 8192-token prefix."""
    w = wi.w
    r = wi.rounds[0]
    g = torch.Generator().manual_seed(seed)
    u = torch.randn(w.D, generator=g, dtype=torch.float64)
    u = u / u.norm()
    s = 1.0 / np.sqrt(w.D)
    q = (4.0 * u).to(torch.bfloat16)
    z = torch.randn(r.k_block["verify"].shape[:2], generator=g, dtype=torch.float64)
    alpha = (score + z) / (s * 4.0)
    kb = (alpha[..., None] * u).to(torch.bfloat16)
    dev = r.q["verify"].device
    for view in VIEWS:
        r.q[view].copy_(q.to(dev).expand_as(r.q[view]))
        r.k_block[view].copy_(kb.to(dev))
        r.v_block[view].copy_(r.v_block["verify"])
    return wi


def test_qwen3_8b_block_bias_mask_sensitivity():
    """Qwen3-8B-shaped layer with block keys scored +8 above the prefix: both views
    match the oracle over every output, and they differ on every row but each
    sequence's last (where the causal row sees the whole block), by O(1) on rows
    that see at most half the block."""
    wi = _bias_block_keys(W.WorkloadInputs(W.WORKLOADS["qwen3_8b"], seed=0, device="cuda"))
    d = DevAttn(wi)
    outs = {}
    for view in VIEWS:
        out = d.run(view)
        ref = oracle.block_attn(*oracle_attn_args(wi, view))
        assert int(d.err.item()) == 0
        assert_attn_close(out, ref, f"qwen3_8b block bias/{view}")
        outs[view] = out.float().cpu().numpy()
    diff = np.abs(outs["diffusion"] - outs["verify"]).max(axis=(1, 2))  # per block row
    K = wi.w.block
    for b in range(wi.meta.B):
        rows = diff[b * K:(b + 1) * K]
        assert rows[:K // 2].min() > 0.1, (b, rows[:K // 2].min())  # at most half the block seen
        assert rows[:K - 1].min() > 0.0, (b, rows[:K - 1].min())
        assert rows[K - 1] == 0.0


def test_views_differ_and_are_deterministic():
    """Same inputs through both views: the DIFFUSION and VERIFY outputs differ on
    every block row but each sequence's last (identical there), and a repeated
    call is bit-identical."""
    wi = _ragged(seed=12)
    d = DevAttn(wi)
    r = wi.rounds[0]
    same = dict(q=r.q["verify"], kb=r.k_block["verify"], vb=r.v_block["verify"])
    a = d.run("verify", max_ctas=5, **same).clone()
    b = d.run("verify", max_ctas=5, **same).clone()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    c = d.run("diffusion", max_ctas=5, **same).clone()
    cu = wi.meta.cu_block.tolist()
    for s in range(wi.meta.B):
        r0, r1 = cu[s], cu[s + 1]
        if r1 - r0 == 0:
            continue
        last_a, last_c = a[r1 - 1], c[r1 - 1]
        assert torch.equal(last_a.view(torch.int16), last_c.view(torch.int16)), s
        if r1 - r0 > 1:
            dd = (a[r0:r1 - 1].float() - c[r0:r1 - 1].float()).abs().amax(dim=(1, 2))
            assert (dd > 0).all(), (s, dd)
