"""Pins for the oracle's block attention (both views) against things other than itself.

* library special cases: torch SDPA in fp64 (unmasked = DIFFUSION with L=0,
  is_causal = VERIFY with L=0, explicit boolean mask for any L, GQA by SDPA's
  own grouping);
* AR equivalence: a VERIFY row equals single-query causal decode at position
  L+i (Orthrus technical summary §2.3 item 2 and the losslessness claim of §3);
* closed forms: q = 0 gives the mean of the visible values; one key with a huge
  score margin gives that key's value;
* invariances: page permutation, split-KV chunking;
* brute force on tiny integer inputs in the pages' own form (a full-sequence
  mask matrix: M_diff of technical summary §2.2 for DIFFUSION, plain causal for
  VERIFY), written in pure Python.
"""
import itertools
import math
import random

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from diffusion_draft_ar_b200 import workloads as W
from tests._helpers import VIEW_ID, oracle_attn_args, small_workload

TOL = 1e-12


def _contiguous_kv(wi: W.WorkloadInputs, b: int):
    """Prefix K/V of sequence b from an identity page table, by reshaping only.

    With an identity table, sequence b owns physical pages
    [sum(pages[:b]), ...) in order, so its tokens are those pages laid end to end.
    """
    m = wi.meta
    assert not wi.w.paged
    first = int(m.pages_per_seq[:b].sum())
    n = int(m.pages_per_seq[b])
    L = int(m.prefix_lens[b])
    k = wi.k_cache[first:first + n].double()  # [n, Hkv, P, D]
    v = wi.v_cache[first:first + n].double()
    k = k.permute(1, 0, 2, 3).reshape(wi.w.Hkv, n * wi.w.page_size, wi.w.D)[:, :L]
    v = v.permute(1, 0, 2, 3).reshape(wi.w.Hkv, n * wi.w.page_size, wi.w.D)[:, :L]
    return k, v


def _sdpa_reference(wi: W.WorkloadInputs, view: str, round_idx: int = 0) -> np.ndarray:
    """fp64 SDPA over [prefix; block] keys with the view's boolean mask."""
    w, m = wi.w, wi.meta
    r = wi.rounds[round_idx]
    out = torch.zeros((m.R, w.Hq, w.D), dtype=torch.float64)
    for b in range(m.B):
        r0, r1 = int(m.cu_block[b]), int(m.cu_block[b + 1])
        K = r1 - r0
        if K == 0:
            continue
        L = int(m.prefix_lens[b])
        kp, vp = _contiguous_kv(wi, b)
        kb = r.k_block[view][r0:r1].double().permute(1, 0, 2)  # [Hkv, K, D]
        vb = r.v_block[view][r0:r1].double().permute(1, 0, 2)
        keys = torch.cat([kp, kb], dim=1)
        vals = torch.cat([vp, vb], dim=1)
        q = r.q[view][r0:r1].double().permute(1, 0, 2)  # [Hq, K, D]
        mask = torch.ones((K, L + K), dtype=torch.bool)
        if view == "verify":
            mask[:, L:] = torch.tril(torch.ones((K, K), dtype=torch.bool))
        o = F.scaled_dot_product_attention(q, keys, vals, attn_mask=mask, enable_gqa=True)
        out[r0:r1] = o.permute(1, 0, 2)
    return out.numpy()


@pytest.mark.parametrize("view", ["diffusion", "verify"])
def test_zero_prefix_is_plain_sdpa(view):
    """L = 0: DIFFUSION is unmasked SDPA, VERIFY is causal SDPA (no explicit mask)."""
    w = small_workload(prefix_len=0, block=6, B=3)
    wi = W.WorkloadInputs(w, seed=3)
    got = oracle.block_attn(*oracle_attn_args(wi, view))
    r = wi.rounds[0]
    for b in range(w.B):
        r0, r1 = int(wi.meta.cu_block[b]), int(wi.meta.cu_block[b + 1])
        q = r.q[view][r0:r1].double().permute(1, 0, 2)
        k = r.k_block[view][r0:r1].double().permute(1, 0, 2)
        v = r.v_block[view][r0:r1].double().permute(1, 0, 2)
        ref = F.scaled_dot_product_attention(q, k, v, is_causal=(view == "verify"),
                                             enable_gqa=True).permute(1, 0, 2).numpy()
        np.testing.assert_allclose(got[r0:r1], ref, rtol=TOL, atol=TOL)


@pytest.mark.parametrize("view", ["diffusion", "verify"])
@pytest.mark.parametrize("L,K,Hq,Hkv,D", [(19, 5, 4, 2, 16), (64, 8, 8, 2, 32), (1, 1, 2, 1, 8),
                                           (130, 32, 4, 1, 16)])
def test_masked_sdpa(view, L, K, Hq, Hkv, D):
    w = small_workload(prefix_len=L, block=K, Hq=Hq, Hkv=Hkv, D=D)
    wi = W.WorkloadInputs(w, seed=L + K)
    got = oracle.block_attn(*oracle_attn_args(wi, view))
    ref = _sdpa_reference(wi, view)
    np.testing.assert_allclose(got, ref, rtol=TOL, atol=TOL)


@pytest.mark.parametrize("view", ["diffusion", "verify"])
def test_ragged_blocks_sdpa(view):
    """Per-sequence prefix and block sizes, including an empty block."""
    w = small_workload(B=4, prefix_range=(0, 40), prefix_len=None, block=None,
                       block_choices=(0, 1, 3, 7))
    wi = W.WorkloadInputs(w, seed=11)
    got = oracle.block_attn(*oracle_attn_args(wi, view))
    ref = _sdpa_reference(wi, view)
    np.testing.assert_allclose(got, ref, rtol=TOL, atol=TOL)


def test_block_bias_mask_sensitivity():
    """Block keys carry a +8 score bias over the prefix, so a wrong in-block mask
    would move outputs by O(1). Both views must match SDPA and differ from each other."""
    w = small_workload(prefix_len=48, block=6, Hq=2, Hkv=1, D=16)
    wi = W.WorkloadInputs(w, seed=5)
    r = wi.rounds[0]
    g = torch.Generator().manual_seed(7)
    u = torch.randn(w.D, generator=g, dtype=torch.float64)
    u = u / u.norm() * 4.0                       # |q| = 4, scale 1/4
    for view in W.VIEW_NAMES:
        r.q[view][:] = u.to(torch.bfloat16)
        r.k_block[view][:] = (2.0 * u).to(torch.bfloat16)   # score 0.25 * 4 * 8 = 8
        r.v_block[view].copy_(r.v_block["diffusion"])
    outs = {}
    for view in W.VIEW_NAMES:
        got = oracle.block_attn(*oracle_attn_args(wi, view))
        np.testing.assert_allclose(got, _sdpa_reference(wi, view), rtol=TOL, atol=TOL)
        outs[view] = got
    assert np.abs(outs["diffusion"] - outs["verify"]).max() > 0.1


@pytest.mark.parametrize("L,K", [(37, 6), (0, 4), (128, 32)])
def test_verify_row_is_single_query_decode(L, K):
    """AR equivalence: VERIFY row i == decode of one query over prefix + block[0..i]."""
    w = small_workload(prefix_len=L, block=K, Hq=4, Hkv=2, D=16, B=2)
    wi = W.WorkloadInputs(w, seed=17)
    got = oracle.block_attn(*oracle_attn_args(wi, "verify"))
    r = wi.rounds[0]

    def decode(q, keys, vals):
        # one query attending over every key it is given (an AR decode step)
        return F.scaled_dot_product_attention(q[None, None], keys[None], vals[None])[0, 0]

    for b in range(w.B):
        kp, vp = _contiguous_kv(wi, b)
        r0 = int(wi.meta.cu_block[b])
        for i in range(K):
            for hq in range(w.Hq):
                h = hq // w.G
                keys = torch.cat([kp[h], r.k_block["verify"][r0:r0 + i + 1, h].double()])
                vals = torch.cat([vp[h], r.v_block["verify"][r0:r0 + i + 1, h].double()])
                ref = decode(r.q["verify"][r0 + i, hq].double(), keys, vals).numpy()
                np.testing.assert_allclose(got[r0 + i, hq], ref, rtol=TOL, atol=TOL)


@pytest.mark.parametrize("view", ["diffusion", "verify"])
def test_zero_query_gives_mean_of_visible_values(view):
    w = small_workload(prefix_len=23, block=5, B=2)
    wi = W.WorkloadInputs(w, seed=2)
    r = wi.rounds[0]
    r.q[view].zero_()
    got = oracle.block_attn(*oracle_attn_args(wi, view))
    for b in range(w.B):
        _, vp = _contiguous_kv(wi, b)
        r0 = int(wi.meta.cu_block[b])
        for i in range(w.block):
            n_blk = w.block if view == "diffusion" else i + 1
            for hq in range(w.Hq):
                h = hq // w.G
                vals = torch.cat([vp[h], r.v_block[view][r0:r0 + n_blk, h].double()])
                np.testing.assert_allclose(got[r0 + i, hq], vals.mean(0).numpy(),
                                           rtol=TOL, atol=TOL)


@pytest.mark.parametrize("view,key_pos", [("diffusion", 3), ("diffusion", 20), ("verify", 21),
                                          ("verify", 10)])
def test_dominant_key_selects_its_value(view, key_pos):
    """A key whose score exceeds every other by >= 60 returns its value row."""
    L, K, D = 19, 5, 16
    w = small_workload(prefix_len=L, block=K, Hq=1, Hkv=1, D=D, B=1)
    wi = W.WorkloadInputs(w, seed=9)
    r = wi.rounds[0]
    r.q[view].zero_()
    r.q[view][..., 0] = 8.0
    wi.k_cache[..., 0] = 0.0
    r.k_block[view][..., 0] = 0.0
    # scale 1/4: score of the chosen key = 8 * 32 / 4 = 64, all others 0
    if key_pos < L:
        page, slot = divmod(key_pos, w.page_size)
        wi.k_cache[page, 0, slot, 0] = 32.0
        v_star = wi.v_cache[page, 0, slot].double().numpy()
    else:
        j = key_pos - L
        r.k_block[view][j, 0, 0] = 32.0
        v_star = r.v_block[view][j, 0].double().numpy()
    got = oracle.block_attn(*oracle_attn_args(wi, view))
    for i in range(K):
        sees = key_pos < L or view == "diffusion" or (key_pos - L) <= i
        if sees:
            np.testing.assert_allclose(got[i, 0], v_star, rtol=0, atol=1e-20)


def test_page_permutation_invariance():
    """Shuffling physical pages (and the table with them) leaves the output unchanged."""
    w = small_workload(prefix_len=45, block=7, B=3, page_size=8)
    wi = W.WorkloadInputs(w, seed=21)
    base = {v: oracle.block_attn(*oracle_attn_args(wi, v)) for v in W.VIEW_NAMES}
    g = torch.Generator().manual_seed(99)
    perm = torch.randperm(wi.meta.num_pages, generator=g)
    kc = torch.empty_like(wi.k_cache)
    vc = torch.empty_like(wi.v_cache)
    kc[perm] = wi.k_cache
    vc[perm] = wi.v_cache
    table = wi.meta.page_table.clone()
    valid = table >= 0
    table[valid] = perm[table[valid].long()].to(torch.int32)
    for v in W.VIEW_NAMES:
        args = list(oracle_attn_args(wi, v, k_cache=kc, v_cache=vc))
        args[8] = table.numpy()
        np.testing.assert_array_equal(oracle.block_attn(*args), base[v])


@pytest.mark.parametrize("view", ["diffusion", "verify"])
@pytest.mark.parametrize("chunk", [1, 8, 13, 64, 2048, 100000])
def test_split_chunks_equal_unsplit(view, chunk):
    w = small_workload(B=3, prefix_len=None, prefix_range=(0, 150), block=None,
                       block_choices=(1, 4, 9))
    wi = W.WorkloadInputs(w, seed=31)
    args = oracle_attn_args(wi, view)
    ref = oracle.block_attn(*args)
    got = oracle.block_attn_split(*args, chunk_tokens=chunk)
    np.testing.assert_allclose(got, ref, rtol=TOL, atol=TOL)


def test_selection_matches_full():
    w = small_workload(prefix_len=33, block=6, B=2)
    wi = W.WorkloadInputs(w, seed=4)
    args = oracle_attn_args(wi, "verify")
    full = oracle.block_attn(*args)
    rows = np.array([0, 5, 7, 11], np.int64)
    heads = np.array([3, 0, 2, 1], np.int32)
    sel = oracle.block_attn(*args, sel=(rows, heads))
    np.testing.assert_array_equal(sel, full[rows, heads])


# ---------------------------------------------------------------------------
# Brute force in the pages' form: a full-sequence mask matrix, pure Python.

def _bf_attention(qs, ks, vs, L, K, view):
    """qs: K query rows; ks/vs: L+K rows (prefix then block). Pure Python, math.exp,
    summing in reverse order. The mask is built as a full (L+K) x (L+K) matrix over
    the whole sequence and the block rows are read off its last K rows."""
    n = L + K
    allowed = [[False] * n for _ in range(n)]
    for a in range(n):
        for c in range(n):
            if view == "verify":
                allowed[a][c] = c <= a                       # ordinary causal
            else:
                if a < L:
                    allowed[a][c] = c <= a                   # clean context, causal
                else:
                    allowed[a][c] = (c < L) or (L <= c < n)  # M_diff: context + whole block
    scale = 1.0 / math.sqrt(len(qs[0]))
    outs = []
    for i in range(K):
        a = L + i
        vis = [c for c in range(n) if allowed[a][c]]
        scores = [scale * sum(x * y for x, y in zip(qs[i], ks[c])) for c in vis]
        top = max(scores)
        wts = [math.exp(s - top) for s in scores]
        tot = 0.0
        for x in reversed(wts):
            tot += x
        o = []
        for d in range(len(vs[0])):
            acc = 0.0
            for idx in reversed(range(len(vis))):
                acc += wts[idx] * vs[vis[idx]][d]
            o.append(acc / tot)
        outs.append(o)
    return outs


def _run_oracle_tiny(qs, ks, vs, L, K, D, view):
    """Pack one (b=0, head=0) problem into oracle arrays with a 1-token page size."""
    to_bits = lambda x: W.bf16_bits(torch.tensor(x, dtype=torch.float64).to(torch.bfloat16))
    q = to_bits(qs).reshape(K, 1, D)
    n_pages = max(L, 1)
    kc = np.zeros((n_pages, 1, 1, D), np.uint16)
    vc = np.zeros((n_pages, 1, 1, D), np.uint16)
    if L:
        kc[:L, 0, 0] = to_bits(ks[:L])
        vc[:L, 0, 0] = to_bits(vs[:L])
    kb = to_bits(ks[L:]).reshape(K, 1, D)
    vb = to_bits(vs[L:]).reshape(K, 1, D)
    table = np.arange(n_pages, dtype=np.int32).reshape(1, -1)
    out = oracle.block_attn(VIEW_ID[view], q, kc, vc, kb, vb, np.array([L], np.int32),
                            np.array([0, K], np.int32), table, threads=1)
    return out[:, 0, :]


@pytest.mark.parametrize("view", ["diffusion", "verify"])
def test_brute_force_exhaustive_tiny(view):
    """Every input with L in {0,1}, K in {1,2}, D=1 and entries in {-1,0,1}."""
    vals = (-1.0, 0.0, 1.0)
    count = 0
    for L, K in [(0, 1), (0, 2), (1, 1), (1, 2)]:
        n_entries = K + 2 * (L + K)
        for combo in itertools.product(vals, repeat=n_entries):
            qs = [[combo[i]] for i in range(K)]
            ks = [[combo[K + j]] for j in range(L + K)]
            vs = [[combo[K + L + K + j]] for j in range(L + K)]
            ref = _bf_attention(qs, ks, vs, L, K, view)
            got = _run_oracle_tiny(qs, ks, vs, L, K, 1, view)
            np.testing.assert_allclose(got, np.array(ref), rtol=TOL, atol=TOL)
            count += 1
    assert count == 3 ** 3 + 3 ** 6 + 3 ** 5 + 3 ** 8


@pytest.mark.parametrize("view", ["diffusion", "verify"])
def test_brute_force_sampled_small(view):
    """Random inputs with L <= 3, K <= 3, D = 2, entries in {-1, 0, 1}."""
    rng = random.Random(1234)
    vals = (-1.0, 0.0, 1.0)
    for _ in range(400):
        L, K, D = rng.randint(0, 3), rng.randint(1, 3), 2
        qs = [[rng.choice(vals) for _ in range(D)] for _ in range(K)]
        ks = [[rng.choice(vals) for _ in range(D)] for _ in range(L + K)]
        vs = [[rng.choice(vals) for _ in range(D)] for _ in range(L + K)]
        ref = _bf_attention(qs, ks, vs, L, K, view)
        got = _run_oracle_tiny(qs, ks, vs, L, K, D, view)
        np.testing.assert_allclose(got, np.array(ref), rtol=TOL, atol=TOL)
