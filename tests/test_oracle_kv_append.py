"""Pins for the oracle's KV append (Orthrus technical summary §2.3 item 3, commit
and truncate the cache; agents-report.net commentary, "core design": the accepted
tokens' KV state is appended to the shared cache).

After appending n_b rows at position L_b, reading the first L_b + n_b tokens of
each sequence through its page table must give the old prefix followed by the
accepted block rows, and every other byte of the cache must be unchanged."""
import numpy as np
import pytest
import torch

import oracle
from diffusion_draft_ar_b200 import workloads as W
from tests._helpers import np_i32, small_workload

SENTINEL = np.uint16(0x7FBF)


def _read_tokens(cache: np.ndarray, table_row: np.ndarray, n_tokens: int, P: int) -> np.ndarray:
    """Tokens 0..n_tokens-1 of one sequence: [n_tokens, Hkv, D], pages laid end to end."""
    n_pages = -(-n_tokens // P)
    pages = cache[table_row[:n_pages]]                  # [n_pages, Hkv, P, D]
    seq = np.concatenate(list(pages.transpose(0, 2, 1, 3)), axis=0)  # [n_pages*P, Hkv, D]
    return seq[:n_tokens]


def _setup(w, seed, accept):
    wi = W.WorkloadInputs(w, seed=seed)
    kc = W.bf16_bits(wi.k_cache).copy()
    vc = W.bf16_bits(wi.v_cache).copy()
    m = wi.meta
    P = w.page_size
    # mark every slot at or beyond each sequence's prefix with the sentinel
    for b in range(m.B):
        L = int(m.prefix_lens[b])
        for pidx in range(int(m.pages_per_seq[b])):
            page = int(m.page_table[b, pidx])
            lo = max(0, L - pidx * P)
            if lo < P:
                kc[page, :, lo:, :] = SENTINEL
                vc[page, :, lo:, :] = SENTINEL
    r = wi.rounds[0]
    kb = W.bf16_bits(r.k_block["verify"])
    vb = W.bf16_bits(r.v_block["verify"])
    return wi, kc, vc, kb, vb, np.array(accept, np.int32)


@pytest.mark.parametrize("update", [True, False])
def test_append_layout_and_sentinels(update):
    w = small_workload(B=3, prefix_len=None, prefix_range=(5, 30), block=None,
                       block_choices=(4, 6), page_size=8, headroom=12)
    wi, kc, vc, kb, vb, acc = _setup(w, 7, [0, 0, 0])
    m = wi.meta
    acc = np.minimum(np.array([3, 1, 6]), np_i32(m.block_lens)).astype(np.int32)
    kc0, vc0 = kc.copy(), vc.copy()
    lens = np_i32(m.prefix_lens).copy()
    rc = oracle.kv_append(kb, vb, np_i32(m.cu_block), acc, lens, np_i32(m.page_table), kc, vc,
                          update_lens=update)
    assert rc == 0
    L0 = np_i32(m.prefix_lens)
    np.testing.assert_array_equal(lens, L0 + acc if update else L0)
    table = np_i32(m.page_table)
    touched = np.zeros(kc.shape[:1] + kc.shape[2:3], bool)  # [page, slot]
    for b in range(m.B):
        L, n, r0 = int(L0[b]), int(acc[b]), int(m.cu_block[b])
        for cache, old, blk in ((kc, kc0, kb), (vc, vc0, vb)):
            got = _read_tokens(cache, table[b], L + n, w.page_size)
            want = np.concatenate([_read_tokens(old, table[b], L, w.page_size), blk[r0:r0 + n]])
            np.testing.assert_array_equal(got, want)
        for i in range(n):
            pg, sl = divmod(L + i, w.page_size)
            touched[table[b, pg], sl] = True
    # every untouched (page, slot) is byte-identical, sentinels included
    for cache, old in ((kc, kc0), (vc, vc0)):
        diff = (cache != old).any(axis=(1, 3))  # [page, slot]
        assert not (diff & ~touched).any()


def test_append_straddles_page_boundary():
    w = small_workload(B=1, prefix_len=62, block=8, page_size=64, headroom=8, paged=True,
                       Hq=2, Hkv=2, D=16)
    wi, kc, vc, kb, vb, acc = _setup(w, 1, [5])
    m = wi.meta
    lens = np_i32(m.prefix_lens).copy()
    table = np_i32(m.page_table)
    assert oracle.kv_append(kb, vb, np_i32(m.cu_block), acc, lens, table, kc, vc) == 0
    assert lens[0] == 67
    # positions 62, 63 in page table[0][0]; 64, 65, 66 in table[0][1]
    np.testing.assert_array_equal(kc[table[0, 0], :, 62], kb[0])
    np.testing.assert_array_equal(kc[table[0, 0], :, 63], kb[1])
    np.testing.assert_array_equal(kc[table[0, 1], :, 0], kb[2])
    np.testing.assert_array_equal(vc[table[0, 1], :, 2], vb[4])
    assert (kc[table[0, 1], :, 3:] == SENTINEL).all()


def test_append_nothing_and_bad_page():
    w = small_workload(B=2, prefix_len=8, block=4, page_size=8, headroom=0)
    wi, kc, vc, kb, vb, acc = _setup(w, 2, [0, 0])
    m = wi.meta
    kc0 = kc.copy()
    lens = np_i32(m.prefix_lens).copy()
    assert oracle.kv_append(kb, vb, np_i32(m.cu_block), acc, lens, np_i32(m.page_table),
                            kc, vc) == 0
    np.testing.assert_array_equal(kc, kc0)
    # no headroom: appending one row needs a page the table does not hold
    acc = np.array([1, 0], np.int32)
    assert oracle.kv_append(kb, vb, np_i32(m.cu_block), acc, lens, np_i32(m.page_table),
                            kc, vc) != 0
    np.testing.assert_array_equal(kc, kc0)


def test_bad_append_leaves_length():
    w = small_workload(B=2, prefix_len=8, block=4, page_size=8, headroom=0)
    wi, kc, vc, kb, vb, _ = _setup(w, 2, [0, 0])
    m = wi.meta
    lens = np_i32(m.prefix_lens).copy()
    acc = np.array([2, 0], np.int32)
    assert oracle.kv_append(kb, vb, np_i32(m.cu_block), acc, lens, np_i32(m.page_table),
                            kc, vc, update_lens=True) != 0
    np.testing.assert_array_equal(lens, np_i32(m.prefix_lens))
