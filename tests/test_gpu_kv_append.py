"""KV append on the GPU against the oracle: bit-exact caches and lengths."""
import numpy as np
import pytest
import torch

import oracle
from diffusion_draft_ar_b200 import workloads as W
from tests._gpu import gpu, lib, needs_cuda
from tests._helpers import np_i32, small_workload

pytestmark = [gpu, needs_cuda]


def _both(wi, accept, update=True, table=None, lens=None):
    """Run the GPU append and the oracle append from the same state; compare."""
    O = lib()
    m = wi.meta
    table = m.page_table if table is None else table
    lens = m.prefix_lens.clone() if lens is None else lens.clone()
    r = wi.rounds[0]
    kb, vb = r.k_block["verify"], r.v_block["verify"]
    # oracle
    kc_o = W.bf16_bits(wi.k_cache).copy()
    vc_o = W.bf16_bits(wi.v_cache).copy()
    lens_o = np_i32(lens).copy()
    rc = oracle.kv_append(W.bf16_bits(kb), W.bf16_bits(vb), np_i32(m.cu_block),
                          np.asarray(accept, np.int32), lens_o, np_i32(table), kc_o, vc_o,
                          update_lens=update)
    # gpu
    kc = wi.k_cache.cuda()
    vc = wi.v_cache.cuda()
    lens_d = lens.cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O.kv_append(kb.cuda(), vb.cuda(), m.cu_block.cuda(), wi.w.max_block,
                torch.as_tensor(np.asarray(accept, np.int32)).cuda(), lens_d, table.cuda(), kc, vc,
                update_lens=update, error_flag=err)
    torch.cuda.synchronize()
    assert np.array_equal(W.bf16_bits(kc), kc_o)
    assert np.array_equal(W.bf16_bits(vc), vc_o)
    np.testing.assert_array_equal(lens_d.cpu().numpy(), lens_o)
    return rc, int(err.item())


def _sentinel_workload(seed, **kw):
    base = dict(name="append", B=5, Hq=8, Hkv=4, D=128, page_size=64, prefix_len=None,
                prefix_range=(0, 300), block=None, block_choices=(1, 7, 32), paged=True,
                headroom=64)
    base.update(kw)
    wi = W.WorkloadInputs(small_workload(**base), seed=seed)
    m = wi.meta
    for b in range(m.B):
        L = int(m.prefix_lens[b])
        for pidx in range(int(m.pages_per_seq[b])):
            lo = max(0, L - base["page_size"] * pidx)
            if lo < base["page_size"]:
                page = int(m.page_table[b, pidx])
                W.sentinel_fill_(wi.k_cache[page, :, lo:])
                W.sentinel_fill_(wi.v_cache[page, :, lo:])
    return wi


@pytest.mark.parametrize("update", [True, False])
def test_random_accepts(update):
    wi = _sentinel_workload(1)
    g = np.random.default_rng(1)
    acc = [int(g.integers(0, k + 1)) for k in wi.meta.block_lens.tolist()]
    rc, err = _both(wi, acc, update)
    assert rc == 0 and err == 0


def test_full_and_zero_accepts_and_page_straddle():
    wi = _sentinel_workload(2, prefix_range=(60, 62), block_choices=(32,))
    acc = [32, 0, 5, 1, 32]
    rc, err = _both(wi, acc)
    assert rc == 0 and err == 0


@pytest.mark.parametrize("D,Hkv,P", [(64, 1, 64), (128, 8, 128), (64, 2, 256)])
def test_shapes(D, Hkv, P):
    wi = _sentinel_workload(3, D=D, Hkv=Hkv, Hq=Hkv, page_size=P)
    acc = wi.meta.block_lens.tolist()
    rc, err = _both(wi, acc)
    assert rc == 0 and err == 0


def test_bad_page_and_bad_length_flagged_like_oracle():
    wi = _sentinel_workload(4, headroom=0, prefix_range=(64, 64))
    acc = [1, 0, 1, 0, 0]  # sequences 0 and 2 need a page the table does not hold
    rc, err = _both(wi, acc)
    assert rc != 0 and err & lib().FLAG_BAD_LENGTH
    wi = _sentinel_workload(5)
    table = wi.meta.page_table.clone()
    L0 = int(wi.meta.prefix_lens[0])
    table[0, L0 // 64] = 10 ** 7
    acc = [1, 1, 1, 1, 1]
    rc, err = _both(wi, acc, table=table)
    assert rc != 0 and err & lib().FLAG_BAD_PAGE


def test_accept_beyond_block_is_rejected():
    wi = _sentinel_workload(6)
    acc = [int(k) + 1 for k in wi.meta.block_lens.tolist()]
    rc, err = _both(wi, acc)
    assert rc != 0 and err & lib().FLAG_BAD_LENGTH


def test_qwen3_8b_append():
    """The Qwen3-8B-shaped workload's append (16 sequences, random pages)."""
    wi = W.WorkloadInputs(W.WORKLOADS["qwen3_8b"], seed=0)
    g = np.random.default_rng(7)
    acc = g.integers(1, 33, 16).tolist()
    rc, err = _both(wi, acc)
    assert rc == 0 and err == 0
