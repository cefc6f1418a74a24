"""GPU-test plumbing: move seeded inputs to the device, call the C ABI through the
binding, and compare with the oracle."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from diffusion_draft_ar_b200 import build as _build
from diffusion_draft_ar_b200 import workloads as W

ATOL = 2e-2     # max |err| against the fp64 oracle
RTOL_RMS = 1e-2  # relative RMS over the compared outputs

gpu = pytest.mark.gpu
needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="no CUDA device")


def lib():
    _build.build()
    from diffusion_draft_ar_b200 import orthrus
    return orthrus


class DevAttn:
    """Device copies of one workload's attention inputs."""

    def __init__(self, wi: W.WorkloadInputs, dev="cuda"):
        m = wi.meta
        self.wi = wi
        self.k_cache = wi.k_cache.to(dev)
        self.v_cache = wi.v_cache.to(dev)
        self.prefix_lens = m.prefix_lens.to(dev)
        self.cu_block = m.cu_block.to(dev)
        self.page_table = m.page_table.to(dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)

    def run(self, view: str, round_idx: int = 0, max_ctas: int = 0, kv_split: int = 0,
            cu_block="default", q=None, kb=None, vb=None, ws_extra: int = 0):
        O = lib()
        r = self.wi.rounds[round_idx]
        w = self.wi.w
        q = (r.q[view] if q is None else q).to("cuda")
        kb = (r.k_block[view] if kb is None else kb).to("cuda")
        vb = (r.v_block[view] if vb is None else vb).to("cuda")
        cu = self.cu_block if isinstance(cu_block, str) else cu_block
        out = torch.full_like(q, float("nan"))
        p = O.attn_params(view, q, self.k_cache, self.v_cache, kb, vb, self.prefix_lens, cu,
                          self.page_table, out, w.max_block, kv_split_tokens=kv_split,
                          max_ctas=max_ctas)
        n = O.block_attn_workspace_size(p)
        assert n > 0
        ws = torch.empty(n + ws_extra, dtype=torch.uint8, device="cuda")
        O.block_attn(view, q, self.k_cache, self.v_cache, kb, vb, self.prefix_lens, cu,
                     self.page_table, out, ws, w.max_block, kv_split_tokens=kv_split,
                     max_ctas=max_ctas, error_flag=self.err)
        torch.cuda.synchronize()
        return out


def oracle_args_dev(wi: W.WorkloadInputs, view: str, round_idx: int = 0):
    from tests._helpers import oracle_attn_args
    return oracle_attn_args(wi, view, round_idx)


def assert_attn_close(got_bf16: torch.Tensor, ref: np.ndarray, what: str = ""):
    """Whole-tensor comparison: max |err| and relative RMS over every compared
    output, the worst (row, head) reported."""
    got = got_bf16.detach().to("cpu").double().numpy()
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    den = np.sqrt(np.sum(ref * ref))
    rel = float(np.sqrt(np.sum(err * err)) / (den if den > 0 else 1.0))
    worst = np.unravel_index(int(np.argmax(err)), err.shape)
    print(f"[parity] {what}: {err.size} outputs, max |err| {err.max():.3e} at {worst}, "
          f"relative RMS {rel:.3e}")
    assert err.max() <= ATOL, f"{what}: max |err| {err.max():.3e} at {worst}"
    assert rel <= RTOL_RMS, f"{what}: relative RMS {rel:.3e}"
    return float(err.max()), rel


def sample_pairs(m: W.BatchMeta, Hq: int, n: int, seed: int):
    """(row, head) pairs: first and last row of every sequence plus random ones."""
    g = np.random.default_rng(seed)
    rows, heads = [], []
    cu = m.cu_block.numpy()
    for b in range(m.B):
        if cu[b + 1] > cu[b]:
            for r in (cu[b], cu[b + 1] - 1):
                rows.append(r)
                heads.append(int(g.integers(0, Hq)))
    R = int(cu[-1])
    rows += list(g.integers(0, R, n))
    heads += list(g.integers(0, Hq, n))
    return np.array(rows, np.int64), np.array(heads, np.int32)
