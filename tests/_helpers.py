"""Shared test plumbing: turn seeded workload tensors into oracle arguments."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from diffusion_draft_ar_b200 import workloads as W

VIEW_ID = {"diffusion": oracle.VIEW_DIFFUSION, "verify": oracle.VIEW_VERIFY}


def np_i32(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").numpy().astype(np.int32)


def oracle_attn_args(wi: W.WorkloadInputs, view: str, round_idx: int = 0,
                     prefix_lens=None, k_cache=None, v_cache=None):
    """Positional oracle arguments (bf16 as uint16 bits) for one view of one round."""
    r = wi.rounds[round_idx]
    m = wi.meta
    return (
        VIEW_ID[view],
        W.bf16_bits(r.q[view]),
        W.bf16_bits(wi.k_cache if k_cache is None else k_cache),
        W.bf16_bits(wi.v_cache if v_cache is None else v_cache),
        W.bf16_bits(r.k_block[view]),
        W.bf16_bits(r.v_block[view]),
        np_i32(m.prefix_lens if prefix_lens is None else prefix_lens),
        np_i32(m.cu_block),
        np_i32(m.page_table),
    )


def rel_rms(a: np.ndarray, b: np.ndarray) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.sqrt(np.sum(b * b))
    return float(np.sqrt(np.sum((a - b) ** 2)) / (den if den > 0 else 1.0))


def small_workload(**kw) -> W.Workload:
    base = dict(name="small", B=2, Hq=4, Hkv=2, D=16, page_size=8, prefix_len=19, block=5,
                paged=False, vocab=None, headroom=8)
    base.update(kw)
    return W.Workload(**base)
