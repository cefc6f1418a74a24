"""Seeded synthetic inputs for the Orthrus block-decoding path.

This module is shared by the CUDA path's tests/bench and by the oracle's tests.
It holds none of the method's arithmetic: it only draws random numbers, builds
page tables and row offsets, and applies the draft rule "take the given target
token with probability p, else a uniform token" to targets the caller supplies.

Workloads (Qwen3 head shapes; vocabulary 151,936 as the Qwen3 stand-in). The
pages evaluate on GSM8K / MATH-500 / AIME / HumanEval / MBPP with trained
Qwen3 weights; none of that is used here, so every tensor is synthetic:

* ``tiny``       B=1, L=256, K=8, 4/1 heads, D=64, contiguous cache, V=512 N(0,1), p=0.7
* ``qwen3_1p7b`` B=1, L=4096, K=32, 16/8 heads, D=128, contiguous, V=151936 N(0, std 2), p=0.8
* ``qwen3_8b``   B=16, L=8192, K=32, 32/8 heads, D=128, 64-token pages in a random
                 permutation, V=151936 N(0,1), p=0.8, plus a KV append
* ``longctx``    B=1, L=131072, K=32, 32/8 heads, D=128, random pages, VERIFY only,
                 split over 2048-token chunks
* ``ragged``     B=64, L_b ~ U{512..32768}, K_b ~ U{8,16,32}, 32/8 heads, D=128,
                 random pages, 8 rounds, V=151936 N(0,1), p_b ~ U[0.5, 0.95]

Draw order (one CPU generator for metadata, one generator on ``device`` for the
bulk tensors, both seeded from ``seed``):
  metadata: prefix lengths, block sizes, match probabilities, page permutation;
  bulk: k_cache, v_cache, then per round: for each view (DIFFUSION, VERIFY)
  q_block, k_block, v_block; then logits, draft coins, alternative drafts.
bf16 tensors are fp32 N(0,1) draws (times std) rounded to bf16 (RNE).
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import torch

VOCAB_QWEN3 = 151936
VIEW_NAMES = ("diffusion", "verify")


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    page_size: int = 64
    prefix_len: int | None = None            # fixed prefix length L
    prefix_range: tuple[int, int] | None = None  # inclusive range of L_b (ragged)
    block: int | None = None                 # fixed block size K
    block_choices: tuple[int, ...] | None = None  # per-sequence K_b choices (ragged)
    paged: bool = False                      # random page permutation vs identity table
    views: tuple[str, ...] = VIEW_NAMES
    vocab: int | None = None                 # None: no consensus step in this workload
    logit_std: float = 1.0
    p_match: float | None = None             # fixed draft-match probability
    p_range: tuple[float, float] | None = None  # per-sequence U[lo, hi] (ragged)
    rounds: int = 1
    headroom: int = 0                        # append slots reserved per sequence
    kv_split_tokens: int = 0                 # 0: library-chosen split
    d_model: int | None = None               # hidden size feeding the LM head (Qwen3 config)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def max_block(self) -> int:
        return self.block if self.block is not None else max(self.block_choices)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: dict[str, Workload] = {
    "tiny": Workload("tiny", B=1, Hq=4, Hkv=1, D=64, prefix_len=256, block=8, paged=False,
                     vocab=512, logit_std=1.0, p_match=0.7, headroom=8),
    "qwen3_1p7b": Workload("qwen3_1p7b", B=1, Hq=16, Hkv=8, D=128, prefix_len=4096, block=32,
                           paged=False, vocab=VOCAB_QWEN3, logit_std=2.0, p_match=0.8,
                           headroom=32, d_model=2048),
    "qwen3_8b": Workload("qwen3_8b", B=16, Hq=32, Hkv=8, D=128, prefix_len=8192, block=32,
                         paged=True, vocab=VOCAB_QWEN3, logit_std=1.0, p_match=0.8,
                         headroom=32, d_model=4096),
    "longctx": Workload("longctx", B=1, Hq=32, Hkv=8, D=128, prefix_len=131072, block=32,
                        paged=True, views=("verify",), vocab=None, headroom=32,
                        kv_split_tokens=2048),
    "ragged": Workload("ragged", B=64, Hq=32, Hkv=8, D=128, prefix_range=(512, 32768),
                       block_choices=(8, 16, 32), paged=True, vocab=VOCAB_QWEN3,
                       logit_std=1.0, p_range=(0.5, 0.95), rounds=8, headroom=8 * 32),
}


@dataclass
class BatchMeta:
    """Per-sequence metadata (int32 CPU tensors unless noted)."""
    prefix_lens: torch.Tensor   # [B]
    block_lens: torch.Tensor    # [B]
    cu_block: torch.Tensor      # [B+1] row offsets of each sequence's block rows
    page_table: torch.Tensor    # [B, max_pages]; unused entries are -1
    num_pages: int
    p_match: torch.Tensor       # [B] float64
    pages_per_seq: torch.Tensor  # [B] pages reserved for prefix + headroom

    @property
    def R(self) -> int:
        return int(self.cu_block[-1])

    @property
    def B(self) -> int:
        return int(self.prefix_lens.shape[0])

    @property
    def max_pages(self) -> int:
        return int(self.page_table.shape[1])


def make_meta(w: Workload, seed: int = 0) -> BatchMeta:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    B = w.B
    if w.prefix_len is not None:
        L = torch.full((B,), w.prefix_len, dtype=torch.int64)
    else:
        lo, hi = w.prefix_range
        L = torch.randint(lo, hi + 1, (B,), generator=g, dtype=torch.int64)
    if w.block is not None:
        K = torch.full((B,), w.block, dtype=torch.int64)
    else:
        choices = torch.tensor(w.block_choices, dtype=torch.int64)
        K = choices[torch.randint(0, len(w.block_choices), (B,), generator=g)]
    if w.p_match is not None:
        p = torch.full((B,), float(w.p_match), dtype=torch.float64)
    elif w.p_range is not None:
        lo, hi = w.p_range
        p = lo + (hi - lo) * torch.rand((B,), generator=g, dtype=torch.float64)
    else:
        p = torch.zeros((B,), dtype=torch.float64)
    P = w.page_size
    pages = (L + w.headroom + P - 1) // P
    num_pages = int(pages.sum())
    max_pages = int(pages.max())
    if w.paged:
        phys = torch.randperm(num_pages, generator=g, dtype=torch.int64)
    else:
        phys = torch.arange(num_pages, dtype=torch.int64)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    off = 0
    for b in range(B):
        n = int(pages[b])
        table[b, :n] = phys[off:off + n].to(torch.int32)
        off += n
    cu = torch.zeros(B + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(K, 0).to(torch.int32)
    return BatchMeta(prefix_lens=L.to(torch.int32), block_lens=K.to(torch.int32), cu_block=cu,
                     page_table=table, num_pages=num_pages, p_match=p,
                     pages_per_seq=pages.to(torch.int32))


def randn_bf16(shape, gen: torch.Generator, device, std: float = 1.0,
               chunk: int = 1 << 26) -> torch.Tensor:
    """bf16 tensor of N(0, std^2) draws, generated in fp32 chunks and rounded (RNE)."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        x = torch.randn(e - s, generator=gen, dtype=torch.float32, device=device)
        if std != 1.0:
            x.mul_(std)
        flat[s:e].copy_(x)
    return out


def randn_f32(shape, gen: torch.Generator, device, std: float = 1.0) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, dtype=torch.float32, device=device)
    if std != 1.0:
        x.mul_(std)
    return x


@dataclass
class RoundInputs:
    """Per-round tensors on the workload's device."""
    q: dict            # view name -> [R, Hq, D] bf16
    k_block: dict      # view name -> [R, Hkv, D] bf16
    v_block: dict      # view name -> [R, Hkv, D] bf16
    logits: torch.Tensor | None = None   # [R, V] fp32
    coins: torch.Tensor | None = None    # [R] fp32 in [0, 1)
    alt: torch.Tensor | None = None      # [R] int32 uniform in [0, V)


class WorkloadInputs:
    """All seeded tensors of one workload, drawn in the documented order."""

    def __init__(self, w: Workload, device="cpu", seed: int = 0, rounds: int | None = None,
                 with_cache: bool = True):
        self.w = w
        self.device = torch.device(device)
        self.seed = seed
        self.meta = make_meta(w, seed)
        g = torch.Generator(device=self.device)
        g.manual_seed(seed + 1)
        self.gen = g
        m = self.meta
        shape = (m.num_pages, w.Hkv, w.page_size, w.D)
        if with_cache:
            self.k_cache = randn_bf16(shape, g, self.device)
            self.v_cache = randn_bf16(shape, g, self.device)
        else:
            self.k_cache = self.v_cache = None
        n_rounds = w.rounds if rounds is None else rounds
        self.rounds = [self._draw_round() for _ in range(n_rounds)]

    def _draw_round(self) -> RoundInputs:
        w, m, g, dev = self.w, self.meta, self.gen, self.device
        R = m.R
        q, kb, vb = {}, {}, {}
        for view in VIEW_NAMES:
            if view not in w.views:
                continue
            q[view] = randn_bf16((R, w.Hq, w.D), g, dev)
            kb[view] = randn_bf16((R, w.Hkv, w.D), g, dev)
            vb[view] = randn_bf16((R, w.Hkv, w.D), g, dev)
        ri = RoundInputs(q=q, k_block=kb, v_block=vb)
        if w.vocab is not None:
            ri.logits = randn_f32((R, w.vocab), g, dev, std=w.logit_std)
            ri.coins = torch.rand((R,), generator=g, dtype=torch.float32, device=dev)
            ri.alt = torch.randint(0, w.vocab, (R,), generator=g, dtype=torch.int64,
                                   device=dev).to(torch.int32)
        return ri

    def row_p_match(self) -> torch.Tensor:
        """Per-row draft-match probability (the owning sequence's p_b)."""
        m = self.meta
        return torch.repeat_interleave(m.p_match, m.block_lens.to(torch.int64))

    def drafts(self, round_idx: int, targets: torch.Tensor) -> torch.Tensor:
        """Draft tokens for a round: ``targets[r]`` with probability p, else ``alt[r]``.

        ``targets`` are the rows' greedy tokens, supplied by the caller (the
        oracle in tests, the device argmax of the logits in the bench).
        """
        ri = self.rounds[round_idx]
        p = self.row_p_match().to(device=ri.coins.device, dtype=torch.float32)
        return drafts_from_targets(targets.to(ri.coins.device), ri.coins, ri.alt, p)


def drafts_from_targets(targets: torch.Tensor, coins: torch.Tensor, alt: torch.Tensor,
                        p: torch.Tensor | float) -> torch.Tensor:
    """Select ``targets`` where ``coins < p`` and ``alt`` elsewhere (int32)."""
    take = coins < p
    return torch.where(take, targets.to(torch.int32), alt.to(torch.int32)).to(torch.int32)


def cache_bytes_per_token(w: Workload) -> int:
    """K and V bytes of one prefix token for all KV heads (bf16)."""
    return 2 * w.Hkv * w.D * 2


def bf16_bits(t: torch.Tensor):
    """Raw 16-bit patterns of a bf16 tensor as a numpy uint16 array (CPU)."""
    import numpy as np
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def sentinel_fill_(t: torch.Tensor, bits: int = 0x7FBF) -> torch.Tensor:
    """Fill a bf16 tensor with a NaN bit pattern (marks never-written slots)."""
    t.view(torch.int16).fill_(bits if bits < 0x8000 else bits - 0x10000)
    return t


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


__all__ = [
    "lm_head_inputs", "Workload", "WORKLOADS", "BatchMeta", "make_meta", "WorkloadInputs", "RoundInputs",
    "drafts_from_targets", "randn_bf16", "randn_f32", "cache_bytes_per_token",
    "bf16_bits", "sentinel_fill_", "ceil_div", "VIEW_NAMES", "VOCAB_QWEN3",
]


def lm_head_inputs(R: int, d_model: int, V: int, device, seed: int = 0):
    """Seeded synthetic LM-head operands: final hidden states N(0, 1) [R, d] and an
    output projection N(0, 1/d) [V, d] (so each score is about N(0, 1)), both
    bf16, drawn on ``device``. Random weights of the shape only: no checkpoint."""
    g = torch.Generator(device=device)
    g.manual_seed(seed + 7)
    hidden = randn_bf16((R, d_model), g, device)
    w = randn_bf16((V, d_model), g, device, std=d_model ** -0.5)
    return hidden, w
