"""End-to-end losslessness of the oracle's round (Orthrus technical summary §2.3:
"this guarantees lossless inference", §3 "strictly lossless generation").

A one-layer, one-head synthetic model with random weights decodes greedily one
token at a time (plain torch fp64, no paging): that is the reference stream.
The Orthrus round built from the oracle -- VERIFY attention over [anchor, drafts],
consensus, append of the committed rows' KV -- must emit exactly the same stream,
whatever the drafts are (here: the true continuation corrupted at random).
This pins the VERIFY mask, the consensus rule, the append positions and the
anchor hand-over together."""
import numpy as np
import pytest
import torch

import oracle
from diffusion_draft_ar_b200 import workloads as W

V, DM, D, P = 64, 16, 16, 8


class TinyModel:
    def __init__(self, seed):
        g = torch.Generator().manual_seed(seed)
        self.E = torch.randn(V, DM, generator=g, dtype=torch.float64)
        self.Pe = 0.5 * torch.randn(512, DM, generator=g, dtype=torch.float64)
        self.Wq = torch.randn(DM, D, generator=g, dtype=torch.float64) / 2
        self.Wk = torch.randn(DM, D, generator=g, dtype=torch.float64) / 2
        self.Wv = torch.randn(DM, D, generator=g, dtype=torch.float64)
        self.Wo = torch.randn(D, V, generator=g, dtype=torch.float64)

    def qkv(self, tok, pos):
        x = self.E[tok] + self.Pe[pos]
        bf = lambda y: y.to(torch.bfloat16)
        return bf(x @ self.Wq), bf(x @ self.Wk), bf(x @ self.Wv)

    def logits(self, o):
        return (torch.as_tensor(o, dtype=torch.float64) @ self.Wo).to(torch.float32)


def sequential_greedy(model, prompt, n_new):
    ks, vs = [], []
    for p, tok in enumerate(prompt[:-1]):
        _, k, v = model.qkv(tok, p)
        ks.append(k)
        vs.append(v)
    anchor, pos, out = prompt[-1], len(prompt) - 1, []
    while len(out) < n_new:
        q, k, v = model.qkv(anchor, pos)
        ks.append(k)
        vs.append(v)
        keys = torch.stack(ks).double()
        vals = torch.stack(vs).double()
        w = torch.softmax((keys @ q.double()) / D ** 0.5, dim=0)
        t = int(torch.argmax(model.logits(w @ vals)))
        out.append(t)
        anchor, pos = t, pos + 1
    return out


def orthrus_rounds(model, prompt, n_new, K, p_true, seed, reference):
    rng = np.random.default_rng(seed)
    n_pages = (len(prompt) + n_new + 2 * K) // P + 2
    table = np.arange(n_pages, dtype=np.int32)[::-1].copy().reshape(1, -1)  # reversed pages
    kc = np.zeros((n_pages, 1, P, D), np.uint16)
    vc = np.zeros((n_pages, 1, P, D), np.uint16)
    lens = np.zeros(1, np.int32)
    # prefill: append the prompt's KV (all but the anchor) through the oracle
    pre = prompt[:-1]
    if pre:
        kb = np.stack([W.bf16_bits(model.qkv(t, p)[1]) for p, t in enumerate(pre)])[:, None]
        vb = np.stack([W.bf16_bits(model.qkv(t, p)[2]) for p, t in enumerate(pre)])[:, None]
        assert oracle.kv_append(kb, vb, np.array([0, len(pre)], np.int32),
                                np.array([len(pre)], np.int32), lens, table, kc, vc) == 0
    anchor, out, rounds = prompt[-1], [], 0
    while len(out) < n_new:
        pos = int(lens[0])
        s = len(out)
        truth = reference[s:s + K] + [0] * K
        drafts = [truth[i] if rng.random() < p_true else int(rng.integers(0, V))
                  for i in range(K)]
        block = [anchor] + drafts[:K - 1]
        qkv = [model.qkv(t, pos + i) for i, t in enumerate(block)]
        q = np.stack([W.bf16_bits(x[0]) for x in qkv])[:, None]
        kb = np.stack([W.bf16_bits(x[1]) for x in qkv])[:, None]
        vb = np.stack([W.bf16_bits(x[2]) for x in qkv])[:, None]
        cu = np.array([0, K], np.int32)
        o = oracle.block_attn(oracle.VIEW_VERIFY, q, kc, vc, kb, vb, lens, cu, table)
        logits = np.stack([model.logits(o[i, 0]).numpy() for i in range(K)])
        acc, nxt, am = oracle.consensus(logits, np.array(drafts, np.int32), cu)
        n = int(acc[0])
        out.extend(int(t) for t in am[:n])
        assert oracle.kv_append(kb, vb, cu, acc, lens, table, kc, vc) == 0
        assert lens[0] == pos + n
        anchor = int(nxt[0])
        rounds += 1
    return out[:n_new], rounds


@pytest.mark.parametrize("K,p_true,seed", [(4, 0.7, 0), (8, 0.9, 1), (3, 0.0, 2), (6, 1.0, 3)])
def test_orthrus_round_emits_sequential_greedy_stream(K, p_true, seed):
    model = TinyModel(seed)
    g = torch.Generator().manual_seed(100 + seed)
    prompt = torch.randint(0, V, (11,), generator=g).tolist()
    n_new = 40
    ref = sequential_greedy(model, prompt, n_new)
    got, rounds = orthrus_rounds(model, prompt, n_new, K, p_true, seed, ref)
    assert got == ref
    if p_true == 1.0:
        assert rounds == -(-n_new // K)       # every draft right: K tokens per round
    if p_true == 0.0:
        assert rounds >= n_new * 0.9          # almost always just the correction
