"""End-to-end Orthrus rounds on the GPU: losslessness and tokens per forward.

The technical summary's decoding loop (§2.3; "lossless" in §3 and §4) runs
entirely through the library: VERIFY attention that also writes the block's K/V
(`orthrus_block_attn_verify_write`), the fused LM head + consensus + commit
(`orthrus_lm_head_consensus` with prefix_lens), and the anchor hand-over.
Every round also runs the DIFFUSION view's attention call on the same cache.

The synthetic model is built so that its greedy decisions have margins far
above bf16/fp32 rounding, which makes exact stream equality a fair test:
  * q(p) = a*u(p), k(p) = a*u(p+1) with u(p) random unit vectors in 64
    dimensions: position p attends (weight > 0.9999) to position p-1, which is
    the cache for a block's first row and the block itself for the others;
  * v(p) = e(token at p), e(.) random unit vectors;
  * LM head rows w[f(s)] = b*e(s) for a random permutation f: the greedy token
    after position p is f(token at p-1), with a margin of about 0.7*b.
So greedy decoding follows x[p+1] = f(x[p-1]) from the prompt. The loop must
emit exactly that stream, for any drafts, in every round:
  - the Orthrus rounds with K-token blocks and drafts right with probability p,
  - the same rounds with one-token blocks (plain sequential greedy on the GPU),
and the committed lengths must follow the accepted counts. The mean accepted
length per round (tokens per forward, TPF) must match the drafts' geometry:
the number of leading right drafts plus one, capped at K.
"""
import numpy as np
import pytest
import torch

from tests._gpu import gpu, lib, needs_cuda

pytestmark = [gpu, needs_cuda]

V, D, P = 64, 64, 64
ALPHA, BETA = 16.0, 8.0


class ShiftModel:
    def __init__(self, seed, max_pos):
        g = torch.Generator().manual_seed(seed)
        u = torch.randn(max_pos + 2, D, generator=g, dtype=torch.float64)
        self.u = u / u.norm(dim=1, keepdim=True)
        e = torch.randn(V, D, generator=g, dtype=torch.float64)
        self.e = e / e.norm(dim=1, keepdim=True)
        self.f = torch.randperm(V, generator=g)
        w = torch.empty(V, D, dtype=torch.float64)
        w[self.f] = BETA * self.e            # w[f(s)] = b * e(s)
        self.w_head = w.to(torch.bfloat16)

    def rows(self, tokens, pos0):
        """q, k, v rows [n, 1, D] (bf16) for tokens at positions pos0 .."""
        p = torch.arange(pos0, pos0 + len(tokens))
        q = (ALPHA * self.u[p]).to(torch.bfloat16)[:, None]
        k = (ALPHA * self.u[p + 1]).to(torch.bfloat16)[:, None]
        v = self.e[torch.as_tensor(tokens)].to(torch.bfloat16)[:, None]
        return q, k, v

    def greedy_stream(self, prompt, n):
        x = list(prompt)
        while len(x) < len(prompt) + n:
            x.append(int(self.f[x[-2]]))
        return x[len(prompt):]


def run_rounds(model, prompt, n_new, K, p_true, seed, reference, max_pos):
    O = lib()
    dev = "cuda"
    rng = np.random.default_rng(seed)
    n_pages = max_pos // P + 2
    table = torch.from_numpy(np.random.default_rng(seed + 1).permutation(n_pages).astype(np.int32))
    table = table.reshape(1, -1).to(dev)
    kc = torch.zeros((n_pages, 1, P, D), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    lens = torch.zeros(1, dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    # prefill: the prompt's K/V except the anchor's
    pre = prompt[:-1]
    _, kp, vp = model.rows(pre, 0)
    O.kv_append(kp.to(dev), vp.to(dev), torch.tensor([0, len(pre)], dtype=torch.int32, device=dev),
                len(pre), torch.tensor([len(pre)], dtype=torch.int32, device=dev), lens, table,
                kc, vc, update_lens=True, error_flag=err)
    cu = torch.tensor([0, K], dtype=torch.int32, device=dev)
    acc = torch.zeros(1, dtype=torch.int32, device=dev)
    nxt = torch.zeros(1, dtype=torch.int32, device=dev)
    am = torch.zeros(K, dtype=torch.int32, device=dev)
    w_head = model.w_head.to(dev)
    ws_lm = torch.empty(O.lm_head_workspace_size(K), dtype=torch.uint8, device=dev)
    ws_attn = None
    anchor, out, accepts, expect = prompt[-1], [], [], []
    pos = len(pre)
    while len(out) < n_new:
        s = len(out)
        truth = reference[s:s + K] + [0] * K
        drafts = [truth[i] if rng.random() < p_true else int(rng.integers(0, V)) for i in range(K)]
        m = 0
        while m < K and drafts[m] == truth[m]:
            m += 1
        expect.append(min(m + 1, K))
        block = [anchor] + drafts[:K - 1]
        q, kb, vb = (t.to(dev) for t in model.rows(block, pos))
        o = torch.empty_like(q)
        p = O.attn_params("verify", q, kc, vc, kb, vb, lens, cu, table, o, K)
        n = O.block_attn_workspace_size(p)
        if ws_attn is None or ws_attn.numel() < n:
            ws_attn = torch.empty(n, dtype=torch.uint8, device=dev)
        # the drafting view reads the same cache (its output is not used here)
        od = torch.empty_like(q)
        O.block_attn("diffusion", q, kc, vc, kb, vb, lens, cu, table, od, ws_attn, K, error_flag=err)
        O.block_attn_verify_write(q, kc, vc, kb, vb, lens, cu, table, o, ws_attn, K, error_flag=err)
        O.lm_head_consensus(o.view(K, D), w_head, torch.tensor(drafts, dtype=torch.int32, device=dev),
                            cu, 1, K, acc, nxt, ws_lm, row_argmax=am, prefix_lens=lens,
                            error_flag=err)
        torch.cuda.synchronize()
        n_acc = int(acc.item())
        out.extend(int(t) for t in am[:n_acc].tolist())
        accepts.append(n_acc)
        pos += n_acc
        assert int(lens.item()) == pos
        anchor = int(nxt.item())
        assert anchor == out[-1]
    assert int(err.item()) == 0
    return out[:n_new], accepts, expect


@pytest.mark.parametrize("K,p_true,seed", [(32, 0.8, 0), (16, 0.9, 1), (8, 0.0, 2), (32, 1.0, 3)])
def test_gpu_rounds_are_lossless(K, p_true, seed):
    n_new, max_pos = 200, 512
    model = ShiftModel(seed, max_pos)
    g = torch.Generator().manual_seed(100 + seed)
    prompt = torch.randint(0, V, (70,), generator=g).tolist()  # crosses a page boundary
    ref = model.greedy_stream(prompt, n_new + K)
    got, accepts, expect = run_rounds(model, prompt, n_new, K, p_true, seed, ref, max_pos)
    assert got == ref[:n_new]
    assert accepts == expect
    tpf = float(np.mean(accepts))
    if p_true == 1.0:
        assert all(a == K for a in accepts)
    if p_true == 0.0:
        assert tpf < 1.1
    print(f"K={K} p={p_true}: {len(accepts)} rounds, tokens per forward {tpf:.2f}")


def test_sequential_greedy_on_gpu_matches():
    """One-token blocks (K = 1): the library's rounds are plain greedy decoding,
    and emit the same stream."""
    n_new, max_pos = 120, 512
    model = ShiftModel(5, max_pos)
    prompt = torch.randint(0, V, (40,), generator=torch.Generator().manual_seed(5)).tolist()
    ref = model.greedy_stream(prompt, n_new + 1)
    got, accepts, _ = run_rounds(model, prompt, n_new, 1, 0.5, 5, ref, max_pos)
    assert got == ref[:n_new]
    assert all(a == 1 for a in accepts)
