"""The library's calls can be captured in a CUDA graph: they allocate nothing,
never synchronise, and read everything they need at launch from device memory.

One round of the Qwen3-1.7B-shaped workload (DIFFUSION attention,
write-then-truncate VERIFY attention, consensus with commit, and the fused LM
head with commit) is run eagerly, then captured once and replayed from the same
initial state. Every output, both caches and the lengths must be bit-identical;
the replayed graph re-reads prefix_lens from device memory, so a second replay
advances from the committed lengths exactly as a second eager round does.
"""
import torch

from diffusion_draft_ar_b200 import workloads as W
from tests._gpu import gpu, lib, needs_cuda

pytestmark = [gpu, needs_cuda]


def test_round_replays_from_a_cuda_graph():
    O = lib()
    w = W.WORKLOADS["qwen3_1p7b"]
    wi = W.WorkloadInputs(w, device="cuda", seed=0, rounds=1)
    m, r = wi.meta, wi.rounds[0]
    dev = "cuda"
    cu, table = m.cu_block.to(dev), m.page_table.to(dev)
    lens0 = m.prefix_lens.to(dev)
    kc0, vc0 = wi.k_cache.clone(), wi.v_cache.clone()
    targets = torch.argmax(r.logits, dim=1).to(torch.int32)
    drafts = wi.drafts(0, targets)
    hidden, w_head = W.lm_head_inputs(m.R, w.d_model, w.vocab, dev)

    # state and outputs, allocated once (nothing is allocated inside the capture)
    kc, vc, lens = wi.k_cache, wi.v_cache, lens0.clone()
    outs = {v: torch.empty_like(r.q[v]) for v in W.VIEW_NAMES}
    acc = torch.zeros(m.B, dtype=torch.int32, device=dev)
    nxt = torch.zeros_like(acc)
    acc2, nxt2 = torch.zeros_like(acc), torch.zeros_like(acc)
    am2 = torch.zeros(m.R, dtype=torch.int32, device=dev)
    lens2 = lens0.clone()
    p = O.attn_params("verify", r.q["verify"], kc, vc, r.k_block["verify"], r.v_block["verify"],
                      lens, cu, table, outs["verify"], w.max_block)
    ws_attn = torch.empty(O.block_attn_workspace_size(p), dtype=torch.uint8, device=dev)
    ws_cons = torch.empty(O.consensus_workspace_size(m.B, w.max_block, w.vocab), dtype=torch.uint8,
                          device=dev)
    ws_lm = torch.empty(O.lm_head_workspace_size(m.R), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def round_():
        O.block_attn("diffusion", r.q["diffusion"], kc, vc, r.k_block["diffusion"],
                     r.v_block["diffusion"], lens, cu, table, outs["diffusion"], ws_attn,
                     w.max_block, error_flag=err)
        O.block_attn_verify_write(r.q["verify"], kc, vc, r.k_block["verify"], r.v_block["verify"],
                                  lens, cu, table, outs["verify"], ws_attn, w.max_block,
                                  error_flag=err)
        O.consensus(r.logits, drafts, cu, m.B, w.max_block, acc, nxt, ws_cons, prefix_lens=lens)
        O.lm_head_consensus(hidden, w_head, drafts, cu, m.B, w.max_block, acc2, nxt2, ws_lm,
                            row_argmax=am2, prefix_lens=lens2, error_flag=err)

    def snapshot():
        torch.cuda.synchronize()
        return [t.clone() for t in (outs["diffusion"], outs["verify"], acc, nxt, lens, acc2, nxt2,
                                    am2, lens2, kc, vc)]

    def reset():
        kc.copy_(kc0)
        vc.copy_(vc0)
        lens.copy_(lens0)
        lens2.copy_(lens0)
        torch.cuda.synchronize()

    # eager: two rounds (the second starts from the committed lengths)
    round_()
    eager1 = snapshot()
    round_()
    eager2 = snapshot()

    reset()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        round_()                  # warm the launch path on the capture stream
    torch.cuda.synchronize()
    reset()
    with torch.cuda.graph(g, stream=s):
        round_()
    torch.cuda.synchronize()
    reset()                       # capture only records; state back to the start
    g.replay()
    replay1 = snapshot()
    g.replay()
    replay2 = snapshot()
    assert int(err.item()) == 0
    for a, b in zip(eager1 + eager2, replay1 + replay2):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    assert not torch.equal(eager1[4], eager2[4])  # the lengths did advance
