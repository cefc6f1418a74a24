"""Back-to-back attention calls on the launch shapes that stress the pipeline
hand-offs: the 2048-token fixed-chunk split of the 131,072-token prefix
(520 CTAs, several per SM in turn) and the Qwen3-8B-shaped batch on one CTA per
SM (units cut across CTAs). Every call must finish without a pipeline wait
running out (ORTHRUS_FLAG_TIMEOUT) and give the same output as the first call.

A hand-off that loses or double-counts one barrier arrival shows up here as an
intermittent timeout: the kernel's bounded waits turn it into a flag, and the
call still returns."""
import pytest
import torch

from diffusion_draft_ar_b200 import workloads as W
from tests._gpu import gpu, lib, needs_cuda

pytestmark = [gpu, needs_cuda]


@pytest.mark.parametrize("name,max_ctas,split,calls", [
    ("longctx", 0, 2048, 2000),
    ("qwen3_8b", 148, 0, 1000),
    ("ragged", 0, 0, 200),
])
def test_back_to_back_calls_never_time_out(name, max_ctas, split, calls):
    O = lib()
    w = W.WORKLOADS[name]
    wi = W.WorkloadInputs(w, device="cuda", seed=0, rounds=1)
    m, r = wi.meta, wi.rounds[0]
    lens, cu, table = m.prefix_lens.cuda(), m.cu_block.cuda(), m.page_table.cuda()
    view = "verify"
    out = torch.empty_like(r.q[view])
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    p = O.attn_params(view, r.q[view], wi.k_cache, wi.v_cache, r.k_block[view], r.v_block[view],
                      lens, cu, table, out, w.max_block, kv_split_tokens=split, max_ctas=max_ctas)
    ws = torch.empty(O.block_attn_workspace_size(p), dtype=torch.uint8, device="cuda")

    def call():
        O.block_attn(view, r.q[view], wi.k_cache, wi.v_cache, r.k_block[view], r.v_block[view],
                     lens, cu, table, out, ws, w.max_block, kv_split_tokens=split,
                     max_ctas=max_ctas, error_flag=err)

    call()
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    first = out.clone()
    batch = 50
    for done in range(0, calls, batch):
        for _ in range(batch):
            call()
        torch.cuda.synchronize()
        f = int(err.item())
        assert f == 0, f"flags {f:#x} after {done + batch} calls"
    assert torch.equal(out, first)
