"""Failure detection without a GPU fault: a copy the pipeline needs is withheld
(ORTHRUS_FAULT_INJECT=1: the first launch of the process withholds one copy per
CTA), so a bounded wait runs out; the kernel must report ORTHRUS_FLAG_TIMEOUT
through the error word, return, and leave the CUDA context usable for the
next, correct call. Runs in a child process so the hook and the short wait
limit (both read once per process) stay local to it."""
import os
import subprocess
import sys

import pytest

from tests._gpu import gpu, needs_cuda

pytestmark = [gpu, needs_cuda]
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import os, sys, numpy as np, torch
sys.path.insert(0, ROOT)
import oracle
from diffusion_draft_ar_b200 import workloads as W
from diffusion_draft_ar_b200 import orthrus as O
from tests._helpers import oracle_attn_args, small_workload
w = small_workload(name="fault", B=3, Hq=8, Hkv=2, D=128, page_size=64, prefix_len=200, block=8,
                   paged=True, headroom=64)
wi = W.WorkloadInputs(w, seed=1)
m, r = wi.meta, wi.rounds[0]
d = lambda t: t.cuda()
args = (d(r.q["verify"]), d(wi.k_cache), d(wi.v_cache), d(r.k_block["verify"]), d(r.v_block["verify"]),
        d(m.prefix_lens), d(m.cu_block), d(m.page_table))
out = torch.zeros_like(args[0])
err = torch.zeros(1, dtype=torch.int32, device="cuda")
p = O.attn_params("verify", *args, out, w.max_block, max_ctas=4)
ws = torch.empty(O.block_attn_workspace_size(p), dtype=torch.uint8, device="cuda")
O.block_attn("verify", *args, out, ws, w.max_block, max_ctas=4, error_flag=err)
torch.cuda.synchronize()
flag = int(err.item())
assert flag & O.FLAG_TIMEOUT, flag
assert O.lib.orthrus_status_from_flags(flag) == O.ERR_TIMEOUT
err.zero_()
O.block_attn("verify", *args, out, ws, w.max_block, max_ctas=4, error_flag=err)
torch.cuda.synchronize()
assert int(err.item()) == 0
ref = oracle.block_attn(*oracle_attn_args(wi, "verify"))
e = np.abs(out.double().cpu().numpy() - ref).max()
assert e <= 2e-2, e
print("FAULT-OK", flag)
'''


def test_withheld_copy_times_out_and_context_survives():
    env = dict(os.environ, ORTHRUS_WAIT_TIMEOUT_MS="50", ORTHRUS_FAULT_INJECT="1",
               PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", "ROOT = %r\n" % ROOT + CHILD], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "FAULT-OK" in r.stdout


CHILD_LM = r"""
import os, sys, numpy as np, torch
sys.path.insert(0, ROOT)
import oracle
from diffusion_draft_ar_b200 import workloads as W
from diffusion_draft_ar_b200 import orthrus as O
g = torch.Generator().manual_seed(2)
R, d, V = 96, 128, 5000
hidden = torch.randint(-1, 2, (R, d), generator=g).to(torch.bfloat16)
w_head = torch.randint(-2, 3, (V, d), generator=g).to(torch.bfloat16)
cu = torch.tensor([0, 32, 64, 96], dtype=torch.int32)
drafts = torch.randint(0, V, (R,), generator=g, dtype=torch.int32)
acc = torch.zeros(3, dtype=torch.int32, device="cuda")
nxt = torch.zeros(3, dtype=torch.int32, device="cuda")
am = torch.zeros(R, dtype=torch.int32, device="cuda")
ws = torch.empty(O.lm_head_workspace_size(R), dtype=torch.uint8, device="cuda")
err = torch.zeros(1, dtype=torch.int32, device="cuda")
args = (hidden.cuda(), w_head.cuda(), drafts.cuda(), cu.cuda(), 3, 32, acc, nxt, ws)
O.lm_head_consensus(*args, row_argmax=am, error_flag=err)
torch.cuda.synchronize()
flag = int(err.item())
assert flag & O.FLAG_TIMEOUT, flag
err.zero_()
O.lm_head_consensus(*args, row_argmax=am, error_flag=err)
torch.cuda.synchronize()
assert int(err.item()) == 0
t = oracle.greedy_tokens(oracle.lm_head_logits(W.bf16_bits(hidden), W.bf16_bits(w_head)))
assert am.cpu().numpy().tolist() == t.tolist()
print("FAULT-OK", flag)
"""


def test_lm_head_withheld_copy_times_out_and_context_survives():
    """The fused LM head's pipeline waits are bounded the same way: a withheld
    w_head copy makes the MMA warp's wait run out; the call reports
    ORTHRUS_FLAG_TIMEOUT, every role winds down, and the next call is exact."""
    env = dict(os.environ, ORTHRUS_WAIT_TIMEOUT_MS="50", ORTHRUS_FAULT_INJECT="1",
               PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", "ROOT = %r\n" % ROOT + CHILD_LM], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "FAULT-OK" in r.stdout
