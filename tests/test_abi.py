"""The C-ABI library without a GPU: it loads, exports every symbol the header
declares, its parameter struct matches the header's layout, and bad arguments
are refused on the host before anything touches CUDA."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

from diffusion_draft_ar_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "orthrus.h")


@pytest.fixture(scope="module")
def O():
    B.build()
    from diffusion_draft_ar_b200 import orthrus
    return orthrus


def declared_functions():
    src = open(HEADER).read()
    return re.findall(r"^ORTHRUS_API\s+[\w\s\*]+?\b(orthrus_\w+)\s*\(", src, flags=re.M)


def test_every_declared_symbol_is_exported(O):
    names = declared_functions()
    assert set(names) >= {"orthrus_block_attn", "orthrus_block_attn_workspace_size",
                          "orthrus_consensus", "orthrus_consensus_workspace_size",
                          "orthrus_kv_append", "orthrus_status_string", "orthrus_last_error",
                          "orthrus_abi_version"}
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB], capture_output=True, text=True,
                         check=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    for n in names:
        assert n in exported, n
        assert hasattr(O.lib, n)
    # nothing else leaks out of the library under an orthrus_ name
    assert {n for n in exported if n.startswith("orthrus_")} == set(names)


def test_abi_version_and_status_strings(O):
    assert O.abi_version() == 1
    for s in range(6):
        assert O.lib.orthrus_status_string(s)
    assert O.lib.orthrus_status_string(99) == b"unknown status"


def test_status_from_flags(O):
    f = O.lib.orthrus_status_from_flags
    assert f(0) == O.OK
    assert f(O.FLAG_TIMEOUT) == O.ERR_TIMEOUT
    assert f(O.FLAG_TIMEOUT | O.FLAG_BAD_PAGE) == O.ERR_TIMEOUT
    assert f(O.FLAG_BAD_PAGE) == O.ERR_DEVICE_CHECK
    assert f(O.FLAG_BAD_LENGTH) == O.ERR_DEVICE_CHECK


def test_noalloc_rejects_requests_beyond_its_array_on_the_host(O):
    """The no-allocation consensus refuses a request whose keys exceed its fixed
    array before any CUDA call (so this runs without a GPU)."""
    V = 151936
    B, K = 300, 32      # 9600 rows x 10 chunks = 96000 keys > 65536
    st = O.lib.orthrus_consensus_noalloc(ctypes.c_void_p(16), V, V, ctypes.c_void_p(16), None,
                                         B, K, ctypes.c_void_p(16), ctypes.c_void_p(16), None,
                                         None)
    assert st == O.ERR_UNSUPPORTED
    assert b"scratch" in O.lib.orthrus_last_error()


def test_param_struct_layout_matches_header(O):
    fields = [f[0] for f in O.AttnParams._fields_]
    prog = ["#include <stdio.h>", "#include <stddef.h>", '#include "orthrus.h"', "int main(void){",
            'printf("%zu\\n", sizeof(orthrus_attn_params));']
    for f in fields:
        prog.append(f'printf("%zu\\n", offsetof(orthrus_attn_params, {f}));')
    prog.append("return 0;}")
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "layout.c")
        exe = os.path.join(d, "layout")
        open(c, "w").write("\n".join(prog))
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), "-o", exe, c], check=True)
        vals = [int(x) for x in subprocess.run([exe], capture_output=True, text=True,
                                                check=True).stdout.split()]
    assert vals[0] == ctypes.sizeof(O.AttnParams)
    for f, off in zip(fields, vals[1:]):
        assert getattr(O.AttnParams, f).offset == off, f


def _params(O, **kw):
    p = O.AttnParams()
    base = dict(view=1, B=2, Hq=8, Hkv=2, D=128, page_size=64, max_pages_per_seq=4, num_pages=8,
                max_block=8, total_rows=16, q_block=0x10000, k_cache=0x20000, v_cache=0x30000,
                k_block=0x40000, v_block=0x50000, prefix_lens=0x60000, cu_block=None,
                page_table=0x70000, softmax_scale=0.0, kv_split_tokens=0, max_ctas=0,
                out=0x80000, workspace=0x90000, workspace_bytes=1 << 30, error_flag=None)
    base.update(kw)
    for k, v in base.items():
        setattr(p, k, v)
    return p


@pytest.mark.parametrize("kw,status", [
    (dict(view=2), 1), (dict(B=-1), 1), (dict(Hq=6, Hkv=4), 1), (dict(Hkv=0), 1),
    (dict(max_block=0), 1), (dict(D=96), 2), (dict(page_size=32), 2), (dict(max_block=65), 2),
    (dict(Hq=16, Hkv=1, max_block=16), 2), (dict(kv_split_tokens=100), 2),
    (dict(kv_split_tokens=-64), 1), (dict(total_rows=-1), 1), (dict(total_rows=4), 1),
    (dict(q_block=None), 1), (dict(out=None), 1), (dict(k_cache=0x20008), 1),
    (dict(workspace=None), 1), (dict(prefix_lens=None), 1), (dict(page_table=None), 1),
    (dict(num_pages=0), 1), (dict(max_pages_per_seq=0), 1),
])
def test_block_attn_rejects_bad_arguments(O, kw, status):
    p = _params(O, **kw)
    assert O.lib.orthrus_block_attn(ctypes.byref(p), None) == status
    assert O.lib.orthrus_last_error() != b""


def test_block_attn_empty_batch_is_a_no_op(O):
    p = _params(O, B=0, q_block=None, out=None)
    assert O.lib.orthrus_block_attn(ctypes.byref(p), None) == 0


def test_block_attn_workspace_size_chunked_mode(O):
    # fixed 2048-token chunks: one partial slot per (unit, chunk), whatever the
    # number of CTAs that walk the slots (max_ctas only caps that grid)
    p = _params(O, B=1, Hq=32, Hkv=8, max_block=32, total_rows=32, max_pages_per_seq=2049,
                num_pages=2049, kv_split_tokens=2048)
    n = O.block_attn_workspace_size(p)
    chunks = -(-2049 * 64 // 2048)
    parts = chunks * 8
    assert n == parts * 128 * 128 * 4 + (-(-parts * 128 * 4 // 256)) * 256
    for cap in (1, 7, 130, 10 ** 6):
        p.max_ctas = cap
        assert O.block_attn_workspace_size(p) == n
    assert O.block_attn_workspace_size(_params(O, D=96, kv_split_tokens=64)) == 0


def test_block_attn_balanced_workspace_holds_two_partials_per_cta(O):
    # balanced ranges over max_ctas CTAs: a CTA's first and last segments may
    # each be a partial
    for cap in (1, 7, 148):
        n = O.block_attn_workspace_size(_params(O, max_ctas=cap))
        parts = 2 * cap
        assert n == parts * 128 * 128 * 4 + (-(-parts * 128 * 4 // 256)) * 256


def test_block_attn_kernel_count(O):
    # fixed chunks and an explicit CTA cap always merge partials: two kernels;
    # invalid parameters: 0 (both decided on the host, no device query)
    p = _params(O, B=1, Hq=32, Hkv=8, max_block=32, total_rows=32, max_pages_per_seq=2049,
                num_pages=2049, kv_split_tokens=2048)
    assert O.block_attn_kernel_count(p) == 2
    assert O.block_attn_kernel_count(_params(O, max_ctas=7)) == 2
    assert O.block_attn_kernel_count(_params(O, D=96, kv_split_tokens=64)) == 0


@pytest.mark.parametrize("args,status", [
    (dict(V=0), 1), (dict(ld=10, V=20), 1), (dict(B=-1), 1), (dict(max_block=0), 1),
    (dict(logits=None), 1), (dict(draft=None), 1), (dict(workspace=None), 1),
    (dict(workspace_bytes=8), 1), (dict(logits=0x10002), 1),
])
def test_consensus_rejects_bad_arguments(O, args, status):
    a = dict(logits=0x10000, ld=512, V=512, draft=0x20000, cu=None, B=2, max_block=8,
             acc=0x30000, nxt=0x40000, am=None, workspace=0x50000, workspace_bytes=1 << 20)
    a.update(args)
    st = O.lib.orthrus_consensus(a["logits"], a["ld"], a["V"], a["draft"], a["cu"], a["B"],
                                 a["max_block"], a["acc"], a["nxt"], a["am"], a["workspace"],
                                 a["workspace_bytes"], None)
    assert st == status


def test_consensus_workspace_size(O):
    assert O.consensus_workspace_size(16, 32, 151936) == 16 * 32 * 10 * 8
    assert O.consensus_workspace_size(1, 8, 512) == 8 * 8
    assert O.consensus_workspace_size(-1, 8, 512) == 0


@pytest.mark.parametrize("args", [
    dict(D=12), dict(Hkv=0), dict(page_size=0), dict(k_block=None), dict(prefix_lens=None),
    dict(k_cache=0x30004), dict(cu=None, max_block=0),
])
def test_kv_append_rejects_bad_arguments(O, args):
    a = dict(k_block=0x10000, v_block=0x20000, cu=0x1000, max_block=8, acc=0x2000, lens=0x3000,
             table=0x4000, k_cache=0x30000, v_cache=0x40000, B=2, Hkv=2, D=128, page_size=64)
    if "prefix_lens" in args:
        a["lens"] = args.pop("prefix_lens")
    a.update(args)
    st = O.lib.orthrus_kv_append(a["k_block"], a["v_block"], a["cu"], a["max_block"], a["acc"],
                                 a["lens"], 1, a["table"], 4, 8, a["k_cache"], a["v_cache"],
                                 a["B"], a["Hkv"], a["D"], a["page_size"], None, None)
    assert st == 1


@pytest.mark.parametrize("kw,status", [
    (dict(view=0), 1), (dict(view=2), 1), (dict(D=96), 2), (dict(q_block=None), 1),
    (dict(k_cache=0x20008), 1), (dict(workspace=None), 1),
])
def test_block_attn_verify_write_rejects_bad_arguments(O, kw, status):
    # write-then-truncate runs the VERIFY view only; the rest as orthrus_block_attn
    p = _params(O, **kw)
    assert O.lib.orthrus_block_attn_verify_write(ctypes.byref(p), None) == status
    assert O.lib.orthrus_last_error() != b""


def test_block_attn_verify_write_empty_batch_is_a_no_op(O):
    p = _params(O, B=0, q_block=None, out=None)
    assert O.lib.orthrus_block_attn_verify_write(ctypes.byref(p), None) == 0


@pytest.mark.parametrize("args,status", [
    (dict(lens=None), 1), (dict(V=0), 1), (dict(workspace=None), 1), (dict(logits=0x10002), 1),
])
def test_consensus_commit_rejects_bad_arguments(O, args, status):
    a = dict(logits=0x10000, ld=512, V=512, draft=0x20000, cu=None, B=2, max_block=8,
             acc=0x30000, nxt=0x40000, am=None, lens=0x60000, workspace=0x50000,
             workspace_bytes=1 << 20)
    a.update(args)
    st = O.lib.orthrus_consensus_commit(a["logits"], a["ld"], a["V"], a["draft"], a["cu"], a["B"],
                                        a["max_block"], a["acc"], a["nxt"], a["am"], a["lens"],
                                        a["workspace"], a["workspace_bytes"], None)
    assert st == status


@pytest.mark.parametrize("args,status", [
    (dict(d=96), 2), (dict(d=0), 1), (dict(V=0), 1), (dict(B=-1), 1), (dict(max_block=0), 1),
    (dict(hidden=None), 1), (dict(w_head=None), 1), (dict(draft=None), 1), (dict(ws=None), 1),
    (dict(hidden=0x10008), 1), (dict(ws_bytes=8), 1), (dict(total_rows=4, cu=None), 1),
])
def test_lm_head_rejects_bad_arguments(O, args, status):
    a = dict(hidden=0x10000, w_head=0x20000, d=128, V=1000, total_rows=0, draft=0x30000,
             cu=0x40000, B=2, max_block=8, acc=0x50000, nxt=0x60000, ws=0x70000,
             ws_bytes=1 << 20)
    a.update(args)
    st = O.lib.orthrus_lm_head_consensus(a["hidden"], a["w_head"], a["d"], a["V"], a["total_rows"],
                                         a["draft"], a["cu"], a["B"], a["max_block"], a["acc"],
                                         a["nxt"], None, None, a["ws"], a["ws_bytes"], None, None)
    assert st == status
    assert O.lib.orthrus_last_error() != b""


def test_lm_head_workspace_size(O):
    assert O.lm_head_workspace_size(512) == 4096
    assert O.lm_head_workspace_size(33) == 512
    assert O.lm_head_workspace_size(0) == 0


@pytest.mark.parametrize("T", [0.0, -1.0, float("inf"), float("nan"), 1e-45])
def test_sampled_consensus_rejects_bad_temperatures_on_the_host(O, T):
    """Temperature 0, negative, infinite, NaN, or so small that 1/T overflows
    fp32: refused before any CUDA call."""
    V = 1000
    st = O.lib.orthrus_consensus_sampled(ctypes.c_void_p(16), V, V, ctypes.c_void_p(16), None,
                                         2, 4, T, 1, 2, ctypes.c_void_p(16), ctypes.c_void_p(16),
                                         None, None, ctypes.c_void_p(16), 1 << 20, None)
    assert st in (O.ERR_INVALID_ARG, O.ERR_UNSUPPORTED)
    assert b"temperature" in O.lib.orthrus_last_error()


def test_plan_struct_layout_matches_header(O):
    fields = [f[0] for f in O.AttnPlan._fields_]
    prog = ["#include <stdio.h>", "#include <stddef.h>", '#include "orthrus.h"', "int main(void){",
            'printf("%zu\\n", sizeof(orthrus_attn_plan));']
    prog += [f'printf("%zu\\n", offsetof(orthrus_attn_plan, {f}));' for f in fields]
    prog.append("return 0;}")
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "plan.c")
        exe = os.path.join(d, "plan")
        open(c, "w").write("\n".join(prog))
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), "-o", exe, c], check=True)
        vals = [int(x) for x in subprocess.run([exe], capture_output=True, text=True,
                                                check=True).stdout.split()]
    assert vals[0] == ctypes.sizeof(O.AttnPlan)
    for f, off in zip(fields, vals[1:]):
        assert getattr(O.AttnPlan, f).offset == off, f


def _shape(O, B, max_pages, max_block=32, **kw):
    """Qwen3-8B-like heads (32 / 8, D = 128) with B sequences of up to
    max_pages 64-token pages."""
    return _params(O, B=B, Hq=32, Hkv=8, D=128, max_block=max_block, total_rows=B * max_block,
                   max_pages_per_seq=max_pages, num_pages=B * max_pages, **kw)


@pytest.mark.parametrize("name,B,pages,kw,want", [
    # 16 x 8192-token prefixes: 128 units on 148 SMs, one CTA per whole unit
    ("qwen3_8b", 16, 129, {}, dict(schedule=1, grid=128, partial_slots=128, kernels=1,
                                   walks_chunks=0, chunk_tiles=129)),
    # one 131,072-token prefix: 8 units cut in proportion over all SMs
    ("longctx", 1, 2049, {}, dict(schedule=2, grid=148, partial_slots=148, kernels=2,
                                   walks_chunks=0, chunk_tiles=0)),
    # the same in 2048-token chunks: 520 slots spread 4 per CTA over 130 walkers
    ("longctx_2048", 1, 2049, dict(kv_split_tokens=2048),
     dict(schedule=1, grid=130, partial_slots=520, kernels=2, walks_chunks=1, chunk_tiles=32)),
    # ... or over an explicit cap
    ("longctx_2048_cap", 1, 2049, dict(kv_split_tokens=2048, max_ctas=7),
     dict(schedule=1, grid=7, partial_slots=520, kernels=2, walks_chunks=1, chunk_tiles=32)),
    # 64 sequences: 512 units > 148 SMs, balanced ranges (two partial slots per CTA)
    ("ragged", 64, 517, {}, dict(schedule=0, grid=148, partial_slots=296, kernels=2,
                                  walks_chunks=0, chunk_tiles=0)),
    # an explicit CTA count is a balanced split
    ("capped", 16, 129, dict(max_ctas=37), dict(schedule=0, grid=37, partial_slots=74, kernels=2,
                                                 walks_chunks=0, chunk_tiles=0)),
    # few units, none long enough to cut (under 8 tiles): one CTA each, no combine
    ("short", 1, 1, dict(max_block=8), dict(schedule=2, grid=8, partial_slots=8, kernels=1,
                                            walks_chunks=0, chunk_tiles=0)),
])
def test_schedule_plans(O, name, B, pages, kw, want):
    p = _shape(O, B, pages, **kw)
    plan = O.block_attn_plan(p, 148)
    got = {k: getattr(plan, k) for k in want}
    assert got == want, name
    if p.kv_split_tokens > 0 or p.max_ctas > 0:  # no device query needed
        assert plan.workspace_bytes == O.block_attn_workspace_size(p)
        assert plan.kernels == O.block_attn_kernel_count(p)
    slots = plan.partial_slots
    assert plan.workspace_bytes == slots * 128 * 128 * 4 + -(-slots * 128 * 4 // 256) * 256


def test_plan_follows_the_sm_count(O):
    p = _shape(O, 16, 129)
    # 128 units: one CTA each from 128 SMs up to 171 (floor(3 * 171 / 4) = 128)
    assert O.block_attn_plan(p, 128).schedule == 1
    assert O.block_attn_plan(p, 171).schedule == 1
    assert O.block_attn_plan(p, 172).schedule == 2   # fewer units than 3/4 of the SMs
    assert O.block_attn_plan(p, 127).schedule == 0   # more units than SMs
    assert O.block_attn_plan(p, 127).grid == 127


def test_plan_refuses_what_the_call_refuses(O):
    with pytest.raises(O.OrthrusError) as e:
        O.block_attn_plan(_params(O, D=96), 148)
    assert e.value.status == O.ERR_UNSUPPORTED
    assert O.lib.orthrus_block_attn_plan(ctypes.byref(_params(O)), 148, None) == O.ERR_INVALID_ARG
