#!/usr/bin/env python
"""Throughput of one Orthrus block-decoding round on B200.

A step is one pass of the whole hot path over one batch:
  block attention (DIFFUSION view) -> block attention (VERIFY view, storing
  the block K/V: write-then-truncate) -> greedy consensus over the verify
  logits, which commits the accepted lengths
on the Qwen3-8B-shaped workload (16 sequences, prefix 8192, block 32, 32/8
heads, head dim 128, 64-token pages in a random permutation, vocabulary 151936),
inputs resident in HBM. L2 is scrubbed before every timed call (a 256 MB write
then a 256 MB read of another buffer, outside the timed interval), so each call
starts with none of its inputs in L2 and no dirty line to write back; the step
time is the sum of the calls' event-timed intervals. prefix_lens is restored
(64-byte device copy) at the start of every step so each step appends at the
same positions.

The same JSON line carries, measured the same way: the separate kv_append
launch on this workload, the other workloads (Qwen3-1.7B layer, long context,
ragged serving batch), the fused LM head, the end-to-end step through the public
calls with host buffers, and the fp64 CPU oracle on a bounded sample.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs its own batch (weak scaling, no data-path
collective); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from diffusion_draft_ar_b200 import dist as D  # noqa: E402
from diffusion_draft_ar_b200 import workloads as W  # noqa: E402

METRIC = "block-attn KV GB/s (% HBM roofline) at K=32; consensus rows/s; blocks/s"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
ATTN_SRC = os.path.join(ROOT, "diffusion_draft_ar_b200", "csrc", "block_attn.cuh")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "block_attn_qwen3_8b.json")
NOMINAL_HBM_GBS = 8000.0        # the roofline the method's target is stated against
NOMINAL_BF16_TFLOPS = 2250.0    # dense bf16 tensor peak (nominal)


# ---------------------------------------------------------------------------
# algorithmic bytes

def attn_bytes(w: W.Workload, m: W.BatchMeta) -> int:
    """Bytes an ideal kernel moves per call: each prefix K/V element once per
    (sequence, KV head), plus the block's Q, K, V and the output."""
    kv = int(m.prefix_lens.to(torch.int64).sum()) * W.cache_bytes_per_token(w)
    R = m.R
    return kv + R * w.Hq * w.D * 2 * 2 + R * w.Hkv * w.D * 2 * 2


def consensus_bytes(w: W.Workload, m: W.BatchMeta) -> int:
    return m.R * w.vocab * 4 + m.R * 4 * 2 + m.B * 8


def append_bytes(w: W.Workload, accepted: int) -> int:
    return accepted * w.Hkv * w.D * 2 * 2 * 2  # read + write, K and V


def attn_flops(w: W.Workload, m: W.BatchMeta, view: str) -> int:
    tot = 0
    for b in range(m.B):
        L, K = int(m.prefix_lens[b]), int(m.block_lens[b])
        keys = K * (L + K) if view == "diffusion" else K * L + K * (K + 1) // 2
        tot += keys * w.Hq
    return 4 * w.D * tot


# ---------------------------------------------------------------------------
# helpers

def peak_hbm():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def peak_bf16():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured cuBLAS bf16 burst"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def measure_lm_head(O, w: W.Workload, m: W.BatchMeta, dev, stream, calls: int = 20):
    """The fused LM head + greedy consensus on the workload's verify rows (the
    step before consensus when the logits are not materialised): hidden [R, d]
    x w_head [V, d]^T, random bf16 operands of the model's shape. Timed alone,
    CUDA events on the launching stream; w_head (> L2) is re-read every call."""
    if w.d_model is None or w.vocab is None:
        return None
    R, d, V = m.R, w.d_model, w.vocab
    hidden, w_head = W.lm_head_inputs(R, d, V, dev)
    cu = m.cu_block.to(dev)
    drafts = torch.zeros(R, dtype=torch.int32, device=dev)
    acc = torch.zeros(m.B, dtype=torch.int32, device=dev)
    nxt = torch.zeros(m.B, dtype=torch.int32, device=dev)
    ws = torch.empty(O.lm_head_workspace_size(R), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    sp = ctypes.c_void_p(stream.cuda_stream)
    args = (hidden.data_ptr(), w_head.data_ptr(), d, V, R, drafts.data_ptr(), cu.data_ptr(), m.B,
            w.max_block, acc.data_ptr(), nxt.data_ptr(), None, None, ws.data_ptr(), ws.numel(),
            err.data_ptr(), sp)

    def call():
        st = O.lib.orthrus_lm_head_consensus(*args)
        if st:
            raise RuntimeError(f"orthrus_lm_head_consensus: {O.lib.orthrus_last_error().decode()}")

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(calls):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"lm_head device error flag {int(err.item())}")
    us = e0.elapsed_time(e1) / calls * 1e3
    flops = 2.0 * R * d * V
    tflops = flops / (us * 1e-6) / 1e12
    peak, src = peak_bf16()
    del hidden, w_head
    return {"workload": f"{w.name} verify rows through the LM head: {R} x {d} x {V} (bf16, fp32 acc)",
            "us": us, "calls": calls, "tflops": tflops,
            "w_head_gbs": 2.0 * V * d / (us * 1e-6) / 1e9,
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                         "frac": tflops / peak, "peak_source": src},
            "kernels_per_call": 2, "note": "memset of the row keys, GEMM+argmax kernel, "
                                           "consensus finalize; logits never written"}


def kernel_code_hash(path) -> str:
    """First 16 hex digits of the sha256 of a CUDA source with its comments,
    indentation and blank lines removed: edits to comments keep the hash, any
    change to the code changes it."""
    text = open(path, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*", "", ln).strip() for ln in text.splitlines())
    code = "\n".join(ln for ln in lines if ln)
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def traffic_per_launch():
    """DRAM bytes per attention launch from the committed ncu figures
    (profiles/block_attn_qwen3_8b.json), or None when they are missing or were
    taken on different kernel code."""
    try:
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)
        if d.get("kernel_code_sha256_16") == kernel_code_hash(ATTN_SRC):
            return int(d["dram_bytes_per_launch_full_size"])
    except Exception:
        pass
    return None


class L2Scrub:
    """Leaves L2 cold and clean before a timed call: a 256 MB write evicts every
    line, then a 256 MB read of another buffer makes the write-backs of those
    dirty lines happen before the call, and L2 ends holding clean lines of an
    unrelated buffer. (A write alone would leave ~126 MB of dirty lines whose
    write-back lands inside the next call: on this pool it slows a bare TMA
    stream over the Qwen3-8B cache from 84 to 100 us.)"""

    def __init__(self, dev, mb: int = 256):
        self.a = torch.empty(mb << 20, dtype=torch.uint8, device=dev)
        self.b = torch.ones(mb << 18, dtype=torch.float32, device=dev)
        self.sink = torch.zeros(1, dtype=torch.float32, device=dev)

    def __call__(self):
        self.a.fill_(1)
        torch.sum(self.b, 0, keepdim=True, out=self.sink)


def timed_calls(calls, n: int, scrub: L2Scrub, stream, before=None):
    """Run `n` steps of `calls` (a list of zero-argument functions), scrubbing L2
    before each call; CUDA events on `stream` bracket each call alone. Returns
    an [n, len(calls)] array of milliseconds."""
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in calls] for _ in range(n)]
    for i in range(n):
        if before is not None:
            before()
        for j, f in enumerate(calls):
            scrub()
            evs[i][j][0].record(stream)
            f()
            evs[i][j][1].record(stream)
    torch.cuda.synchronize()
    return np.array([[e0.elapsed_time(e1) for e0, e1 in row] for row in evs])


def hbm_roofline(nbytes: float, flops: float, us: float) -> dict:
    """Achieved bandwidth and both roofline fractions: against the measured copy
    bandwidth, and against max(bytes / 8 TB/s, FLOPs / 2.25 PFLOP/s)."""
    peak, src = peak_hbm()
    gbs = nbytes / (us * 1e-6) / 1e9
    t_nom = max(nbytes / (NOMINAL_HBM_GBS * 1e9), flops / (NOMINAL_BF16_TFLOPS * 1e12))
    return {"us": us, "gbs": gbs, "frac": gbs / peak, "peak_gbs": peak, "peak_source": src,
            "frac_8tbs": t_nom / (us * 1e-6)}


class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_index: int):
        self.proc = None
        self.out = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(dev_index).uuid)
        except Exception:
            uuid = None
        self.cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                    "-lms", "100"] + (["-i", uuid] if uuid else [])

    def start(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        rows = [l.split(",") for l in out.strip().splitlines() if l.count(",") >= 8]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4)
                          if r[5 + i].strip().lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# CPU oracle on a bounded sample (reference arm and cpu_baseline)

class OracleSample:
    """One sequence of the workload: both attention views, its consensus rows and
    its append, computed by the fp64 CPU oracle."""

    def __init__(self, w: W.Workload, seed: int = 0, threads: int | None = None):
        import oracle
        self.oracle = oracle
        self.w1 = w.with_(B=1)
        self.wi = W.WorkloadInputs(self.w1, seed=seed)
        m, r = self.wi.meta, self.wi.rounds[0]
        self.args = {}
        for view in W.VIEW_NAMES:
            self.args[view] = (0 if view == "diffusion" else 1, W.bf16_bits(r.q[view]),
                               W.bf16_bits(self.wi.k_cache), W.bf16_bits(self.wi.v_cache),
                               W.bf16_bits(r.k_block[view]), W.bf16_bits(r.v_block[view]),
                               m.prefix_lens.numpy(), m.cu_block.numpy(), m.page_table.numpy())
        self.logits = r.logits.numpy()
        _, _, t = oracle.consensus(self.logits, np.zeros(m.R, np.int32), m.cu_block.numpy())
        self.drafts = self.wi.drafts(0, torch.from_numpy(t)).numpy()
        self.kc = W.bf16_bits(self.wi.k_cache).copy()
        self.vc = W.bf16_bits(self.wi.v_cache).copy()
        self.bytes = 0
        for view in W.VIEW_NAMES:
            self.bytes += attn_bytes(self.w1, m)
        self.bytes += consensus_bytes(self.w1, m)
        self.threads = threads or oracle.default_threads()

    def run(self) -> int:
        o, m = self.oracle, self.wi.meta
        for view in W.VIEW_NAMES:
            o.block_attn(*self.args[view], threads=self.threads)
        acc, _, _ = o.consensus(self.logits, self.drafts, m.cu_block.numpy(), threads=self.threads)
        lens = m.prefix_lens.numpy().copy()
        r = self.wi.rounds[0]
        o.kv_append(W.bf16_bits(r.k_block["verify"]), W.bf16_bits(r.v_block["verify"]),
                    m.cu_block.numpy(), acc, lens, m.page_table.numpy(), self.kc, self.vc)
        return self.bytes + append_bytes(self.w1, int(acc.sum()))


def _time_oracle(w: W.Workload, budget_s: float, threads: int | None = None):
    s = OracleSample(w, threads=threads)
    done, nbytes, t0 = 0, 0, time.perf_counter()
    while True:
        nbytes += s.run()
        done += 1
        el = time.perf_counter() - t0
        if el >= budget_s or done >= w.B:
            break
    return s, done, nbytes, el


def cpu_baseline(w: W.Workload, budget_s: float = 10.0, single_thread: bool = True) -> dict:
    s, done, nbytes, el = _time_oracle(w, budget_s)
    out = {"value": nbytes / el / 1e9, "unit": UNIT, "cores": s.threads, "kind": "oracle",
           "sample": f"{done} sequence(s) of {w.name} (both attention views over L={w.prefix_len}, "
                     f"consensus over {w.max_block} rows x V={w.vocab}, append), fp64 C oracle, "
                     f"{el:.1f} s"}
    if single_thread:
        # the same oracle on one host thread, on the two small workloads
        st = {}
        for name in ("tiny", "qwen3_1p7b"):
            s1, d1, b1, e1 = _time_oracle(W.WORKLOADS[name], min(budget_s, 5.0), threads=1)
            st[name] = {"value": b1 / e1 / 1e9, "unit": UNIT, "cores": 1,
                        "ms_per_sequence": 1e3 * e1 / d1,
                        "sample": f"{d1} sequence(s): both views, consensus, append"}
        out["single_thread"] = st
    return out


def run_reference(args):
    world, rank, _ = int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0
    if rank != 0:
        return
    w = W.WORKLOADS[args.workload]
    s = OracleSample(w)
    for _ in range(args.warmup):
        s.run()
    times, nbytes = [], 0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        nbytes += s.run()
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = nbytes / total / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "sample": "one sequence per step", "B": w.B,
                   "prefix_len": w.prefix_len, "block": w.block, "Hq": w.Hq, "Hkv": w.Hkv,
                   "D": w.D, "page_size": w.page_size, "vocab": w.vocab},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": s.threads, "kind": "oracle",
                         "sample": "one sequence of the workload per step (both views, "
                                   "consensus, append), fp64 C oracle"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm

class AttnCall:
    """One prepared orthrus_block_attn (or _verify_write) call on device inputs."""

    def __init__(self, O, view, q, k_cache, v_cache, kb, vb, lens, cu, table, max_block,
                 err, stream, kv_split: int = 0, write: bool = False):
        self.O = O
        self.out = torch.empty_like(q)
        self.p = O.attn_params(view, q, k_cache, v_cache, kb, vb, lens, cu, table, self.out,
                               max_block, kv_split_tokens=kv_split, error_flag=err)
        self.ws = torch.empty(max(256, O.block_attn_workspace_size(self.p)), dtype=torch.uint8,
                              device=q.device)
        self.p.workspace, self.p.workspace_bytes = self.ws.data_ptr(), self.ws.numel()
        self.kernels = O.block_attn_kernel_count(self.p)
        self.P = ctypes.byref(self.p)
        self.sp = ctypes.c_void_p(stream.cuda_stream)
        self.fn = O.lib.orthrus_block_attn_verify_write if write else O.lib.orthrus_block_attn

    def __call__(self):
        st = self.fn(self.P, self.sp)
        if st:
            raise RuntimeError(f"attention call failed: {self.O.lib.orthrus_last_error().decode()}")


class ConsensusCall:
    def __init__(self, O, logits, drafts, cu, B, max_block, stream, lens=None):
        dev = logits.device
        self.O = O
        self.acc = torch.zeros(B, dtype=torch.int32, device=dev)
        self.nxt = torch.zeros(B, dtype=torch.int32, device=dev)
        self.ws = torch.empty(O.consensus_workspace_size(B, max_block, logits.shape[1]),
                              dtype=torch.uint8, device=dev)
        sp = ctypes.c_void_p(stream.cuda_stream)
        V = logits.shape[1]
        base = (logits.data_ptr(), V, V, drafts.data_ptr(), cu.data_ptr(), B, max_block,
                self.acc.data_ptr(), self.nxt.data_ptr(), None)
        if lens is None:
            self.fn, self.args = O.lib.orthrus_consensus, base + (self.ws.data_ptr(),
                                                                  self.ws.numel(), sp)
        else:
            self.fn, self.args = O.lib.orthrus_consensus_commit, base + (
                lens.data_ptr(), self.ws.data_ptr(), self.ws.numel(), sp)

    def __call__(self):
        st = self.fn(*self.args)
        if st:
            raise RuntimeError(f"consensus failed: {self.O.lib.orthrus_last_error().decode()}")


def check_flag(err, what):
    v = int(err.item())
    if v:
        raise RuntimeError(f"{what}: device error flag {v}")


def measure_workload(O, name: str, dev, stream, scrub, calls: int, seed: int = 0) -> dict:
    """Per-call times (L2 scrubbed before each call) of one workload's attention
    views, and, where the workload has a vocabulary, its consensus and a whole
    round (DIFFUSION, write-then-truncate VERIFY, consensus with commit)."""
    w = W.WORKLOADS[name]
    wi = W.WorkloadInputs(w, device=dev, seed=seed, rounds=1)
    m, r = wi.meta, wi.rounds[0]
    lens0 = m.prefix_lens.to(dev)
    lens = lens0.clone()
    cu, table = m.cu_block.to(dev), m.page_table.to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    kv = int(m.prefix_lens.to(torch.int64).sum()) * W.cache_bytes_per_token(w)
    res = {"workload": name, "B": m.B, "rows": m.R, "prefix_tokens": int(m.prefix_lens.sum()),
           "kv_bytes": kv, "calls": calls, "views": {}}
    b_attn = attn_bytes(w, m)
    for view in w.views:
        variants = [("library schedule", 0)]
        if w.kv_split_tokens:
            variants.append((f"{w.kv_split_tokens}-token chunks", w.kv_split_tokens))
        for label, split in variants:
            c = AttnCall(O, view, r.q[view], wi.k_cache, wi.v_cache, r.k_block[view],
                         r.v_block[view], lens, cu, table, w.max_block, err, stream,
                         kv_split=split)
            for _ in range(3):
                scrub(); c()
            t = timed_calls([c], calls, scrub, stream)[:, 0]
            check_flag(err, f"{name}/{view}")
            us = float(np.median(t)) * 1e3
            d = hbm_roofline(b_attn, attn_flops(w, m, view), us)
            d.update({"us_mean": float(t.mean()) * 1e3, "kernels": c.kernels,
                      "algorithmic_bytes": b_attn, "blocks_per_s": m.B / (us * 1e-6),
                      "tokens_verified_per_s": m.R / (us * 1e-6) if view == "verify" else None})
            res["views"][view if len(variants) == 1 else f"{view} ({label})"] = d
    if w.vocab is not None and set(w.views) == set(W.VIEW_NAMES):
        targets = torch.argmax(r.logits, dim=1).to(torch.int32)
        drafts = wi.drafts(0, targets)
        diff = AttnCall(O, "diffusion", r.q["diffusion"], wi.k_cache, wi.v_cache,
                        r.k_block["diffusion"], r.v_block["diffusion"], lens, cu, table,
                        w.max_block, err, stream)
        ver = AttnCall(O, "verify", r.q["verify"], wi.k_cache, wi.v_cache, r.k_block["verify"],
                       r.v_block["verify"], lens, cu, table, w.max_block, err, stream,
                       write=True)
        cons = ConsensusCall(O, r.logits, drafts, cu, m.B, w.max_block, stream, lens=lens)
        restore = lambda: lens.copy_(lens0, non_blocking=True)
        for _ in range(3):
            restore()
            for f in (diff, ver, cons):
                scrub(); f()
        t = timed_calls([diff, ver, cons], calls, scrub, stream, before=restore)
        check_flag(err, f"{name} round")
        t_c = float(np.median(t[:, 2])) * 1e3
        b_c = consensus_bytes(w, m)
        round_us = float(np.median(t.sum(1))) * 1e3
        res["consensus"] = {"us": t_c, "gbs": b_c / (t_c * 1e-6) / 1e9,
                            "frac": b_c / (t_c * 1e-6) / 1e9 / peak_hbm()[0],
                            "rows_per_s": m.R / (t_c * 1e-6), "algorithmic_bytes": b_c}
        res["round"] = {"us": round_us, "blocks_per_s": m.B / (round_us * 1e-6),
                        "tokens_verified_per_s": m.R / (round_us * 1e-6),
                        "mean_accept_len": float(cons.acc.float().mean()),
                        "calls": "DIFFUSION attention, write-then-truncate VERIFY attention, "
                                 "consensus with commit"}
    del wi
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    world, rank, local = D.init("nccl", timeout_s=300)
    from diffusion_draft_ar_b200 import orthrus as O
    w = W.WORKLOADS[args.workload]
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    scrub = L2Scrub(dev)
    wi = W.WorkloadInputs(w, device=dev, seed=D.rank_seed(0, rank))
    m, r = wi.meta, wi.rounds[0]
    lens0 = m.prefix_lens.to(dev)
    lens = lens0.clone()
    cu = m.cu_block.to(dev)
    table = m.page_table.to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    write = args.commit == "write"
    targets = torch.argmax(r.logits, dim=1).to(torch.int32)
    drafts = wi.drafts(0, targets)
    diff = AttnCall(O, "diffusion", r.q["diffusion"], wi.k_cache, wi.v_cache,
                    r.k_block["diffusion"], r.v_block["diffusion"], lens, cu, table, w.max_block,
                    err, stream, kv_split=w.kv_split_tokens)
    ver = AttnCall(O, "verify", r.q["verify"], wi.k_cache, wi.v_cache, r.k_block["verify"],
                   r.v_block["verify"], lens, cu, table, w.max_block, err, stream,
                   kv_split=w.kv_split_tokens, write=write)
    cons = ConsensusCall(O, r.logits, drafts, cu, m.B, w.max_block, stream,
                         lens=lens if write else None)
    sp = ctypes.c_void_p(stream.cuda_stream)
    kb, vb = r.k_block["verify"], r.v_block["verify"]
    app_args = (kb.data_ptr(), vb.data_ptr(), cu.data_ptr(), w.max_block, cons.acc.data_ptr(),
                lens.data_ptr(), 1, table.data_ptr(), m.max_pages, m.num_pages,
                wi.k_cache.data_ptr(), wi.v_cache.data_ptr(), m.B, w.Hkv, w.D, w.page_size,
                err.data_ptr(), sp)

    def append():
        st = O.lib.orthrus_kv_append(*app_args)
        if st:
            raise RuntimeError(f"kv_append failed: {O.lib.orthrus_last_error().decode()}")

    step_calls = [diff, ver, cons] + ([] if write else [append])
    launches_per_step = diff.kernels + ver.kernels + 2 + (0 if write else 1)
    restore = lambda: lens.copy_(lens0, non_blocking=True)

    for _ in range(args.warmup):
        restore()
        for f in step_calls:
            scrub(); f()
    torch.cuda.synchronize()
    check_flag(err, "warm-up")

    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index)
    sampler.start()
    time.sleep(0.3)  # let the sampler take its first reading
    D.barrier(world)
    torch.cuda.synchronize()
    t_start.record(stream)
    part = timed_calls(step_calls, args.steps, scrub, stream, before=restore)  # ms
    t_end.record(stream)
    torch.cuda.synchronize()
    D.barrier(world)
    clocks = sampler.stop()
    check_flag(err, "timed steps")
    wall_ms = D.max_over_ranks(t_start.elapsed_time(t_end), world) / args.steps
    ms_step = D.max_over_ranks(float(part.sum(1).mean()), world)
    t_diff, t_ver, t_cons = (float(x) for x in part[:, :3].mean(0))
    t_app = float(part[:, 3].mean()) if not write else None

    accepted = int(cons.acc.sum().item())
    mean_accept = accepted / m.B
    b_attn = attn_bytes(w, m)
    b_step = 2 * b_attn + consensus_bytes(w, m) + append_bytes(w, accepted)
    value = world * b_step / (ms_step * 1e-3) / 1e9
    attn_ms = 0.5 * (t_diff + t_ver)
    flops = 0.5 * (attn_flops(w, m, "diffusion") + attn_flops(w, m, "verify"))
    roof_att = hbm_roofline(b_attn, flops, attn_ms * 1e3)

    # ---- the separate append launch on the same rows (accept lengths of the last step)
    app_calls = 50
    for _ in range(3):
        restore(); scrub(); append()
    t = timed_calls([append], app_calls, scrub, stream, before=restore)[:, 0]
    check_flag(err, "kv_append")
    app_us = float(np.median(t)) * 1e3
    b_app = append_bytes(w, accepted)
    kv_append = {"us": app_us, "gbs": b_app / (app_us * 1e-6) / 1e9,
                 "frac": b_app / (app_us * 1e-6) / 1e9 / peak_hbm()[0],
                 "algorithmic_bytes": b_app, "accepted_rows": accepted, "calls": app_calls,
                 "note": "orthrus_kv_append of the accepted VERIFY rows (K and V, read + write), "
                         "prefix lengths restored before each call; latency-bound at this size"}

    # ---- consensus at temperature 1 (Gumbel-max sample) on the same logits
    s_acc = torch.zeros(m.B, dtype=torch.int32, device=dev)
    s_nxt = torch.zeros(m.B, dtype=torch.int32, device=dev)
    s_args = (r.logits.data_ptr(), w.vocab, w.vocab, drafts.data_ptr(), cu.data_ptr(), m.B,
              w.max_block, 1.0, 1234, 0, s_acc.data_ptr(), s_nxt.data_ptr(), None, None,
              cons.ws.data_ptr(), cons.ws.numel(), sp)

    def sampled():
        st = O.lib.orthrus_consensus_sampled(*s_args)
        if st:
            raise RuntimeError(f"consensus_sampled failed: {O.lib.orthrus_last_error().decode()}")

    for _ in range(3):
        scrub(); sampled()
    t = timed_calls([sampled], 20, scrub, stream)[:, 0]
    smp_us = float(np.median(t)) * 1e3
    consensus_sampled = {
        "us": smp_us, "temperature": 1.0,
        "gbs": consensus_bytes(w, m) / (smp_us * 1e-6) / 1e9,
        "rows_per_s": m.R / (smp_us * 1e-6),
        "vs_greedy": smp_us / (t_cons * 1e3),
        "note": "orthrus_consensus_sampled: Philox4x32-10 noise and two logarithms per "
                "logit on the fly (no noise read from memory); ALU-bound"}

    # ---- end to end through the public API: pinned host inputs in, results out ----
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    h_in = {k: t.cpu().pin_memory() for k, t in (
        ("qd", r.q["diffusion"]), ("kd", r.k_block["diffusion"]), ("vd", r.v_block["diffusion"]),
        ("qv", r.q["verify"]), ("kv", r.k_block["verify"]), ("vv", r.v_block["verify"]),
        ("logits", r.logits), ("drafts", drafts))}
    d_in = {"qd": r.q["diffusion"], "kd": r.k_block["diffusion"], "vd": r.v_block["diffusion"],
            "qv": r.q["verify"], "kv": r.k_block["verify"], "vv": r.v_block["verify"],
            "logits": r.logits, "drafts": drafts}
    h_out = {"od": torch.empty_like(diff.out, device="cpu").pin_memory(),
             "ov": torch.empty_like(ver.out, device="cpu").pin_memory(),
             "acc": torch.empty_like(cons.acc, device="cpu").pin_memory(),
             "nxt": torch.empty_like(cons.nxt, device="cpu").pin_memory()}
    d_out = {"od": diff.out, "ov": ver.out, "acc": cons.acc, "nxt": cons.nxt}
    h2d = sum(t.numel() * t.element_size() for t in h_in.values())
    d2h = sum(t.numel() * t.element_size() for t in h_out.values())
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    D.barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(e2e_steps):
        for k in h_in:
            d_in[k].copy_(h_in[k], non_blocking=True)
        restore()
        for f in step_calls:
            f()
        for k in h_out:
            h_out[k].copy_(d_out[k], non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    D.barrier(world)
    check_flag(err, "e2e")
    e2e_ms = D.max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps
    e2e_value = world * b_step / (e2e_ms * 1e-3) / 1e9
    del wi, h_in, h_out
    torch.cuda.empty_cache()

    # ---- the other workloads, each timed alone ----
    configs = {}
    if not args.no_configs:
        for name in ("qwen3_1p7b", "longctx", "ragged"):
            configs[name] = measure_workload(O, name, dev, stream, scrub, args.config_calls)

    lm_head = None if args.no_lm_head else measure_lm_head(O, w, m, dev, stream)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, budget_s=args.cpu_seconds)

    if rank == 0:
        roof = {"bound": "hbm", "achieved": roof_att["gbs"], "peak": roof_att["peak_gbs"],
                "unit": "GB/s", "frac": roof_att["frac"], "frac_8tbs": roof_att["frac_8tbs"],
                "traffic": traffic_per_launch(),
                "kernel": "orthrus_block_attn (attention + split combine), mean of both views",
                "algorithmic_bytes_per_launch": b_attn, "us_per_launch": attn_ms * 1e3,
                "peak_source": f"{roof_att['peak_source']} HBM copy bandwidth (MEASURED_PEAKS)",
                "frac_8tbs_definition": "max(bytes / 8 TB/s, FLOPs / 2.25 PFLOP/s) / time",
                "l2": "scrubbed before every launch",
                "tensor_tflops": flops / (attn_ms * 1e-3) / 1e12}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16 Q/K/V, fp32 logits; no weights)",
            "config": {"workload": w.name, "B": w.B, "prefix_len": w.prefix_len, "block": w.block,
                       "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D, "page_size": w.page_size,
                       "vocab": w.vocab,
                       "pages": "random permutation" if w.paged else "contiguous",
                       "parallelism": f"dp{world} (independent batches)",
                       "l2": "flushed before every timed call (256 MB write, then 256 MB read "
                             "of another buffer, outside the timed interval); ms_per_step is "
                             "the sum of the calls' event-timed intervals"},
            "ms_per_step_incl_flush": wall_ms,
            "block_attn_gbs": roof_att["gbs"], "block_attn_us": {"diffusion": t_diff * 1e3,
                                                                 "verify": t_ver * 1e3},
            "consensus_rows_per_s": world * m.R / (t_cons * 1e-3),
            "consensus_us": t_cons * 1e3,
            "consensus_gbs": consensus_bytes(w, m) / (t_cons * 1e-3) / 1e9,
            "kv_append_us": t_app * 1e3 if t_app is not None else None,
            "kv_append": kv_append,
            "consensus_sampled": consensus_sampled,
            "commit": ("write-then-truncate (VERIFY attention stores the block K/V; "
                       "consensus advances the lengths)") if write else
                      "separate kv_append of the accepted rows",
            "blocks_per_s": world * m.B / (ms_step * 1e-3),
            "tokens_verified_per_s": world * m.R / (t_ver * 1e-3),
            "mean_accept_len": mean_accept,
            "roofline": roof,
            "configs": configs,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps, "ms_per_step": e2e_ms,
                    "note": "per step: pinned H2D of both views' q/k/v blocks, logits and drafts; "
                            "D2H of both outputs, accept lengths and next tokens; "
                            "the KV cache stays resident; no L2 flush"},
            "gpu_launches": args.steps * launches_per_step,
            "lm_head": lm_head,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    D.finish(world)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    # the step needs both attention views and a vocabulary (longctx is VERIFY-only
    # attention: a parity case, timed by its own tests)
    steps_ok = sorted(n for n, w in W.WORKLOADS.items()
                      if w.vocab is not None and set(w.views) == set(W.VIEW_NAMES))
    ap.add_argument("--workload", default="qwen3_8b", choices=steps_ok)
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-lm-head", action="store_true",
                    help="skip the separate fused LM-head measurement")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the Qwen3-1.7B, long-context and ragged measurements")
    ap.add_argument("--config-calls", type=int, default=20,
                    help="timed calls per measurement on the other workloads")
    ap.add_argument("--commit", choices=["write", "append"], default="write",
                    help="write: VERIFY attention stores the block K/V and consensus advances "
                         "the lengths (write-then-truncate); append: separate kv_append launch")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
