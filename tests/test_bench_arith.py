"""The benchmark's algorithmic bytes and FLOPs, against their closed forms.

The roofline fractions divide these by measured times, so they are pinned
here on the CPU. Each expected value is written out from the definition,
not taken from the code under test:
  - attention reads each prefix K and V element once per (sequence, KV
    head): 2 tensors x Hkv x D x 2 bytes per prefix token, plus Q, the
    block's K/V and the output;
  - FLOPs are 4 x D x (visible keys summed over query rows and heads): all
    L + K keys in the DIFFUSION view, L + i + 1 for block row i in VERIFY;
  - consensus reads 4 x V bytes per row.
"""
import os
import tempfile

import pytest

import bench
from diffusion_draft_ar_b200 import workloads as W


@pytest.fixture(scope="module")
def q8():
    w = W.WORKLOADS["qwen3_8b"]
    return w, W.make_meta(w, seed=0)


def test_attention_bytes_qwen3_8b(q8):
    w, m = q8
    B, L, K, Hq, Hkv, D = 16, 8192, 32, 32, 8, 128
    kv = B * L * 2 * Hkv * D * 2          # 536,870,912
    q_out = 2 * B * K * Hq * D * 2        # Q in, O out: 4,194,304 each
    blk = B * K * Hkv * D * 2 * 2         # block K and V: 2,097,152
    assert kv + q_out + blk == 547_356_672
    assert bench.attn_bytes(w, m) == 547_356_672


def test_attention_flops_qwen3_8b(q8):
    w, m = q8
    B, L, K, Hq, D = 16, 8192, 32, 32, 128
    diff = 4 * D * B * Hq * K * (L + K)
    ver = 4 * D * B * Hq * (K * L + K * (K + 1) // 2)
    assert diff == 68_987_912_192 and ver == 68_857_888_768
    assert bench.attn_flops(w, m, "diffusion") == diff
    assert bench.attn_flops(w, m, "verify") == ver


def test_consensus_and_append_bytes(q8):
    w, m = q8
    R, V, B = 512, 151936, 16
    assert bench.consensus_bytes(w, m) == R * V * 4 + R * 4 * 2 + B * 8
    assert R * V * 4 == 311_164_928
    # one accepted row: read and write K and V for every KV head
    assert bench.append_bytes(w, 1) == 2 * 2 * w.Hkv * w.D * 2 == 8192


def test_traffic_file_follows_the_kernel_code(monkeypatch):
    """The bench reports DRAM traffic only while the committed ncu figures were
    taken on the current kernel code: a comment edit keeps them, a code edit
    drops them."""
    import json
    src = "// kernel source\n__global__ void k(int* p) {\n  p[0] = 1;  // store\n}\n"
    with tempfile.TemporaryDirectory() as d:
        k = os.path.join(d, "k.cuh")
        open(k, "w").write(src)
        h = bench.kernel_code_hash(k)
        s = os.path.join(d, "s.json")
        json.dump({"kernel_code_sha256_16": h, "dram_bytes_per_launch_full_size": 1234},
                  open(s, "w"))
        monkeypatch.setattr(bench, "ATTN_SRC", k)
        monkeypatch.setattr(bench, "TRAFFIC_FILE", s)
        assert bench.traffic_per_launch() == 1234
        open(k, "w").write("/* header */\n" + src.replace("// store", "// the store") + "\n\n")
        assert bench.traffic_per_launch() == 1234
        open(k, "w").write(src.replace("p[0] = 1;", "p[0] = 2;"))
        assert bench.traffic_per_launch() is None


def test_roofline_fractions():
    """Both fractions from their definitions: against the measured copy
    bandwidth, and against max(bytes / 8 TB/s, FLOPs / 2.25 PFLOP/s)."""
    nbytes, flops, us = 547_356_672, 68_987_912_192, 100.0
    d = bench.hbm_roofline(nbytes, flops, us)
    assert abs(d["gbs"] - 5473.56672) < 1e-6
    assert abs(d["frac"] - d["gbs"] / bench.peak_hbm()[0]) < 1e-12
    # bytes / 8 TB/s = 68.42 us dominates FLOPs / 2.25 PF = 30.66 us
    assert abs(d["frac_8tbs"] - (nbytes / 8e12) / 100e-6) < 1e-12
    # a compute-heavy case takes the FLOP term
    d2 = bench.hbm_roofline(1e6, 2.25e9, 10.0)
    assert abs(d2["frac_8tbs"] - (2.25e9 / 2.25e15) / 10e-6) < 1e-12
