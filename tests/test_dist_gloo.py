"""The multi-rank host logic on CPU with two gloo ranks: joining, barrier, the
max-over-ranks timing reduction, per-rank seeds and sharding."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from diffusion_draft_ar_b200 import dist as D


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    try:
        w, r, _ = D.init(backend="gloo", timeout_s=60)
        D.barrier(w)
        t = D.max_over_ranks(10.0 + r, w, device="cpu")
        seeds = D.rank_seed(0, r)
        sh = list(D.shard(10, r, w))
        D.barrier(w)
        D.finish(w)
        q.put((r, w, t, seeds, sh))
    except Exception as e:  # pragma: no cover - reported to the parent
        q.put((rank, "error", repr(e), None, None))


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, t0, s0, sh0), (r1, w1, t1, s1, sh1) = res
    assert w0 == w1 == 2
    assert t0 == t1 == 11.0          # both ranks see the slowest rank's time
    assert s0 != s1                  # each rank draws its own batch
    assert sorted(sh0 + sh1) == list(range(10)) and not set(sh0) & set(sh1)


def test_single_rank_helpers():
    assert D.max_over_ranks(3.5, 1) == 3.5
    assert list(D.shard(7, 0, 1)) == list(range(7))
    assert D.weak_scaling_throughput(16, 2.0, 4) == pytest.approx(4 * 16 / 2e-3)
