"""The N > 1 host path of bench.py on CPU: world-size-2 gloo process groups
(no GPU).  The layer shards by token batches with no collective on the data
path, so the only cross-rank step is the max-over-ranks timing."""
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from tests.conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    v = bench.max_over_ranks(1.5 * (rank + 1), "cpu")
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, v))


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=5) for _ in range(2))
    assert got == {0: 3.0, 1: 3.0}


def test_max_over_ranks_without_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5) == 2.5


def test_reference_arm_on_a_non_zero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_line_on_rank_zero():
    """The reference arm (the fp64 oracle on host cores) prints one JSON line
    with the contract's keys, on the tiny layer so that it takes seconds."""
    import json
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "tiny", "--steps", "2", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["steps"] == 2 and d["warmup"] >= 3 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"]


def test_weight_bytes_streamed_counts_the_activated_experts():
    import numpy as np
    sys.path.insert(0, ROOT)
    import bench
    from mixture_experts_layer_56_b200 import synthetic as S
    wl = S.WORKLOADS["decode1"]
    counts = np.zeros(wl.n_routed, dtype=np.int64)
    counts[[3, 7, 11, 20, 40, 63]] = 1  # six routed experts hit by one token
    per_expert = wl.d * wl.inter * 2  # bf16 bytes of one d x I matrix
    assert bench.weight_bytes_streamed(wl, counts, gate_up_only=True) == (6 + 2) * 2 * per_expert
    assert bench.weight_bytes_streamed(wl, counts) == (6 + 2) * 3 * per_expert + \
        wl.n_routed * wl.d * 2
