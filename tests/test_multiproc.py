"""The multi-process host logic of bench.py on CPU: two gloo ranks.

Each rank runs its own batch (different seeds, same shapes: weak scaling with no
exchange on the data path) and the job's time is the maximum over ranks.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        w = bench.rank_workload("c4", rank, batch=3)
        mine = 10.0 + 7.5 * rank
        got = bench.max_over_ranks(mine, "cpu")
        q = torch.from_numpy(w.query_bits().astype(np.int64).ravel()[:64])
        first = [torch.zeros_like(q) for _ in range(world)]
        dist.all_gather(first, q)  # test plumbing only: compare the ranks' inputs
        out[rank] = (got, w.seed, w.B, w.Hq, w.D, bool(torch.equal(first[0], first[1])))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling_and_max_time():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    r0, r1 = out[0], out[1]
    assert r0[0] == r1[0] == 17.5             # max over ranks, the same on every rank
    assert r0[1] != r1[1]                     # independent batches
    assert r0[2:5] == r1[2:5] == (3, 16, 128)  # same shapes per rank
    assert r0[5] is False                     # different query data


def test_single_process_max_is_identity():
    import bench
    assert bench.max_over_ranks(3.25, "cpu") == 3.25


def test_reference_arm_prints_the_contract_line():
    """bench.py --impl reference (the CPU oracle) prints one JSON line with the contract keys."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--config", "c0",
                        "--steps", "1", "--warmup", "3", "--cpu-seconds", "2"], capture_output=True, text=True, timeout=300, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    # c0 has two (sequence, kv head) units: one worker process each on a host with two or more cores
    assert d["cpu_baseline"]["cores"] == min(2, os.cpu_count()) and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["cpu_baseline"]["one_thread"] > 0 and d["cpu_baseline"]["nproc"] == os.cpu_count()
