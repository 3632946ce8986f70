"""The benchmark's multi-rank host logic on CPU (gloo, world size 2).

With --gpus N every rank decodes its own batch (weak scaling, no data-path
collective).  The only cross-rank steps are a barrier and the max over the
ranks' device times; this checks both, and the whole-job value, without a
GPU.
"""

from __future__ import annotations

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        t = [0.25, 0.40][rank]
        bench.dist_barrier(world)
        m = bench.max_over_ranks(t, world, "cpu")
        v = bench.aggregate_value(512 * 100, world, m)
        q.put((rank, m, v))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get() for _ in range(2))
    for rank, m, v in res:
        assert m == pytest.approx(0.40)
        assert v == pytest.approx(512 * 100 * 2 / 0.40)


def test_single_rank_helpers():
    import bench
    assert bench.max_over_ranks(1.5, 1, "cpu") == 1.5
    assert bench.aggregate_value(1000, 1, 0.5) == 2000


def test_world_plan():
    import bench
    assert bench.world_plan(1, {}) == "run"
    assert bench.world_plan(4, {}) == "spawn"
    assert bench.world_plan(2, {"WORLD_SIZE": "2"}) == "run"
    with pytest.raises(SystemExit):
        bench.world_plan(8, {"WORLD_SIZE": "1"})
    with pytest.raises(SystemExit):
        bench.world_plan(0, {})
    cmd = bench.spawn_command(2, ["--gpus", "2"], 29999)
    assert "--nproc-per-node=2" in cmd and cmd[-2:] == ["--gpus", "2"]


def test_gpus_flag_launches_that_many_ranks():
    # --gpus 2 with no launcher: bench.py starts 2 local ranks itself.  The
    # oracle arm runs on CPU (gloo), so the launched world size shows in its
    # line without a GPU.
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    env["DL_BENCH_BACKEND"] = "gloo"
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--impl",
                          "reference", "--workload", "gdn_tiny", "--steps", "2", "--warmup", "3"],
                         env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(x) for x in out.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    assert lines[0]["n_gpus"] == 2 and lines[0]["impl"] == "reference"
