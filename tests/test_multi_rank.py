"""The bench's multi-GPU logic on CPU: independent replicas (no data-path
collective), a barrier, the max of per-rank times, and the whole-job value,
with two gloo ranks on 127.0.0.1."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench

    dist = bench.dist_init(world, "gloo")
    bench.barrier(dist)
    my_time = 0.5 + rank          # rank 1 is the slowest
    t = bench.max_over_ranks(my_time, dist)
    value = bench.aggregate_value(1_000_000, 10, world, t)
    bench.barrier(dist)
    dist.destroy_process_group()
    q.put((rank, t, value))


def test_replicas_take_max_time_and_sum_work():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, t, value in got:
        assert t == pytest.approx(1.5)                       # max over ranks
        assert value == pytest.approx(1_000_000 * 10 * 2 / 1.5 / 1e9)   # all ranks' bytes / slowest time


def test_reference_arm_two_ranks_rank0_only():
    """--impl reference under torchrun with 2 ranks: rank 0 prints the one JSON
    line, rank 1 exits 0 without work."""
    env = dict(os.environ, MASTER_ADDR="127.0.0.1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--workload", "m_skinny"]
    proc = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert proc.returncode == 0, proc.stderr[-2000:]
    lines = [ln for ln in proc.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
