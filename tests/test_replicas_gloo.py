"""The multi-GPU path of the benchmark on CPU: two gloo ranks.

The layer shards over tokens with no exchange, so N GPUs run N independent
replicas; the only collectives are the barriers and the max of the per-rank
step times.  These tests run that host logic with world size 2 on the CPU:
every rank takes the same collective steps, the slowest rank sets the step
time, the whole-job throughput counts every rank's tokens, each rank gets its
own batch, and a rank that fails before a collective makes the other rank's
collective end with an error instead of hanging.
"""
import os
import socket
import sys
from datetime import timedelta

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port, timeout_s=60):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=timedelta(seconds=timeout_s))


def _worker_max(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    _init(rank, world, port)
    try:
        r, w, lr = bench.rank_env()
        assert (r, w, lr) == (rank, world, rank)
        step_ms = [1.0 + rank, 5.0 - rank]           # rank 0 slower on the 2nd value
        dist.barrier()
        got = bench.max_over_ranks(step_ms, world)
        dist.barrier()
        q.put((rank, got, bench.aggregate_tokens_per_s(128, world, got[0]),
               bench.replica_seed(rank)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_max_and_count_all_tokens():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker_max, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, got, tps, seed in res:
        assert got == [2.0, 5.0]                      # max over ranks, element-wise
        assert tps == pytest.approx(2 * 128 / 2e-3)    # both ranks' tokens / slowest time
    assert [r[3] for r in res] == [0, 1]              # distinct batches per rank


def _worker_fail(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    _init(rank, world, port, timeout_s=5)
    if rank == 1:
        # this rank fails between steps, before the next collective
        os._exit(3)
    try:
        bench.max_over_ranks([1.0], world)
        q.put("returned")
    except Exception as e:  # the surviving rank's collective errors out
        q.put("error:" + type(e).__name__)


def test_failed_rank_ends_the_other_ranks_collective_with_an_error():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker_fail, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert procs[1].exitcode == 3
    msg = q.get(timeout=30)
    assert msg.startswith("error:")


def test_bench_starts_the_ranks_it_is_asked_for():
    """`bench.py --gpus 2` without torchrun starts two ranks itself (through
    torch.distributed.run); the launcher check joins them over gloo without any
    CUDA work and reports both."""
    import json
    import subprocess
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        env.pop(k, None)
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                          "--launcher-check"], capture_output=True, text=True, timeout=300,
                         env=env, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [json.loads(x) for x in res.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    rec = lines[0]
    assert rec["launcher_check"] and rec["n_gpus"] == 2 and rec["gpus_requested"] == 2
    assert rec["ranks"] == [0, 1] and rec["pids"] == 2


def test_bench_refuses_a_world_size_other_than_gpus():
    import subprocess
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                          "--launcher-check"], capture_output=True, text=True, timeout=300,
                         env=env, cwd=ROOT)
    assert res.returncode != 0 and "--gpus 2 but 1 ranks" in res.stderr
