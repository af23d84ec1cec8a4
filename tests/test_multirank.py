"""World-size-2 checks of bench.py's multi-rank host logic on CPU (gloo): the slowest rank
sets the time, the job value counts every rank's queries, ranks draw different batches."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms = [10.0, 25.0][rank]
    got = bench.max_over_ranks(ms, dist, torch.device("cpu"))
    dist.barrier()
    q.put((rank, got, bench.rank_seed(1234, rank)))
    dist.destroy_process_group()


def test_two_rank_max_and_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert res[0][1] == res[1][1] == 25.0
    assert res[0][2] != res[1][2]


def test_job_throughput_weak_scaling():
    import bench
    assert bench.job_throughput(32, 1, 10, 1000.0) == 320.0
    assert bench.job_throughput(32, 8, 10, 1000.0) == 2560.0
    assert bench.max_over_ranks(3.0, None, None) == 3.0


def test_bench_spawns_ranks_for_gpus_n():
    """bench.py --gpus 2 outside a launcher starts two ranks itself (torch.distributed.run on
    127.0.0.1); the reference arm runs on rank 0 only (host cores, no GPU needed) and
    reports the job's rank count."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2",
                        "--impl", "reference", "--workload", "decode_full_b1_ctx4k",
                        "--steps", "1", "--warmup", "0", "--cpu-budget", "1"],
                       capture_output=True, text=True, timeout=600, env=env, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, r.stdout
    assert lines[0]["n_gpus"] == 2 and lines[0]["impl"] == "reference"
    assert lines[0]["cpu_baseline"]["cores"] == (os.cpu_count() or 1)


def test_bench_rejects_gpus_world_mismatch():
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2"],
                       capture_output=True, text=True, timeout=300, env=env, cwd=root)
    assert r.returncode != 0 and "WORLD_SIZE" in r.stderr
