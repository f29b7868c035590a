"""Multi-rank host logic of bench.py on CPU: two gloo ranks combine their
device times with a max and report whole-job weak-scaling throughput."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench

    assert bench.dist_env() == (world, rank, rank)
    bench.init_dist(world, "gloo")
    try:
        mx = bench.max_over_ranks(times[rank], world)
        value = bench.weak_scaling_value(1e12, world, mx)
        dist.barrier()
        q.put((rank, mx, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_weak_scaling():
    world = 2
    times = [80.0, 95.5]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, mx, value in got:
        assert mx == max(times)
        # 2 ranks x 1 TFLOP each in 95.5 ms
        assert value == pytest.approx(2 * 1e12 / 0.0955 / 1e12)


def test_single_rank_is_identity():
    import bench

    assert bench.max_over_ranks(12.5, 1) == 12.5
    assert bench.weak_scaling_value(4e12, 1, 1000.0) == pytest.approx(4.0)


def test_bench_gpus_flag_launches_that_many_ranks():
    """`python bench.py --gpus 2` re-executes itself under
    torch.distributed.run with two local ranks (127.0.0.1); rank 0 alone
    prints the line of the reference arm (here on the tiny workload, CPU
    only) with n_gpus = 2, the other rank exits 0 without work."""
    import json
    import subprocess
    import sys

    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "0", "--cpu-seconds", "0.5"],
                       capture_output=True, text=True, timeout=240, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, r.stdout
    assert lines[0]["impl"] == "reference" and lines[0]["n_gpus"] == 2


def test_bench_refuses_a_world_size_other_than_gpus():
    import subprocess
    import sys

    env = dict(os.environ, WORLD_SIZE="3", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference",
                        "--workload", "tiny", "--steps", "1"], capture_output=True, text=True, timeout=120,
                       env=env, cwd=ROOT)
    assert r.returncode == 2 and "WORLD_SIZE=3" in r.stderr
