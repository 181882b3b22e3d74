"""The multi-rank logic of bench.py on CPU: two gloo ranks, as torchrun would
launch them, agree on the slowest rank's time; whole-job throughput counts
every replica; the reference arm's non-zero ranks exit without work."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        vals = bench.max_over_ranks(dist, [10.0 + rank, 5.0 * (world - rank)])
        out.put((rank, vals))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got[0] == got[1] == [11.0, 10.0]


def test_step_throughput_counts_every_replica():
    sys.path.insert(0, ROOT)
    import bench
    gbs1, sps1 = bench.step_throughput(1, 100, 250.0)
    gbs4, sps4 = bench.step_throughput(4, 100, 250.0)
    assert gbs4 == pytest.approx(4 * gbs1) and sps4 == pytest.approx(4 * sps1)
    assert sps1 == pytest.approx(400.0)
    assert gbs1 == pytest.approx(bench.STEP_GEMV_BYTES * 400.0 / 1e9)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "3", "--warmup", "3", "--gpus", "2"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
