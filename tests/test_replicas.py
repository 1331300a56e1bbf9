"""Host logic of the multi-GPU path (replicas only: every rank runs the whole layer on its
own batch; the only collective is the max over ranks of the step time). Run on CPU with the
gloo backend, world size 2."""
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, results):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.reduce_step_time(2.0 + rank, world)  # rank 1 is the slow one
        results[rank] = (ms, bench.job_throughput(8192, world, ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_step_time_is_max_over_ranks_and_value_counts_all_ranks():
    port = 29500 + os.getpid() % 1000
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_rank_main, args=(2, port, results), nprocs=2, start_method="spawn",
                           join=True)
        res = dict(results)
    assert res[0][0] == res[1][0] == 3.0
    assert res[0][1] == pytest.approx(2 * 8192 / 3e-3)


def test_single_rank_needs_no_collective():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.reduce_step_time(1.5, 1) == 1.5
    assert bench.job_throughput(4096, 1, 0.5) == pytest.approx(4096 / 0.5e-3)


def test_reference_arm_runs_on_rank0_only():
    """Under torchrun the reference arm's non-zero ranks exit 0 without output or work."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "1", "--workload", "tiny"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
