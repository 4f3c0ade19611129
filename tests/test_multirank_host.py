"""Host logic of the multi-GPU benchmark path, run as two gloo ranks on the CPU.

On N GPUs bench.py runs one independent replica of the workload per GPU (the Nd simulated
ranks live inside each GPU; there is no data-path collective).  What crosses ranks is the
barrier and the max-over-ranks timing; the whole-job rate is the sum over replicas."""
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    import datetime
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    dist.barrier()
    got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 3.5], dist, "cpu")
    out[rank] = got
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world, port = 2, 29611
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert res[0] == res[1] == [2.0, 10.0, 3.5]


def test_whole_job_rate_is_weak_scaling_sum():
    import bench
    one = bench.whole_job_rate(1_000_000, 1, 2.0)
    assert one == pytest.approx(5e8)
    assert bench.whole_job_rate(1_000_000, 8, 2.0) == pytest.approx(8 * one)
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--gpus", "2", "--steps", "1", "--warmup", "3"], env=env,
                         capture_output=True, text=True, timeout=120)
    assert res.returncode == 0 and res.stdout.strip() == ""


def _dist_worker(rank, world, port, out):
    import datetime
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    from zero_sharded_optimizer_03_b200.dist import combine_step_totals, rank_window
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    ws = torch.zeros(16, dtype=torch.uint8)  # the pending totals sit at bytes 4 and 8
    flag = ws[4:8].view(torch.int32)
    sumsq = ws[8:16].view(torch.float64)
    flag.fill_(1 if rank == 1 else 0)
    sumsq.fill_(0.25 * (rank + 1))
    combine_step_totals(flag, sumsq)
    out[rank] = (int(flag.item()), float(sumsq.item()),
                 [rank_window(1_000_003, world, q) for q in range(world)])
    dist.destroy_process_group()


def test_dist_step_totals_and_windows_two_gloo_ranks():
    world, port = 2, 29623
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_dist_worker, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert res[0][0] == res[1][0] == 1          # any rank's overflow skips every rank
    assert res[0][1] == res[1][1] == 0.75       # sums of squares add up
    windows = res[0][2]
    assert windows == [(0, 500002, 500002), (500002, 1000003, 500002)]
