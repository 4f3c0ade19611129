"""Host logic of the multi-GPU paths, run as two gloo ranks on the CPU.

On N GPUs bench.py runs the real data-parallel step (one rank per GPU, the fused kernel over
peer memory, NCCL for the step totals: zero_sharded_optimizer_03_b200.dist) for flat ZeRO-1/2
workloads, and one independent replica per GPU for the others.  These tests cover what crosses
ranks without a GPU: the max-over-ranks timing, the rank windows, the MAX/SUM combination of the
step totals and the order and arguments of DistZero.step's calls (device calls stubbed)."""
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


def _dist_step_worker(rank, world, port, N, out):
    """One rank of DistZero over gloo with the device entry points replaced by recorders."""
    import datetime
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    from zero_sharded_optimizer_03_b200 import dist as zd
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))

    class Handle:  # every rank's address of a buffer, as symmetric memory's rendezvous gives
        def __init__(self, t):
            ptrs = [None] * world
            dist.all_gather_object(ptrs, t.data_ptr())
            self.buffer_ptrs = ptrs

    class FakeSymm:
        empty = staticmethod(lambda n, dtype, device: torch.zeros(n, dtype=dtype, device=device))
        rendezvous = staticmethod(lambda t, name: Handle(t))

    calls = []
    step_no = [0]

    def fused_window(Nd, lo, hi, st, hp, finalize, s):
        step_no[0] += 1
        calls.append(("fused_window", Nd, lo, hi, bool(finalize),
                      [st.grads[q] for q in range(Nd)], [st.params[q] for q in range(Nd)],
                      [st.master[k] for k in range(2)], [st.exp_avg_sq[k] for k in range(2)]))
        # this rank's pending totals, as the kernel leaves them: rank 1 overflows on step 2
        dz.flag.fill_(1 if (rank == 1 and step_no[0] == 2) else 0)
        dz.sumsq.fill_(0.25 * (rank + 1))

    def end_step_flip(ws, s):  # the combined totals must be in place when the step ends
        calls.append(("end_step_flip", int(dz.flag.item()), float(dz.sumsq.item())))

    def repair_window(Nd, lo, hi, st, s):
        calls.append(("repair_window", Nd, lo, hi))

    zd.zero_fused_window = fused_window
    zd.zero_end_step_flip = end_step_flip
    zd.zero_repair_window = repair_window
    zd.zero_workspace_init = lambda ws, t, s: calls.append(("init", t))
    zd.zero_allgather = lambda *a: calls.append(("allgather", a[2], a[3], a[4]))
    orig_barrier = zd.DistZero.barrier
    zd.DistZero.barrier = lambda self: (calls.append(("barrier",)), orig_barrier(self))
    dz = zd.DistZero(N, device="cpu", symm=FakeSymm)
    dz.init(0)
    dz.publish_weights = lambda: None  # needs zero_read_result (a device read)
    hp = object()
    for _ in range(3):
        dz.step(hp)
    out[rank] = dict(window=(dz.lo, dz.hi, dz.S), calls=calls,
                     grad=dz.grad.data_ptr(), param=dz.param.data_ptr(),
                     master=[m.data_ptr() for m in dz.master],
                     exp_avg_sq=[v.data_ptr() for v in dz.exp_avg_sq])
    dist.destroy_process_group()


def test_dist_step_call_order_and_arguments_two_gloo_ranks():
    """DistZero.step on two gloo ranks with the device calls stubbed: every rank runs barrier ->
    fused pass over its own window (step left open, peers' buffers as operands, state rebased to
    global indices) -> MAX/SUM combine of the step totals -> end of step -> repair of its window
    -> barrier, and an overflow on one rank reaches every rank before the step ends."""
    world, port, N = 2, 29641, 1_000_003
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_dist_step_worker, args=(world, port, N, out), nprocs=world,
                           join=True, start_method="spawn")
        res = dict(out)
    S = (N + world - 1) // world
    grads = [res[q]["grad"] for q in range(world)]
    params = [res[q]["param"] for q in range(world)]
    for rank in range(world):
        r = res[rank]
        lo, hi = min(rank * S, N), min((rank + 1) * S, N)
        assert r["window"] == (lo, hi, S)
        calls = r["calls"]
        assert calls[0] == ("init", 0)
        steps = calls[1:]
        assert len(steps) == 3 * 5
        for k in range(3):
            b0, fw, flip, rep, b1 = steps[5 * k:5 * k + 5]
            assert b0 == ("barrier",) and b1 == ("barrier",)
            name, Nd, flo, fhi, finalize, g, p, master, vsq = fw
            assert (name, Nd, flo, fhi, finalize) == ("fused_window", world, lo, hi, False)
            assert g == grads and p == params  # every rank's gradient and weight replica
            assert master == [m - 4 * lo for m in r["master"]]  # base + lo = first element
            assert vsq == [v - 4 * lo for v in r["exp_avg_sq"]]
            assert flip == ("end_step_flip", 1 if k == 1 else 0, 0.25 + 0.5)
            assert rep == ("repair_window", world, lo, hi)
