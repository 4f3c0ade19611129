"""Real data parallelism (one process per GPU, symmetric-memory peer buffers, NCCL for the step
totals), run through torchrun with one rank per available GPU (this check uses one GPU)."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.gpu
def test_dist_zero_matches_oracle_one_rank_per_gpu():
    nproc = 1  # ranks must not share a GPU: their kernels wait on one another
    env = dict(os.environ, ZERO_DIST_N="100003", NCCL_NVLS_ENABLE="0",
               TORCH_SYMM_MEM_DISABLE_MULTICAST="1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node",
           str(nproc), "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "tests", "_dist_worker.py")]
    res = subprocess.run(["timeout", "-k", "30", "300"] + cmd, env=env, capture_output=True,
                         text=True)
    assert res.returncode == 0, res.stdout[-2000:] + res.stderr[-4000:]
    lines = [json.loads(x) for x in res.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == nproc
    for r in lines:
        assert r["flags_ok"] and r["overflow_seq"] == [0, 1, 0], r
        assert r["master_exact"] and r["exp_avg_sq_exact"] and r["replica_exact"], r
        assert r["sumsq_rel"] <= 1e-5, r


# ----------------------------------------------------------------------------- rank windows

def _run_windows(Nd, N, gdt, steps=3, inject=(2, 0, 7), dynamic=False):
    """Nd data-parallel ranks emulated in one process on one GPU, each with its own buffers laid
    out as dist.DistZero lays them out (full gradient and weight replicas, an S-element state
    shard rebased to global indices, its own workspace).  A step is every rank's
    zero_fused_window over its window with the step left open (rank 0 first; no kernel waits on
    another), the ranks' pending overflow flags combined with MAX and sums of squares with SUM
    into every workspace (what NCCL does across GPUs), then zero_end_step_flip and
    zero_repair_window per rank.  Compared with the CPU oracle element by element."""
    import numpy as np
    import torch

    import oracle
    import synth
    import zero_sharded_optimizer_03_b200 as zero
    from zero_sharded_optimizer_03_b200.dist import PENDING_FLAG_OFFSET, PENDING_SUMSQ_OFFSET
    from zero_sharded_optimizer_03_b200.dist import rank_window, shard_state

    dev = torch.device("cuda")
    s = torch.cuda.current_stream().cuda_stream
    sdt = synth.BF16 if gdt == zero.ZERO_BF16 else synth.FP16
    odt = oracle.BF16 if gdt == zero.ZERO_BF16 else oracle.FP16
    tdt = torch.bfloat16 if gdt == zero.ZERO_BF16 else torch.float16
    inf_bits = 0x7F80 if sdt == synth.BF16 else 0x7C00
    hp = dict(lr=1e-3, weight_decay=0.01, loss_scale=1024.0 if sdt == synth.FP16 else 1.0)
    sigma = 0.1024 if sdt == synth.FP16 else 1e-3
    chp = zero.hparams(**hp)
    n = max(N, 1)
    grads = [torch.zeros(n, dtype=tdt, device=dev) for _ in range(Nd)]
    params = [torch.zeros(n, dtype=torch.bfloat16, device=dev) for _ in range(Nd)]
    master0 = synth.fill_host(synth.NORMAL, synth.F32, synth.SEED, synth.MASTER_STREAM, N,
                              sigma=0.02)
    ranks = []
    for r in range(Nd):
        lo, hi, S = rank_window(N, Nd, r)
        views, bases = shard_state(S, lo, dev, torch)
        views["master"][0][:hi - lo].copy_(torch.from_numpy(master0[lo:hi]))
        ws = torch.zeros(zero.zero_workspace_bytes(), dtype=torch.uint8, device=dev)
        st = zero.zero_state_t()
        st.grad_dtype = gdt
        st.flags = zero.ZERO_FUSED | zero.ZERO_NO_TMA
        for q in range(Nd):
            st.grads[q] = grads[q].data_ptr()
            st.params[q] = params[q].data_ptr()
        for k in range(2):
            st.master[k] = bases["master"][k]
            st.exp_avg[k] = bases["exp_avg"][k]
            st.exp_avg_sq[k] = bases["exp_avg_sq"][k]
        st.workspace = ws.data_ptr()
        zero.zero_workspace_init(ws.data_ptr(), 0, s)
        if dynamic:  # every rank keeps the same scaler, driven by the combined overflow flag
            zero.zero_loss_scaler_init(ws.data_ptr(), 1024.0, 2.0, 0.5, 2, s)
        # the initial all-gather: every rank writes bf16 of its shard into every replica
        zero.zero_allgather(bases["master"][0], [p.data_ptr() for p in params], Nd, lo, hi,
                            zero.ZERO_GATE_ALWAYS, None, s)
        ranks.append(dict(lo=lo, hi=hi, views=views, ws=ws, st=st))
    S, Np, _ = oracle.partition(N, Nd)
    om = np.zeros(Np, np.float32)
    om[:N] = master0
    mm, vm = np.zeros(Np, np.float32), np.zeros(Np, np.float32)
    oreps = [oracle.f32_to_bf16(master0) for _ in range(Nd)]
    t, scale, good = 0, 1024.0, 0
    hpx = dict(hp, dynamic_scale=True, scale_interval=2, scale_growth=2.0, scale_backoff=0.5)
    for k in range(1, steps + 1):
        if dynamic:  # the gradients carry the scale in force when the step starts
            sigma = float(np.float32(1e-4 * scale))
        hg = [synth.fill_host(synth.NORMAL, sdt, synth.SEED, synth.grad_stream(k, q), N,
                              sigma=sigma) for q in range(Nd)]
        if inject is not None and k == inject[0] and N > inject[2]:
            hg[inject[1]][inject[2]] = inf_bits
        for q in range(Nd):
            grads[q][:N].view(torch.int16).copy_(torch.from_numpy(hg[q].view(np.int16)))
        for R in ranks:
            zero.zero_fused_window(Nd, R["lo"], R["hi"], R["st"], chp, False, s)
        flags = torch.stack([R["ws"][PENDING_FLAG_OFFSET:PENDING_FLAG_OFFSET + 4]
                             .view(torch.int32) for R in ranks])
        sums = torch.stack([R["ws"][PENDING_SUMSQ_OFFSET:PENDING_SUMSQ_OFFSET + 8]
                            .view(torch.float64) for R in ranks])
        fmax, ssum = flags.max(), sums.sum()
        for R in ranks:
            R["ws"][PENDING_FLAG_OFFSET:PENDING_FLAG_OFFSET + 4].view(torch.int32).copy_(fmax)
            R["ws"][PENDING_SUMSQ_OFFSET:PENDING_SUMSQ_OFFSET + 8].view(torch.float64).copy_(ssum)
        for R in ranks:
            zero.zero_end_step_flip(R["ws"].data_ptr(), s)
            zero.zero_repair_window(Nd, R["lo"], R["hi"], R["st"], s)
        if dynamic:
            t, ovf, ss, scale, good = oracle.zero12_step_ex(Nd, N, 0, odt, hg, om, mm, vm, oreps,
                                                            hpx, t, scale, good)
        else:
            t, ovf, ss = oracle.zero12_step(Nd, N, 0, odt, hg, om, mm, vm, oreps, hp, t)
        for R in ranks:
            res = zero.zero_read_result(R["ws"].data_ptr(), s)
            assert (res["overflow"], res["step"]) == (ovf, t), (k, res)
            if dynamic:
                assert (res["loss_scale"], res["good_steps"]) == (scale, good), (k, res)
            if not ovf:
                assert abs(res["grad_sumsq"] - ss) <= 1e-5 * ss
    torch.cuda.synchronize()
    for r, R in enumerate(ranks):
        live = zero.zero_read_result(R["ws"].data_ptr(), s)["live"]
        lo, hi = R["lo"], R["hi"]
        for name, want in (("master", om), ("exp_avg", mm), ("exp_avg_sq", vm)):
            got = R["views"][name][live][:hi - lo].cpu().numpy()
            assert got.tobytes() == want[lo:hi].tobytes(), "rank %d %s" % (r, name)
    for q in range(Nd):
        got = params[q][:N].view(torch.int16).cpu().numpy().view(np.uint16)
        assert got.tobytes() == oreps[q].tobytes(), "replica %d" % q
    return ranks


@pytest.mark.gpu
@pytest.mark.parametrize("Nd,N,gdt", [(2, 1_000_003, 0), (3, 100_003, 1), (8, 5_000_011, 0),
                                      (4, 5, 0), (5, 2_049, 1)])
def test_rank_windows_emulated_in_one_process_match_oracle(Nd, N, gdt):
    """The multi-rank window path with Nd > 1 on one GPU: ragged last windows, windows starting
    at indices that are not multiples of 8 (N = 1,000,003 over 2 ranks: the second window starts
    at 500,002), a rank that owns nothing (N = 5 over 4 ranks), fp16 and bf16, three steps with
    an overflow planted in rank 0's gradient on step 2 (every rank skips, then repairs its window
    of every replica).  Every element of every rank's shard and of every replica equals the
    oracle's."""
    ranks = _run_windows(Nd, N, gdt)
    if (Nd, N) == (2, 1_000_003):
        assert ranks[1]["lo"] == 500_002 and ranks[1]["lo"] % 8 != 0
    if (Nd, N) == (4, 5):
        assert ranks[3]["lo"] == ranks[3]["hi"] == 5


@pytest.mark.gpu
def test_rank_windows_with_dynamic_loss_scale_match_oracle():
    """The window path with the dynamic loss scaler: fp16 gradients carry each step's scale,
    every rank's workspace keeps a scaler, and the combined overflow flag (an inf in rank 0's
    gradient on step 2) backs it off on every rank alike; two clean steps grow it.  Five steps
    over 3 ranks, every element and every rank's scale sequence equal the oracle's."""
    _run_windows(3, 100_003, 1, steps=5, dynamic=True)


@pytest.mark.gpu
def test_single_finalized_window_matches_oracle_and_repairs():
    """zero_fused_window with finalize over the whole vector (one GPU, the step ended by the
    pass itself): three steps with an overflow on step 2; after the skip every replica is
    rewritten from the unchanged state, and every element equals the oracle's."""
    import numpy as np
    import torch

    import oracle
    import synth
    import zero_sharded_optimizer_03_b200 as zero
    Nd, N = 4, 300_007
    s = torch.cuda.current_stream().cuda_stream
    hp = dict(lr=1e-3, weight_decay=0.01, loss_scale=1.0)
    buf = zero.ZeroBuffers(2, Nd, N)
    master0 = synth.fill_host(synth.NORMAL, synth.F32, synth.SEED, synth.MASTER_STREAM, N,
                              sigma=0.02)
    buf.master[0][:N].copy_(torch.from_numpy(master0))
    buf.init_workspace(0)
    buf.sync_params_from_master()
    S, Np, _ = oracle.partition(N, Nd)
    om = np.zeros(Np, np.float32)
    om[:N] = master0
    mm, vm = np.zeros(Np, np.float32), np.zeros(Np, np.float32)
    oreps = [oracle.f32_to_bf16(master0) for _ in range(Nd)]
    t = 0
    for k in (1, 2, 3):
        hg = [synth.fill_host(synth.NORMAL, synth.BF16, synth.SEED, synth.grad_stream(k, q), N,
                              sigma=1e-3) for q in range(Nd)]
        if k == 2:
            hg[1][4321] = 0x7F80
        for q in range(Nd):
            buf.grads[q].view(torch.int16).copy_(torch.from_numpy(hg[q].view(np.int16)))
        zero.zero_fused_window(Nd, 0, N, buf.state, zero.hparams(**hp), True, s)
        t, ovf, ss = oracle.zero12_step(Nd, N, 0, oracle.BF16, hg, om, mm, vm, oreps, hp, t)
        res = buf.result()
        assert (res["overflow"], res["step"]) == (ovf, t) == (int(k == 2), (1, 1, 2)[k - 1])
        for q in range(Nd):  # the replicas hold the committed weights after every step
            got = buf.params[q].view(torch.int16).cpu().numpy().view(np.uint16)
            assert got.tobytes() == oreps[q].tobytes(), (k, q)
    live = buf.live()
    assert buf.master[live].cpu().numpy().tobytes() == om.tobytes()
    assert buf.exp_avg_sq[live].cpu().numpy().tobytes() == vm.tobytes()


def _random_window_cases(n_cases=12, seed=2028):
    import numpy as np
    rng = np.random.default_rng(seed)
    cases = []
    for k in range(n_cases):
        Nd = int(rng.choice([2, 3, 4, 5, 7, 8]))
        N = int(rng.choice([9, 1001, 65_537, 200_003, 524_291]))
        gdt = int(rng.choice([0, 1]))
        dynamic = bool(gdt == 1 and rng.random() < 0.5)
        rank = int(rng.integers(0, Nd))
        index = int(rng.integers(0, N))
        inject = (2, rank, index) if rng.random() < 0.7 else None
        cases.append((k, Nd, N, gdt, dynamic, inject))
    return cases


@pytest.mark.gpu
@pytest.mark.parametrize("case", _random_window_cases(), ids=lambda c: "case%d" % c[0])
def test_randomized_rank_windows_against_oracle(case):
    """Seeded random rank-window cases (Nd, N, gradient dtype, dynamic loss scale, an overflow in
    a random rank's gradient at a random index or none), four steps each, every element of every
    rank's shard and replica against the oracle."""
    k, Nd, N, gdt, dynamic, inject = case
    _run_windows(Nd, N, gdt, steps=4, inject=inject, dynamic=dynamic)
