"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle, element by element.

Tolerances (fixed by the method's precision: fp32 state, bf16 weights): fp32 master / m / v
within max relative error 1e-6 (expected 0: both sides use the same fp32 operation order and
rank-order summation), bf16 weights within 1 ulp (expected 0), overflow flag, step counter
and shard / padding layout exact, sum of squares within 1e-5 relative (summation order
differs).  Small and ragged sizes are compared in full; the five workloads at full size are
compared on sampled elements the oracle evaluates one by one (plus properties that hold at
any size).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import zero_sharded_optimizer_03_b200 as zero
from _gpu import (HP_ADAM_LR1E3, HP_ADAMW_GPT2, HP_ADAMW_FP16_LS1024, HP_ADAMW_ZERO3, HP_ADAMW_WIDE, LLAMA7B_LAYER, SEED, SampledOracle, at,
                  assert_bf16_close, assert_f32_close, boundaries, f32, fill, free, grads_at,
                  put_bits, sample_indices, stream, u16)

pytestmark = pytest.mark.gpu

DT = {zero.ZERO_BF16: (oracle.BF16, synth.BF16), zero.ZERO_FP16: (oracle.FP16, synth.FP16)}


def _init_state(buf, N, t0=0, m_kind=synth.ZERO, v_kind=synth.ZERO, m_sigma=0.0, v_sigma=0.0):
    fill(buf.master[0], synth.NORMAL, synth.F32, synth.MASTER_STREAM, n=N, sigma=0.02)
    if m_kind != synth.ZERO:
        fill(buf.exp_avg[0], m_kind, synth.F32, synth.M_STREAM, n=N, sigma=m_sigma)
        fill(buf.exp_avg_sq[0], v_kind, synth.F32, synth.V_STREAM, n=N, sigma=v_sigma)
    buf.init_workspace(t0)
    buf.sync_params_from_master()


def _host_state(N, Np, m_kind=synth.ZERO, v_kind=synth.ZERO, m_sigma=0.0, v_sigma=0.0):
    p = np.zeros(Np, np.float32)
    m = np.zeros(Np, np.float32)
    v = np.zeros(Np, np.float32)
    p[:N] = synth.fill_host(synth.NORMAL, synth.F32, SEED, synth.MASTER_STREAM, N, sigma=0.02)
    if m_kind != synth.ZERO:
        m[:N] = synth.fill_host(m_kind, synth.F32, SEED, synth.M_STREAM, N, sigma=m_sigma)
        v[:N] = synth.fill_host(v_kind, synth.F32, SEED, synth.V_STREAM, N, sigma=v_sigma)
    return p, m, v


def _compare_full(buf, om, mm, vm, oreps, t, ss, tag):
    res = buf.result()
    assert res["step"] == t, (tag, res)
    live = buf.live()
    assert_f32_close(f32(buf.master[live]), om, tag + " master")
    assert_f32_close(f32(buf.exp_avg[live]), mm, tag + " exp_avg")
    assert_f32_close(f32(buf.exp_avg_sq[live]), vm, tag + " exp_avg_sq")
    for r, rep in enumerate(oreps):
        assert_bf16_close(u16(buf.params[r]), rep, "%s replica %d" % (tag, r))
    if ss is not None and ss > 0:
        assert abs(res["grad_sumsq"] - ss) <= 1e-5 * ss, (res["grad_sumsq"], ss)
    return res


# ----------------------------------------------------------------------------- generator

@pytest.mark.parametrize("kind,dtype", [(synth.NORMAL, synth.BF16), (synth.NORMAL, synth.FP16),
                                        (synth.NORMAL, synth.F32), (synth.ABS, synth.F32),
                                        (synth.SQUARE, synth.F32), (synth.HEAVY, synth.BF16)])
def test_device_generator_matches_host(kind, dtype):
    n, first = 300_001, 12_345
    tdt = {synth.BF16: torch.bfloat16, synth.FP16: torch.float16, synth.F32: torch.float32}[dtype]
    t = torch.empty(n, dtype=tdt, device="cuda")
    fill(t, kind, dtype, 77, sigma=1e-3, tail_sigma=1.0, first=first)
    want = synth.fill_host(kind, dtype, SEED, 77, n, sigma=1e-3, tail_sigma=1.0, first=first)
    got = u16(t) if dtype != synth.F32 else t.cpu().numpy()
    assert got.tobytes() == want.tobytes()


# ----------------------------------------------------------------------------- config 1, full

@pytest.mark.parametrize("flags", [zero.ZERO_FUSED, zero.ZERO_TWO_PASS])
@pytest.mark.parametrize("stage", [1, 2])
def test_zero2_1m_nd4_single_step_full(stage, flags):
    """N = 1,000,003 (padded to ceil(N/4)), Nd = 4, bf16 grads ~N(0,1e-3) per rank, master
    ~N(0,0.02), m = v = 0, Adam lr 1e-3 (wd 0), step 1: every element compared."""
    Nd, N = 4, 1_000_003
    buf = zero.ZeroBuffers(stage, Nd, N, flags=flags)
    _init_state(buf, N)
    S, Np, pad = oracle.partition(N, Nd)
    assert (buf.Np, pad) == (Np, 1)
    om, mm, vm = _host_state(N, Np)
    grads = [synth.fill_host(synth.NORMAL, synth.BF16, SEED, synth.grad_stream(1, r), N,
                             sigma=1e-3) for r in range(Nd)]
    for r in range(Nd):
        fill(buf.grads[r], synth.NORMAL, synth.BF16, synth.grad_stream(1, r), sigma=1e-3)
    buf.step(zero.hparams(**HP_ADAM_LR1E3))
    oreps = [np.zeros(N, np.uint16) for _ in range(Nd)]
    t, ovf, ss = oracle.zero12_step(Nd, N, 0, oracle.BF16, grads, om, mm, vm, oreps, HP_ADAM_LR1E3, 0)
    res = _compare_full(buf, om, mm, vm, oreps, t, ss, "1M Nd=4")
    assert res["overflow"] == 0 and res["skipped"] == 0
    live = buf.live()
    # every rank's shard view holds exactly that rank's elements; the padding stays zero
    mast = f32(buf.master[live])
    for r in range(Nd):
        lo, hi = r * S, min((r + 1) * S, N)
        assert mast[lo:hi].tobytes() == om[lo:hi].tobytes()
    assert (mast[N:] == 0).all() and (f32(buf.exp_avg[live])[N:] == 0).all()
    # step 1 of Adam moves every weight by at most lr
    assert np.abs(mast[:N] - _host_state(N, Np)[0][:N]).max() <= 1e-3 * (1 + 1e-6)
    del buf
    free()


# ----------------------------------------------------------------------------- small / ragged

CASES = [(0, 4), (1, 1), (1, 4), (7, 3), (8, 8), (9, 2), (15, 64), (17, 5), (1000, 3),
         (4097, 8), (65_537, 7), (262_147, 16)]


@pytest.mark.parametrize("N,Nd", CASES)
@pytest.mark.parametrize("gdt", [zero.ZERO_BF16, zero.ZERO_FP16])
@pytest.mark.parametrize("flags,bucket", [(zero.ZERO_FUSED, 0), (zero.ZERO_FUSED, 1001),
                                          (zero.ZERO_FUSED | zero.ZERO_FORCE_TMA, 0),
                                          (zero.ZERO_FUSED | zero.ZERO_FORCE_TMA, 5000),
                                          (zero.ZERO_TWO_PASS, 0), (zero.ZERO_TWO_PASS, 777)])
def test_small_ragged_three_steps(N, Nd, gdt, flags, bucket):
    odt, sdt = DT[gdt]
    hp = dict(HP_ADAMW_FP16_LS1024) if gdt == zero.ZERO_FP16 else dict(HP_ADAMW_GPT2)
    sigma = 1e-4 * 1024 if gdt == zero.ZERO_FP16 else 1e-3
    buf = zero.ZeroBuffers(2, Nd, N, grad_dtype=gdt, flags=flags)
    _init_state(buf, N)
    S, Np, _ = oracle.partition(N, Nd)
    om, mm, vm = _host_state(N, Np)
    oreps = [np.zeros(N, np.uint16) for _ in range(Nd)]
    t = 0
    ss = None
    for k in range(1, 4):
        grads = [synth.fill_host(synth.NORMAL, sdt, SEED, synth.grad_stream(k, r), N,
                                 sigma=sigma) for r in range(Nd)]
        for r in range(Nd):
            if N:
                fill(buf.grads[r], synth.NORMAL, sdt, synth.grad_stream(k, r), n=N, sigma=sigma)
        buf.step(zero.hparams(**hp), bucket=bucket)
        t, ovf, ss = oracle.zero12_step(Nd, N, bucket, odt, grads, om, mm, vm, oreps, hp, t)
    _compare_full(buf, om, mm, vm, oreps, t, ss, "N=%d Nd=%d" % (N, Nd))
    del buf
    free()


def test_unaligned_views_take_the_scalar_path():
    """Buffers that start 2 or 4 bytes past a 16-byte boundary are legal and give the same
    results as aligned ones."""
    Nd, N = 3, 5003
    hp = dict(HP_ADAMW_GPT2)
    S, Np, _ = oracle.partition(N, Nd)
    big = [torch.zeros(N + 1, dtype=torch.bfloat16, device="cuda") for _ in range(2 * Nd)]
    st_big = [torch.zeros(Np + 1, dtype=torch.float32, device="cuda") for _ in range(6)]
    grads = [b[1:] for b in big[:Nd]]
    reps = [b[1:] for b in big[Nd:]]
    states = [b[1:] for b in st_big]
    ws = torch.zeros(zero.zero_workspace_bytes(), dtype=torch.uint8, device="cuda")
    st = zero.zero_state_t()
    st.grad_dtype = zero.ZERO_BF16
    st.flags = zero.ZERO_FUSED
    for r in range(Nd):
        st.grads[r] = grads[r].data_ptr()
        st.params[r] = reps[r].data_ptr()
    for k in range(2):
        st.master[k] = states[k].data_ptr()
        st.exp_avg[k] = states[2 + k].data_ptr()
        st.exp_avg_sq[k] = states[4 + k].data_ptr()
    st.workspace = ws.data_ptr()
    om, mm, vm = _host_state(N, Np)
    states[0].copy_(torch.from_numpy(om))
    zero.zero_workspace_init(ws.data_ptr(), 0, stream())
    oreps = [np.zeros(N, np.uint16) for _ in range(Nd)]
    t = 0
    for k in range(1, 3):
        hg = [synth.fill_host(synth.NORMAL, synth.BF16, SEED, synth.grad_stream(k, r), N,
                              sigma=1e-3) for r in range(Nd)]
        for r in range(Nd):
            grads[r].view(torch.int16).copy_(torch.from_numpy(hg[r].view(np.int16)))
        zero.zero_step(1, Nd, N, 0, st, zero.hparams(**hp), stream())
        t, _, _ = oracle.zero12_step(Nd, N, 0, oracle.BF16, hg, om, mm, vm, oreps, hp, t)
    live = zero.zero_read_result(ws.data_ptr(), stream())["live"]
    assert_f32_close(states[live].cpu().numpy(), om, "unaligned master")
    assert_f32_close(states[4 + live].cpu().numpy(), vm, "unaligned exp_avg_sq")
    for r in range(Nd):
        assert_bf16_close(u16(reps[r]), oreps[r], "unaligned replica")


@pytest.mark.parametrize("Nd,gdt", [(1, zero.ZERO_BF16), (8, zero.ZERO_BF16), (9, zero.ZERO_FP16),
                                    (16, zero.ZERO_FP16), (64, zero.ZERO_BF16)])
def test_tma_and_register_kernels_identical(Nd, gdt):
    """The TMA-pipelined and register-pipelined fused kernels give the same bytes (whole tiles,
    a ragged tail and an unaligned bucket start), and the same flag; sums of squares agree to
    the reduction-order tolerance."""
    N = 2048 * 301 + 1237
    sdt = DT[gdt][1]
    outs = []
    for flags in (zero.ZERO_FUSED | zero.ZERO_FORCE_TMA, zero.ZERO_FUSED | zero.ZERO_NO_TMA):
        buf = zero.ZeroBuffers(2, Nd, N, grad_dtype=gdt, flags=flags)
        _init_state(buf, N, t0=3, m_kind=synth.ABS, v_kind=synth.SQUARE, m_sigma=1e-3,
                    v_sigma=1e-6)
        for k in (1, 2):
            for r in range(Nd):
                fill(buf.grads[r], synth.NORMAL, sdt, synth.grad_stream(k, r), sigma=1e-3)
            buf.step(zero.hparams(**HP_ADAMW_GPT2), bucket=100_001)
        res = buf.result()
        live = buf.live()
        outs.append((res, f32(buf.master[live]).tobytes(), f32(buf.exp_avg[live]).tobytes(),
                     f32(buf.exp_avg_sq[live]).tobytes(),
                     [u16(p).tobytes() for p in buf.params]))
        del buf
    (ra, *a), (rb, *b) = outs
    assert a == b
    assert (ra["step"], ra["overflow"], ra["error"]) == (rb["step"], rb["overflow"], 0) == (5, 0, 0)
    assert abs(ra["grad_sumsq"] - rb["grad_sumsq"]) <= 1e-5 * rb["grad_sumsq"]
    free()


# 64 vectors per thread of one wave: 148 SMs x 3 CTAs x 256 threads x 64 x 8 elements (1 to 4
# replicas per batch), 148 x 2 x 256 x 64 x 8 (batches of 8)
CHUNKED_MIN_N = {1: 58_195_968, 6: 58_195_968, 8: 58_195_968, 12: 38_797_312}


@pytest.mark.parametrize("Nd,gdt,flags", [(1, zero.ZERO_BF16, zero.ZERO_NO_TMA),
                                          (2, zero.ZERO_BF16, zero.ZERO_NO_TMA),
                                          (6, zero.ZERO_FP16, zero.ZERO_NO_TMA),
                                          (8, zero.ZERO_BF16, zero.ZERO_NO_TMA),
                                          (12, zero.ZERO_BF16, zero.ZERO_NO_TMA),
                                          (16, zero.ZERO_FP16, zero.ZERO_FORCE_TMA)])
def test_long_windows_match_oracle(Nd, gdt, flags):
    """Windows long enough for the load-balanced schedules -- the fused kernel's dynamically
    scheduled chunks (Nd = 1, 6, 8 in batches of 4 replicas, 12 in batches of 8: just above the
    length that switches them on), its fixed grid-stride split (Nd = 2) and the TMA kernel's
    multi-wave grid (Nd = 16: 16.4M elements, 3 waves) -- against the oracle at every element:
    two steps, a ragged tail."""
    N = CHUNKED_MIN_N.get(Nd, 2048 * 8000) + 1237
    odt, sdt = DT[gdt]
    ls = 64.0 if gdt == zero.ZERO_FP16 else 1.0
    hp = dict(lr=1e-3, weight_decay=0.01, loss_scale=ls)
    buf = zero.ZeroBuffers(2, Nd, N, grad_dtype=gdt, flags=zero.ZERO_FUSED | flags)
    _init_state(buf, N)
    S, Np, _ = oracle.partition(N, Nd)
    om, mm, vm = _host_state(N, Np)
    oreps = [oracle.f32_to_bf16(om[:N]) for _ in range(Nd)]
    t = 0
    for step in (1, 2):
        sigma = float(np.float32(1e-3 * ls))
        hg = [synth.fill_host(synth.NORMAL, sdt, SEED, synth.grad_stream(step, r), N, sigma=sigma)
              for r in range(Nd)]
        for r in range(Nd):
            fill(buf.grads[r], synth.NORMAL, sdt, synth.grad_stream(step, r), sigma=sigma)
        buf.step(zero.hparams(**hp))
        t, ovf, ss = oracle.zero12_step(Nd, N, 0, odt, hg, om, mm, vm, oreps, hp, t)
    res = _compare_full(buf, om, mm, vm, oreps, t, ss, "long window Nd=%d" % Nd)
    assert res["error"] == 0 and res["skipped"] == 0
    del buf
    free()


@pytest.mark.parametrize("flags", [zero.ZERO_FUSED, zero.ZERO_TWO_PASS])
def test_summed_gradient_option_matches_oracle(flags):
    """grad_average = 0: the reduced gradient is the rank-order sum divided by the loss scale
    only (no 1/Nd), on the fused and the two-pass paths; two steps, every element."""
    Nd, N = 5, 30_011
    hp = dict(lr=1e-3, weight_decay=0.01, loss_scale=4.0, grad_average=False)
    buf = zero.ZeroBuffers(2, Nd, N, flags=flags)
    _init_state(buf, N)
    S, Np, _ = oracle.partition(N, Nd)
    om, mm, vm = _host_state(N, Np)
    oreps = [oracle.f32_to_bf16(om[:N]) for _ in range(Nd)]
    t = 0
    for step in (1, 2):
        hg = [synth.fill_host(synth.NORMAL, synth.BF16, SEED, synth.grad_stream(step, r), N,
                              sigma=4e-3) for r in range(Nd)]
        for r in range(Nd):
            fill(buf.grads[r], synth.NORMAL, synth.BF16, synth.grad_stream(step, r), sigma=4e-3)
        buf.step(zero.hparams(**hp))
        t, ovf, ss = oracle.zero12_step(Nd, N, 0, oracle.BF16, hg, om, mm, vm, oreps, hp, t)
    _compare_full(buf, om, mm, vm, oreps, t, ss, "summed gradient")
    del buf
    free()


def test_stage1_and_stage2_identical():
    Nd, N = 8, 300_001
    outs = []
    for stage in (1, 2):
        buf = zero.ZeroBuffers(stage, Nd, N)
        _init_state(buf, N)
        for k in (1, 2):
            for r in range(Nd):
                fill(buf.grads[r], synth.NORMAL, synth.BF16, synth.grad_stream(k, r), sigma=1e-3)
            buf.step(zero.hparams(**HP_ADAMW_GPT2))
        live = buf.live()
        outs.append((f32(buf.master[live]).tobytes(), u16(buf.params[5]).tobytes()))
        del buf
    assert outs[0] == outs[1]
    free()


def test_bucketed_equals_unbucketed_and_repeatable():
    Nd, N = 4, 1_000_003
    outs = []
    for bucket in (0, 100_000, 77_777, 1_000_003, 3):
        buf = zero.ZeroBuffers(2, Nd, N)
        _init_state(buf, N)
        for r in range(Nd):
            fill(buf.grads[r], synth.NORMAL, synth.BF16, synth.grad_stream(1, r), sigma=1e-3)
        buf.step(zero.hparams(**HP_ADAMW_GPT2), bucket=bucket)
        live = buf.live()
        outs.append((f32(buf.master[live]).tobytes(), f32(buf.exp_avg_sq[live]).tobytes(),
                     u16(buf.params[3]).tobytes()))
        del buf
    assert all(o == outs[0] for o in outs)
    free()


# ----------------------------------------------------------------------------- overflow skip

@pytest.mark.parametrize("flags", [zero.ZERO_FUSED, zero.ZERO_TWO_PASS])
@pytest.mark.parametrize("bad", [0x7F80, 0xFF80, 0x7FC1, "pair"])
def test_overflow_skips_then_recovers(flags, bad):
    Nd, N = 4, 200_003
    hp = dict(HP_ADAMW_GPT2)
    buf = zero.ZeroBuffers(2, Nd, N, flags=flags)
    _init_state(buf, N, t0=10)
    S, Np, _ = oracle.partition(N, Nd)
    om, mm, vm = _host_state(N, Np)
    oreps = [oracle.f32_to_bf16(om[:N]) for _ in range(Nd)]
    t = 10
    # step A: clean
    hg = [synth.fill_host(synth.NORMAL, synth.BF16, SEED, synth.grad_stream(1, r), N, sigma=1e-3)
          for r in range(Nd)]
    for r in range(Nd):
        fill(buf.grads[r], synth.NORMAL, synth.BF16, synth.grad_stream(1, r), sigma=1e-3)
    buf.step(zero.hparams(**hp))
    t, _, _ = oracle.zero12_step(Nd, N, 0, oracle.BF16, hg, om, mm, vm, oreps, hp, t)
    live = buf.live()
    snap = [f32(buf.master[live]).tobytes(), f32(buf.exp_avg[live]).tobytes(),
            f32(buf.exp_avg_sq[live]).tobytes()] + [u16(p).tobytes() for p in buf.params]
    # step B: one non-finite gradient element somewhere -> the whole step is skipped
    hg = [synth.fill_host(synth.NORMAL, synth.BF16, SEED, synth.grad_stream(2, r), N, sigma=1e-3)
          for r in range(Nd)]
    for r in range(Nd):
        fill(buf.grads[r], synth.NORMAL, synth.BF16, synth.grad_stream(2, r), sigma=1e-3)
    if bad == "pair":  # +inf and -inf at the same element of two ranks: the sum is NaN
        for r, bits in ((1, 0x7F80), (2, 0xFF80)):
            put_bits(buf.grads[r], 12_345, bits)
            hg[r][12_345] = bits
    else:
        put_bits(buf.grads[3], N - 1, bad)
        hg[3][N - 1] = bad
    buf.step(zero.hparams(**hp))
    t2, ovf, _ = oracle.zero12_step(Nd, N, 0, oracle.BF16, hg, om, mm, vm, oreps, hp, t)
    assert ovf == 1 and t2 == t
    res = buf.result()
    assert res["overflow"] == 1 and res["skipped"] == 1 and res["step"] == t
    live = buf.live()
    now = [f32(buf.master[live]).tobytes(), f32(buf.exp_avg[live]).tobytes(),
           f32(buf.exp_avg_sq[live]).tobytes()] + [u16(p).tobytes() for p in buf.params]
    assert now == snap, "a skipped step changed the state or the replicas"
    # step C: clean again, continues from the unchanged state with t + 1
    hg = [synth.fill_host(synth.NORMAL, synth.BF16, SEED, synth.grad_stream(3, r), N, sigma=1e-3)
          for r in range(Nd)]
    for r in range(Nd):
        fill(buf.grads[r], synth.NORMAL, synth.BF16, synth.grad_stream(3, r), sigma=1e-3)
    buf.step(zero.hparams(**hp))
    t, _, ss = oracle.zero12_step(Nd, N, 0, oracle.BF16, hg, om, mm, vm, oreps, hp, t)
    res = _compare_full(buf, om, mm, vm, oreps, t, ss, "after skip")
    assert res["overflow"] == 0 and res["skipped"] == 1 and res["step"] == 12
    del buf
    free()


def test_bounded_wait_gives_up_reports_error_and_device_stays_usable():
    """A load that never lands (test hook: the producer of CTA 0 skips one unit) must not hang
    the GPU: the consumers give up after 1 s, the step is skipped with the error word set, the
    state and replicas keep their values, and the next step runs normally."""
    Nd, N = 8, 2048 * 400
    hp = dict(HP_ADAMW_GPT2)
    buf = zero.ZeroBuffers(2, Nd, N, flags=zero.ZERO_FUSED | zero.ZERO_FORCE_TMA)
    _init_state(buf, N)
    for r in range(Nd):
        fill(buf.grads[r], synth.NORMAL, synth.BF16, synth.grad_stream(1, r), sigma=1e-3)
    snap = [f32(buf.master[0]).tobytes()] + [u16(p).tobytes() for p in buf.params]
    zero.zero_test_inject_stall(2)  # CTA 0, tile 1, its gradient chunk
    buf.step(zero.hparams(**hp))
    with pytest.raises(zero.ZeroTimeout) as e:  # the synchronizing read reports the timeout
        buf.result()
    assert e.value.code == zero.ZERO_ETIMEOUT
    res = e.value.result
    assert res["error"] != 0 and res["overflow"] == 1 and res["skipped"] == 1 and res["step"] == 0
    assert res["live"] == 0
    assert [f32(buf.master[0]).tobytes()] + [u16(p).tobytes() for p in buf.params] == snap
    buf.step(zero.hparams(**hp))  # the hook was one-shot: this step commits
    with pytest.raises(zero.ZeroTimeout) as e:  # the error word is sticky until init
        buf.result()
    res = e.value.result
    assert res["overflow"] == 0 and res["step"] == 1 and res["live"] == 1
    S, Np, _ = oracle.partition(N, Nd)
    om, mm, vm = _host_state(N, Np)
    grads = [synth.fill_host(synth.NORMAL, synth.BF16, SEED, synth.grad_stream(1, r), N,
                             sigma=1e-3) for r in range(Nd)]
    oreps = [np.zeros(N, np.uint16) for _ in range(Nd)]
    oracle.zero12_step(Nd, N, 0, oracle.BF16, grads, om, mm, vm, oreps, hp, 0)
    assert_f32_close(f32(buf.master[1]), om, "after a timed-out step")
    del buf
    free()


# ----------------------------------------------------------------------------- scaler, clipping

@pytest.mark.parametrize("flags", [zero.ZERO_FUSED, zero.ZERO_FUSED | zero.ZERO_FORCE_TMA,
                                   zero.ZERO_TWO_PASS])
def test_dynamic_loss_scaler_matches_oracle(flags):
    """fp16 gradients carrying the workspace's loss scale; an overflow on step 3 halves the
    scale and skips; two clean steps double it.  Every element and the scale sequence."""
    Nd, N = 4, 2048 * 60 + 5
    hp = dict(lr=1e-3, weight_decay=0.01, dynamic_scale=True, scale_interval=2,
              scale_growth=2.0, scale_backoff=0.5)
    buf = zero.ZeroBuffers(2, Nd, N, grad_dtype=zero.ZERO_FP16, flags=flags)
    _init_state(buf, N)
    zero.zero_loss_scaler_init(buf.ws.data_ptr(), 1024.0, 2.0, 0.5, 2, stream())
    S, Np, _ = oracle.partition(N, Nd)
    om, mm, vm = _host_state(N, Np)
    oreps = [oracle.f32_to_bf16(om[:N]) for _ in range(Nd)]
    t, scale, good = 0, 1024.0, 0
    seen = []
    for k in range(1, 7):
        res = buf.result()
        assert res["dynamic_scale"] == 1 and res["loss_scale"] == scale
        sigma = float(np.float32(1e-4 * scale))
        hg = [synth.fill_host(synth.NORMAL, synth.FP16, SEED, synth.grad_stream(k, r), N,
                              sigma=sigma) for r in range(Nd)]
        for r in range(Nd):
            fill(buf.grads[r], synth.NORMAL, synth.FP16, synth.grad_stream(k, r), sigma=sigma)
        if k == 3:
            put_bits(buf.grads[2], 777, 0x7C00)
            hg[2][777] = 0x7C00
        buf.step(zero.hparams(lr=1e-3, weight_decay=0.01))
        t, ovf, ss, scale, good = oracle.zero12_step_ex(Nd, N, 0, oracle.FP16, hg, om, mm, vm,
                                                        oreps, hp, t, scale, good)
        res = buf.result()
        assert res["overflow"] == ovf == (1 if k == 3 else 0)
        assert (res["loss_scale"], res["good_steps"]) == (scale, good)
        seen.append(scale)
    assert seen == [1024.0, 2048.0, 1024.0, 1024.0, 2048.0, 2048.0]
    _compare_full(buf, om, mm, vm, oreps, t, ss, "dynamic scale")
    del buf
    free()


@pytest.mark.parametrize("Nd,N,bucket", [(8, 300_007, 0), (3, 100_003, 20_001)])
def test_clipping_two_pass_matches_oracle(Nd, N, bucket):
    hp = dict(lr=1e-3, weight_decay=0.01, loss_scale=1.0, max_grad_norm=0.05)
    buf = zero.ZeroBuffers(2, Nd, N, flags=zero.ZERO_TWO_PASS)
    _init_state(buf, N)
    S, Np, _ = oracle.partition(N, Nd)
    om, mm, vm = _host_state(N, Np)
    oreps = [np.zeros(N, np.uint16) for _ in range(Nd)]
    t = 0
    for k in (1, 2, 3):
        hg = [synth.fill_host(synth.NORMAL, synth.BF16, SEED, synth.grad_stream(k, r), N,
                              sigma=1e-3) for r in range(Nd)]
        for r in range(Nd):
            fill(buf.grads[r], synth.NORMAL, synth.BF16, synth.grad_stream(k, r), sigma=1e-3)
        buf.step(zero.hparams(lr=1e-3, weight_decay=0.01, max_grad_norm=0.05), bucket=bucket)
        t, ovf, ss, _, _ = oracle.zero12_step_ex(Nd, N, bucket, oracle.BF16, hg, om, mm, vm, oreps,
                                                 hp, t)
        assert np.sqrt(ss) > 0.05  # clipping is active
    _compare_full(buf, om, mm, vm, oreps, t, ss, "clipped two-pass")
    del buf
    free()


def test_clipping_zero3_matches_flat_oracle():
    """ZeRO-3 computes what unsharded data parallelism computes, so the clipped ZeRO-3 step on
    unpadded layers equals the clipped flat step on the concatenated gradients."""
    Nd, L, nl = 4, 4096, 3
    N = L * nl
    hp = dict(lr=1e-3, weight_decay=0.01, loss_scale=1.0, max_grad_norm=0.01)
    buf = zero.ZeroBuffers(3, Nd, N, layer_len=L, per_layer_buffers=True)
    om = synth.fill_host(synth.NORMAL, synth.F32, SEED, synth.MASTER_STREAM, N, sigma=0.02)
    buf.master[0].copy_(torch.from_numpy(om))
    buf.init_workspace(0)
    buf.sync_params_from_master()
    mm = np.zeros(N, np.float32)
    vm = np.zeros(N, np.float32)
    oreps = [np.zeros(N, np.uint16) for _ in range(Nd)]
    t = 0
    for k in (1, 2):
        flat = [synth.fill_host(synth.NORMAL, synth.BF16, SEED, synth.grad_stream(k, r), N,
                                sigma=1e-3) for r in range(Nd)]
        for r in range(Nd):
            buf.grads[r].view(torch.int16).copy_(torch.from_numpy(flat[r].view(np.int16)))
        buf.step(zero.hparams(lr=1e-3, weight_decay=0.01, max_grad_norm=0.01))
        t, ovf, ss, _, _ = oracle.zero12_step_ex(Nd, N, 0, oracle.BF16, flat, om, mm, vm, oreps,
                                                 hp, t)
    res = buf.result()
    assert res["step"] == t == 2 and abs(res["grad_sumsq"] - ss) <= 1e-5 * ss
    assert_f32_close(f32(buf.master[0]), om, "zero3 clipped master")
    assert_f32_close(f32(buf.exp_avg_sq[0]), vm, "zero3 clipped exp_avg_sq")
    assert_bf16_close(u16(buf.param_shard), oreps[0], "zero3 clipped bf16 shard")
    del buf
    free()


@pytest.mark.parametrize("max_norm", [0.0, 0.01])
def test_bf16_grad_shard_zero3_and_two_pass_match_oracle(max_norm):
    """The reduced gradient kept as bf16: ZeRO-3 (per-layer) and the two-pass ZeRO-2 step both
    equal the oracle's bf16-kept variant (ZeRO-3 against the flat oracle: same arithmetic)."""
    Nd, L, nl = 4, 8192, 3
    N = L * nl
    hp = dict(lr=1e-3, weight_decay=0.01, loss_scale=1.0, max_grad_norm=max_norm, bf16_grad=True)
    chp = zero.hparams(lr=1e-3, weight_decay=0.01, max_grad_norm=max_norm)
    z3 = zero.ZeroBuffers(3, Nd, N, layer_len=L, per_layer_buffers=True,
                          flags=zero.ZERO_BF16_GRAD_SHARD)
    tp = zero.ZeroBuffers(2, Nd, N, flags=zero.ZERO_TWO_PASS | zero.ZERO_BF16_GRAD_SHARD)
    assert z3.grad_shard.dtype == torch.bfloat16 and tp.grad_shard.dtype == torch.bfloat16
    om = synth.fill_host(synth.NORMAL, synth.F32, SEED, synth.MASTER_STREAM, N, sigma=0.02)
    for b in (z3, tp):
        b.master[0].copy_(torch.from_numpy(om))
        b.init_workspace(0)
        b.sync_params_from_master()
    mm = np.zeros(N, np.float32)
    vm = np.zeros(N, np.float32)
    oreps = [np.zeros(N, np.uint16) for _ in range(Nd)]
    t = 0
    for k in (1, 2):
        flat = [synth.fill_host(synth.NORMAL, synth.BF16, SEED, synth.grad_stream(k, r), N,
                                sigma=1e-3) for r in range(Nd)]
        for b in (z3, tp):
            for r in range(Nd):
                b.grads[r].view(torch.int16).copy_(torch.from_numpy(flat[r].view(np.int16)))
            b.step(chp)
        t, ovf, ss, _, _ = oracle.zero12_step_ex(Nd, N, 0, oracle.BF16, flat, om, mm, vm, oreps,
                                                 hp, t)
    for b, tag in ((z3, "zero3"), (tp, "two-pass")):
        res = b.result()
        assert res["step"] == t == 2 and abs(res["grad_sumsq"] - ss) <= 1e-5 * ss
        assert_f32_close(f32(b.master[0]), om, tag + " bf16-grad master")
        assert_f32_close(f32(b.exp_avg[0]), mm, tag + " bf16-grad exp_avg")
        assert_f32_close(f32(b.exp_avg_sq[0]), vm, tag + " bf16-grad exp_avg_sq")
    assert_bf16_close(u16(z3.param_shard), oreps[0], "zero3 bf16-grad weights")
    for r in range(Nd):
        assert_bf16_close(u16(tp.params[r]), oreps[r], "two-pass bf16-grad replica")
    del z3, tp
    free()


# ----------------------------------------------------------------------------- randomized

def _random_cases(n_cases=40, seed=2026):
    rng = np.random.default_rng(seed)
    cases = []
    for k in range(n_cases):
        N = int(rng.choice([0, 1, 7, 9, 63, 4095, 4097, 20_000, 65_536 + 5, 150_001, 300_000]))
        Nd = int(rng.choice([1, 2, 3, 4, 5, 8, 13, 16, 31, 64]))
        gdt = int(rng.choice([zero.ZERO_BF16, zero.ZERO_FP16]))
        path = str(rng.choice(["fused", "tma", "two-pass", "two-pass-g16"]))
        bucket = int(rng.choice([0, 0, 1000, 2048 * 3 + 5, 50_001]))
        clip = path.startswith("two-pass") and bool(rng.random() < 0.5)
        dyn = bool(rng.random() < 0.3)
        cases.append((k, N, Nd, gdt, path, bucket, clip, dyn))
    return cases


@pytest.mark.parametrize("case", _random_cases(), ids=lambda c: "case%d" % c[0])
def test_randomized_against_oracle(case):
    """Seeded random shapes, paths and options, two steps each, every element compared."""
    k, N, Nd, gdt, path, bucket, clip, dyn = case
    odt, sdt = DT[gdt]
    flags = {"fused": zero.ZERO_FUSED, "tma": zero.ZERO_FUSED | zero.ZERO_FORCE_TMA,
             "two-pass": zero.ZERO_TWO_PASS,
             "two-pass-g16": zero.ZERO_TWO_PASS | zero.ZERO_BF16_GRAD_SHARD}[path]
    max_norm = 1e-3 if clip else 0.0
    ls = 64.0 if gdt == zero.ZERO_FP16 else 1.0
    hp = dict(lr=1e-3, weight_decay=0.01, loss_scale=ls, max_grad_norm=max_norm,
              bf16_grad=path == "two-pass-g16", dynamic_scale=dyn, scale_interval=1)
    buf = zero.ZeroBuffers(2, Nd, N, grad_dtype=gdt, flags=flags)
    _init_state(buf, N, t0=int(k))
    if dyn:
        zero.zero_loss_scaler_init(buf.ws.data_ptr(), ls, 2.0, 0.5, 1, stream())
    S, Np, _ = oracle.partition(N, Nd)
    om, mm, vm = _host_state(N, Np)
    oreps = [oracle.f32_to_bf16(om[:N]) for _ in range(Nd)]
    t, scale, good = int(k), ls, 0
    for step in (1, 2):
        sigma = float(np.float32(1e-3 * scale)) if gdt == zero.ZERO_FP16 else 1e-3
        hg = [synth.fill_host(synth.NORMAL, sdt, SEED, synth.grad_stream(step, r), N, sigma=sigma)
              for r in range(Nd)]
        for r in range(Nd):
            if N:
                fill(buf.grads[r], synth.NORMAL, sdt, synth.grad_stream(step, r), n=N,
                     sigma=sigma)
        buf.step(zero.hparams(lr=1e-3, weight_decay=0.01, loss_scale=ls,
                              max_grad_norm=max_norm), bucket=bucket)
        t, ovf, ss, scale, good = oracle.zero12_step_ex(Nd, N, bucket, odt, hg, om, mm, vm, oreps,
                                                        hp, t, scale, good)
    res = _compare_full(buf, om, mm, vm, oreps, t, ss, "case %d" % k)
    if dyn:
        assert res["loss_scale"] == scale
    del buf
    free()


def _random_zero3_cases(n_cases=24, seed=2027):
    rng = np.random.default_rng(seed)
    cases = []
    for k in range(n_cases):
        Nd = int(rng.choice([1, 2, 3, 4, 5, 8, 13, 16]))
        L = int(rng.choice([1, 7, 1000, 4096, 4097, 20_000, 65_536, 65_541]))
        nl = int(rng.integers(1, 5))
        N = L * nl - int(rng.integers(0, L)) if nl > 1 else L  # the last layer may be shorter
        gdt = int(rng.choice([zero.ZERO_BF16, zero.ZERO_FP16]))
        path = ["two-phase", "two-phase-g16", "tma-gather", "fused-layers"][k % 4]
        clip = path.startswith("two-phase") and bool(rng.random() < 0.5)
        dyn = bool(rng.random() < 0.3)
        inject = bool(rng.random() < 0.25)
        cases.append((k, N, L, Nd, gdt, path, clip, dyn, inject))
    return cases


@pytest.mark.parametrize("case", _random_zero3_cases(), ids=lambda c: "case%d" % c[0])
def test_randomized_zero3_against_flat_oracle(case):
    """Seeded random ZeRO-3 layer shapes, paths and options, three steps each: ZeRO-3 computes
    what unsharded data parallelism computes, so every real element equals the flat oracle step
    on the concatenated layers (state, bf16 shards, the next step's gathered weights)."""
    k, N, L, Nd, gdt, path, clip, dyn, inject = case
    odt, sdt = DT[gdt]
    flags = {"two-phase": zero.ZERO_FUSED, "two-phase-g16": zero.ZERO_BF16_GRAD_SHARD,
             "tma-gather": zero.ZERO_FORCE_TMA, "fused-layers": zero.ZERO_FUSED_LAYERS}[path]
    max_norm = 1e-3 if clip else 0.0
    ls = 64.0 if gdt == zero.ZERO_FP16 else 1.0
    hp = dict(lr=1e-3, weight_decay=0.01, loss_scale=ls, max_grad_norm=max_norm,
              bf16_grad=path == "two-phase-g16", dynamic_scale=dyn, scale_interval=1)
    buf = zero.ZeroBuffers(3, Nd, N, grad_dtype=gdt, flags=flags, layer_len=L,
                           per_layer_buffers=True)
    # real elements of the padded per-layer layout, in flat order
    real = np.concatenate([np.arange(Ll) + sum(buf.layer_padded[:l])
                           for l, Ll in enumerate(buf.layer_sizes)]).astype(np.int64)
    om = synth.fill_host(synth.NORMAL, synth.F32, SEED, synth.MASTER_STREAM, N, sigma=0.02)
    full = np.zeros(buf.Np, np.float32)
    full[real] = om
    buf.master[0].copy_(torch.from_numpy(full))
    buf.init_workspace(0)
    if dyn:
        zero.zero_loss_scaler_init(buf.ws.data_ptr(), ls, 2.0, 0.5, 1, stream())
    buf.sync_params_from_master()
    _, Np, _ = oracle.partition(N, Nd)  # the flat oracle works on the flat padded layout
    om = np.concatenate([om, np.zeros(Np - N, np.float32)])
    mm = np.zeros(Np, np.float32)
    vm = np.zeros(Np, np.float32)
    oreps = [oracle.f32_to_bf16(om[:N]) for _ in range(Nd)]
    t, scale, good = 0, ls, 0
    for step in (1, 2, 3):
        prev = oreps[0].copy()
        sigma = float(np.float32(1e-3 * scale)) if gdt == zero.ZERO_FP16 else 1e-3
        hg = [synth.fill_host(synth.NORMAL, sdt, SEED, synth.grad_stream(step, r), N, sigma=sigma)
              for r in range(Nd)]
        if inject and step == 2:
            hg[Nd - 1][N // 2] = 0x7F80 if gdt == zero.ZERO_BF16 else 0x7C00  # +inf
        for r in range(Nd):
            buf.grads[r].view(torch.int16).copy_(torch.from_numpy(hg[r].view(np.int16)))
        buf.step(zero.hparams(lr=1e-3, weight_decay=0.01, loss_scale=ls, max_grad_norm=max_norm))
        t, ovf, ss, scale, good = oracle.zero12_step_ex(Nd, N, 0, odt, hg, om, mm, vm, oreps,
                                                        hp, t, scale, good)
        for r in range(Nd):  # the forward gather of this step saw the previous weights
            assert u16(buf.params[r]).tobytes() == prev.tobytes(), "case %d gather" % k
    res = buf.result()
    assert res["step"] == t and res["skipped"] == (1 if inject else 0), (case, res)
    if ss > 0 and np.isfinite(ss):
        assert abs(res["grad_sumsq"] - ss) <= 1e-5 * ss
    if dyn:
        assert res["loss_scale"] == scale
    live = buf.live()
    idx = torch.from_numpy(real).cuda()
    assert_f32_close(f32(buf.master[live][idx]), om[:N], "case %d master" % k)
    assert_f32_close(f32(buf.exp_avg[live][idx]), mm[:N], "case %d exp_avg" % k)
    assert_f32_close(f32(buf.exp_avg_sq[live][idx]), vm[:N], "case %d exp_avg_sq" % k)
    assert_bf16_close(u16(buf.param_shard[idx]), oreps[0], "case %d bf16 shard" % k)
    del buf
    free()


# ----------------------------------------------------------------------------- CUDA graphs

@pytest.mark.parametrize("stage,flags,bucket", [(2, zero.ZERO_FUSED, 0), (2, zero.ZERO_FUSED, 20_000),
                                                (2, zero.ZERO_FUSED | zero.ZERO_FORCE_TMA, 0),
                                                (2, zero.ZERO_TWO_PASS, 0), (3, zero.ZERO_FUSED, 0),
                                                (3, zero.ZERO_FUSED_LAYERS, 0)])
def test_step_captured_in_a_cuda_graph_matches_eager(stage, flags, bucket):
    """The whole step is device-resident (step counter, live copy, overflow decision and loss
    scale live in the workspace), so it can be captured once and replayed: three replays with
    fresh gradients give the same bytes as three eager steps, including a skipped one (with
    buckets: later buckets are programmatic dependent launches inside the graph)."""
    Nd, N, L = 4, 2048 * 40 + 8, 2048 * 10 + 2
    hp = zero.hparams(lr=1e-3, weight_decay=0.01)
    outs = []
    for use_graph in (False, True):
        buf = (zero.ZeroBuffers(3, Nd, N, flags=flags, layer_len=L, per_layer_buffers=True)
               if stage == 3 else zero.ZeroBuffers(stage, Nd, N, flags=flags))
        fill(buf.master[0], synth.NORMAL, synth.F32, synth.MASTER_STREAM, n=N, sigma=0.02)
        buf.init_workspace(0)
        buf.sync_params_from_master()
        graph = None
        side = torch.cuda.Stream()
        for k in (1, 2, 3):
            for r in range(Nd):
                fill(buf.grads[r], synth.NORMAL, synth.BF16, synth.grad_stream(k, r), sigma=1e-3)
            if k == 2:
                put_bits(buf.grads[1], 5, 0x7F80)
            if not use_graph:
                buf.step(hp, bucket=bucket)
                continue
            if graph is None:
                side.wait_stream(torch.cuda.current_stream())
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph, stream=side):
                    zero.zero_step(buf.stage, Nd, N, buf.layer_len if stage == 3 else bucket,
                                   buf.state, hp, side.cuda_stream)
                torch.cuda.current_stream().wait_stream(side)
            graph.replay()  # capture does not run the work: every step comes from a replay
        torch.cuda.synchronize()
        res = buf.result()
        live = buf.live()
        outs.append((res["step"], res["skipped"], f32(buf.master[live]).tobytes(),
                     f32(buf.exp_avg_sq[live]).tobytes(),
                     u16(buf.param_shard if stage == 3 else buf.params[Nd - 1]).tobytes()))
        del graph, buf
    assert outs[0][:2] == outs[1][:2] == (2, 1)
    assert outs[0] == outs[1]
    free()


# ----------------------------------------------------------------------------- ZeRO-Offload

@pytest.mark.parametrize("gdt,dynamic,max_norm", [(zero.ZERO_BF16, False, 0.0),
                                                  (zero.ZERO_FP16, True, 0.05)])
def test_offload_step_matches_oracle(gdt, dynamic, max_norm):
    """Reduce-scatter on the GPU, AdamW on host memory, weights back to every replica: host
    state and device replicas equal the oracle's; an overflow on step 2 is skipped."""
    Nd, N, chunk = 4, 1_000_003, 300_000
    odt, sdt = DT[gdt]
    hp = dict(lr=1e-3, weight_decay=0.01, loss_scale=1.0, max_grad_norm=max_norm,
              dynamic_scale=dynamic, scale_interval=2)
    buf = zero.ZeroOffloadBuffers(Nd, N, grad_dtype=gdt, chunk=chunk, host_threads=4)
    S, Np, _ = oracle.partition(N, Nd)
    om, mm, vm = _host_state(N, Np)
    buf.master.copy_(torch.from_numpy(om[:N]))
    buf.init_workspace(0)
    if dynamic:
        zero.zero_loss_scaler_init(buf.ws.data_ptr(), 512.0, 2.0, 0.5, 2, stream())
    buf.sync_params_from_master()
    oreps = [oracle.f32_to_bf16(om[:N]) for _ in range(Nd)]
    t, scale, good = 0, 512.0, 0
    for k in (1, 2, 3, 4):
        sigma = float(np.float32(1e-4 * scale)) if dynamic else 1e-3
        hg = [synth.fill_host(synth.NORMAL, sdt, SEED, synth.grad_stream(k, r), N, sigma=sigma)
              for r in range(Nd)]
        for r in range(Nd):
            fill(buf.grads[r], synth.NORMAL, sdt, synth.grad_stream(k, r), sigma=sigma)
        if k == 2:
            bits = 0x7C00 if sdt == synth.FP16 else 0x7F80
            put_bits(buf.grads[1], N - 3, bits)
            hg[1][N - 3] = bits
        buf.step(zero.hparams(lr=1e-3, weight_decay=0.01, max_grad_norm=max_norm))
        t, ovf, ss, scale, good = oracle.zero12_step_ex(Nd, N, 0, odt, hg, om, mm, vm, oreps, hp,
                                                        t, scale, good)
        res = buf.result()
        assert res["overflow"] == ovf == (1 if k == 2 else 0) and res["step"] == t
        if dynamic:
            assert res["loss_scale"] == scale
    torch.cuda.synchronize()
    assert_f32_close(buf.master.numpy(), om[:N], "offload master")
    assert_f32_close(buf.exp_avg.numpy(), mm[:N], "offload exp_avg")
    assert_f32_close(buf.exp_avg_sq.numpy(), vm[:N], "offload exp_avg_sq")
    for r in range(Nd):
        assert_bf16_close(u16(buf.params[r]), oreps[r], "offload replica %d" % r)
    del buf
    free()


# ----------------------------------------------------------------------------- building blocks

def test_building_blocks_two_pass_matches_oracle():
    """begin -> reduce_scatter (per rank's shard) -> adam (per shard) -> allgather -> end."""
    Nd, N = 5, 123_457
    hp = dict(HP_ADAMW_FP16_LS1024)
    S, Np, _ = oracle.partition(N, Nd)
    sigma = 0.1024
    grads = [torch.zeros(N, dtype=torch.float16, device="cuda") for _ in range(Nd)]
    reps = [torch.zeros(N, dtype=torch.bfloat16, device="cuda") for _ in range(Nd)]
    p = torch.zeros(Np, device="cuda")
    m = torch.zeros(Np, device="cuda")
    v = torch.zeros(Np, device="cuda")
    gsh = torch.zeros(Np, device="cuda")
    ws = torch.zeros(zero.zero_workspace_bytes(), dtype=torch.uint8, device="cuda")
    om, mm, vm = _host_state(N, Np)
    p.copy_(torch.from_numpy(om))
    zero.zero_workspace_init(ws.data_ptr(), 0, stream())
    chp = zero.hparams(**hp)
    oreps = [np.zeros(N, np.uint16) for _ in range(Nd)]
    t = 0
    for k in (1, 2):
        hg = [synth.fill_host(synth.NORMAL, synth.FP16, SEED, synth.grad_stream(k, r), N,
                              sigma=sigma) for r in range(Nd)]
        for r in range(Nd):
            fill(grads[r], synth.NORMAL, synth.FP16, synth.grad_stream(k, r), sigma=sigma)
        zero.zero_begin_step(ws.data_ptr(), stream())
        gp = [g.data_ptr() for g in grads]
        for r in range(Nd):  # every rank reduce-scatters its own shard
            lo, hi = min(r * S, N), min((r + 1) * S, N)
            zero.zero_reduce_scatter(gp, zero.ZERO_FP16, Nd, lo, hi, chp, gsh.data_ptr(),
                                     ws.data_ptr(), stream())
        for r in range(Nd):
            lo, hi = min(r * S, N), min((r + 1) * S, N)
            zero.zero_adam_shard(p.data_ptr(), m.data_ptr(), v.data_ptr(), gsh.data_ptr(), lo, hi,
                                 chp, None, ws.data_ptr(), stream())
        zero.zero_allgather(p.data_ptr(), [x.data_ptr() for x in reps], Nd, 0, N,
                            zero.ZERO_GATE_NO_OVERFLOW, ws.data_ptr(), stream())
        res_mid = zero.zero_read_result(ws.data_ptr(), stream())
        zero.zero_end_step(ws.data_ptr(), stream())
        t, ovf, ss = oracle.zero12_step(Nd, N, 0, oracle.FP16, hg, om, mm, vm, oreps, hp, t)
        g_or, _, _ = oracle.reduce_scatter(Nd, N, oracle.FP16, hg, hp)
        assert_f32_close(gsh.cpu().numpy(), g_or, "reduced gradient shard")
        assert abs(res_mid["pending_sumsq"] - ss) <= 1e-5 * ss
    res = zero.zero_read_result(ws.data_ptr(), stream())
    assert res["step"] == 2 and res["overflow"] == 0
    assert_f32_close(p.cpu().numpy(), om, "master")
    assert_f32_close(m.cpu().numpy(), mm, "exp_avg")
    assert_f32_close(v.cpu().numpy(), vm, "exp_avg_sq")
    for r in range(Nd):
        assert_bf16_close(u16(reps[r]), oreps[r], "replica")


def test_empty_step_advances_t():
    buf = zero.ZeroBuffers(2, 4, 0)
    buf.init_workspace(5)
    buf.step(zero.hparams(**HP_ADAM_LR1E3))
    res = buf.result()
    assert res["step"] == 6 and res["overflow"] == 0 and res["grad_sumsq"] == 0.0


# ----------------------------------------------------------------------------- ZeRO-3

@pytest.mark.parametrize("L,Nd,nout", [(202_375, 8, 8), (1001, 3, 1), (7, 4, 2), (64, 64, 3),
                                       (25_296_896 // 64, 8, 8)])
def test_gather_layer_full(L, Nd, nout):
    S, Np, _ = oracle.partition(L, Nd)
    flat = torch.zeros(Np, dtype=torch.bfloat16, device="cuda")
    fill(flat, synth.NORMAL, synth.BF16, 99, n=L, sigma=0.02)
    shards = [flat[r * S:(r + 1) * S] for r in range(Nd)]
    outs = [torch.zeros(L, dtype=torch.bfloat16, device="cuda") for _ in range(nout)]
    zero.zero3_gather_layer([s.data_ptr() for s in shards], Nd, L, [o.data_ptr() for o in outs],
                            stream())
    want = oracle.zero3_gather(Nd, L, [u16(s) for s in shards])
    for o in outs:
        assert u16(o).tobytes() == want.tobytes()


@pytest.mark.parametrize("path", ["register-gather", "tma-gather", "fused-layers"])
@pytest.mark.parametrize("layer_len,N,Nd", [(1000, 5333, 3), (4096, 4096 * 3, 8),
                                            (12_345, 12_345 * 2 + 17, 4), (65_536, 65_536 * 3, 8)])
def test_zero3_step_matches_oracle(layer_len, N, Nd, path):
    """zero_step(stage=3): per-layer gather from the bf16 shards (register kernel, or the TMA
    fan-out with ZERO_FORCE_TMA), per-layer reduce-scatter, then Adam on every shard and the
    bf16 shard update -- or, with ZERO_FUSED_LAYERS, one speculative fused pass per layer into
    the other state copy; four steps, the third overflowing (+inf in one replica of the last
    layer), every element."""
    flags = {"register-gather": zero.ZERO_FUSED, "tma-gather": zero.ZERO_FORCE_TMA,
             "fused-layers": zero.ZERO_FUSED_LAYERS}[path]
    buf = zero.ZeroBuffers(3, Nd, N, flags=flags, layer_len=layer_len, per_layer_buffers=True)
    sizes = buf.layer_sizes
    hp = dict(HP_ADAMW_ZERO3)
    total = buf.Np
    om = np.zeros(total, np.float32)
    off = 0
    for l, (Ll, Lp) in enumerate(zip(sizes, buf.layer_padded)):
        om[off:off + Ll] = synth.fill_host(synth.NORMAL, synth.F32, SEED, 1000 + l, Ll, sigma=0.02)
        off += Lp
    buf.master[0].copy_(torch.from_numpy(om))
    buf.init_workspace(0)
    buf.sync_params_from_master()
    mm = np.zeros(total, np.float32)
    vm = np.zeros(total, np.float32)
    sh16 = oracle.f32_to_bf16(om)
    assert u16(buf.param_shard).tobytes() == sh16.tobytes()
    t = 0
    for k in (1, 2, 3, 4):
        hgrads, gathered = [], []
        for l, Ll in enumerate(sizes):
            for r in range(Nd):
                hg = synth.fill_host(synth.NORMAL, synth.BF16, SEED, synth.grad_stream(k, r, l),
                                     Ll, sigma=1e-3)
                if k == 3 and l == len(sizes) - 1 and r == Nd - 1:
                    hg[Ll // 2] = 0x7F80  # +inf: the whole step is skipped
                hgrads.append(hg)
                buf.grads[r][l * layer_len:l * layer_len + Ll].view(torch.int16).copy_(
                    torch.from_numpy(hg.view(np.int16)))
                gathered.append(np.zeros(Ll, np.uint16))
        buf.step(zero.hparams(**hp))
        t, ovf, ss = oracle.zero3_step(Nd, sizes, oracle.BF16, hgrads, om, mm, vm, sh16, gathered,
                                       hp, t)
        for l, Ll in enumerate(sizes):
            for r in range(Nd):
                got = u16(buf.params[r][l * layer_len:l * layer_len + Ll])
                assert got.tobytes() == gathered[l * Nd + r].tobytes(), "gather layer %d" % l
        if k == 3:
            assert buf.result()["overflow"] == 1 and buf.result()["skipped"] == 1
            assert u16(buf.param_shard).tobytes() == sh16.tobytes(), "skipped step changed shards"
    res = buf.result()
    assert res["step"] == t == 3 and res["skipped"] == 1
    assert abs(res["grad_sumsq"] - ss) <= 1e-5 * ss
    live = buf.live()
    assert live == (1 if path == "fused-layers" else 0)  # three committed flips
    assert_f32_close(f32(buf.master[live]), om, "zero3 master")
    assert_f32_close(f32(buf.exp_avg[live]), mm, "zero3 exp_avg")
    assert_f32_close(f32(buf.exp_avg_sq[live]), vm, "zero3 exp_avg_sq")
    assert_bf16_close(u16(buf.param_shard), sh16, "zero3 bf16 shard")
    del buf
    free()


# ----------------------------------------------------------------------------- full-size workloads

def _sampled_run(stage, Nd, N, steps, hp, gdt, sigma, bucket=0, flags=zero.ZERO_FUSED,
                 kind=synth.NORMAL, tail_sigma=0.0, t0=0, m_kind=synth.ZERO, v_kind=synth.ZERO,
                 m_sigma=0.0, v_sigma=0.0, inject=None, n_random=100_000, extra=()):
    odt, sdt = DT[gdt]
    buf = zero.ZeroBuffers(stage, Nd, N, grad_dtype=gdt, flags=flags)
    _init_state(buf, N, t0, m_kind, v_kind, m_sigma, v_sigma)
    inj_rank, inj_idx = inject[1] if inject else (None, None)
    idx = sample_indices(N, n_random, list(extra) + ([inj_idx] if inject else []))
    p0 = synth.values(synth.NORMAL, synth.F32, SEED, synth.MASTER_STREAM, idx, 0.02)
    m0 = synth.values(m_kind, synth.F32, SEED, synth.M_STREAM, idx, m_sigma)
    v0 = synth.values(v_kind, synth.F32, SEED, synth.V_STREAM, idx, v_sigma)
    so = SampledOracle(idx, Nd, odt, p0, m0, v0, t0)
    chp = zero.hparams(**hp)
    for k in range(1, steps + 1):
        for r in range(Nd):
            fill(buf.grads[r], kind, sdt, synth.grad_stream(k, r), sigma=sigma,
                 tail_sigma=tail_sigma)
        g_en = grads_at(idx, Nd, sdt, k, sigma, kind, tail_sigma)
        skip = bool(inject) and k == inject[0]
        if skip:
            put_bits(buf.grads[inj_rank], inj_idx, 0x7F80 if sdt == synth.BF16 else 0x7C00)
            g_en[np.searchsorted(idx, inj_idx), inj_rank] = 0x7F80 if sdt == synth.BF16 else 0x7C00
        live_before = buf.live()
        before = at(buf.master[live_before], idx) if skip else None
        buf.step(chp, bucket=bucket)
        so.step(g_en, hp, skip)
        res = buf.result()
        assert res["overflow"] == int(skip), (k, res)
        live = buf.live()
        if skip:
            assert live == live_before
            assert at(buf.master[live], idx).tobytes() == before.tobytes()
        assert_f32_close(at(buf.master[live], idx), so.p, "step %d master" % k)
        assert_f32_close(at(buf.exp_avg[live], idx), so.m, "step %d exp_avg" % k)
        assert_f32_close(at(buf.exp_avg_sq[live], idx), so.v, "step %d exp_avg_sq" % k)
        for r in sorted({0, Nd // 2, Nd - 1}):
            assert_bf16_close(at(buf.params[r], idx), so.out16, "step %d replica %d" % (k, r))
    res = buf.result()
    assert res["step"] == so.t
    # every rank received the same weights (the all-gather is complete), whole vector
    for r in range(1, Nd):
        assert torch.equal(buf.params[r].view(torch.int16), buf.params[0].view(torch.int16))
    return buf, res, so


def test_zero1_gpt2_small_124m_nd8_ten_steps():
    """N = 124,439,808 (GPT-2 small), Nd = 8, ZeRO-1, 10 AdamW steps (lr 6e-4, wd 0.01), fresh
    bf16 grads ~N(0,1e-3) every step, bf16 weights all-gathered to 8 replicas each step."""
    N, Nd = 124_439_808, 8
    S = oracle.partition(N, Nd)[0]
    buf, res, so = _sampled_run(1, Nd, N, 10, HP_ADAMW_GPT2, zero.ZERO_BF16, 1e-3,
                                extra=boundaries(S, N))
    # property at full size: the reduced gradient is the mean of 8 N(0, 1e-3) replicas, so
    # E[sum g^2] = N * 1e-6 / 8 (the generator's variance is 1 - 2^-32)
    assert abs(res["grad_sumsq"] / (N * 1e-6 / 8) - 1) < 0.01
    assert res["skipped"] == 0
    del buf
    free()


def test_zero2_1p3b_nd16_fp16_buckets_with_overflow():
    """N = 1.3e9 in 25M-element buckets, Nd = 16, fp16 grads ~N(0,1e-4)*1024 carrying loss
    scale 1024 (unscaled in the kernel); +inf planted at a seeded (rank, index) on step 3,
    which must skip that step; 5 AdamW steps."""
    N, Nd, B = 1_300_000_000, 16, 25_000_000
    S = oracle.partition(N, Nd)[0]
    site = synth.inject_site(SEED, Nd, N)
    buf, res, so = _sampled_run(2, Nd, N, 5, HP_ADAMW_FP16_LS1024, zero.ZERO_FP16, 1e-4 * 1024, bucket=B,
                                inject=(3, site), n_random=50_000,
                                extra=boundaries(S, N) + boundaries(B, N))
    assert res["step"] == 4 and res["skipped"] == 1
    del buf
    free()


def test_zero2_2p28_nd64_wide_fan_in():
    """N = 2^28, Nd = 64, bf16 grads ~N(0,1e-3) with 1% of values x1e3 (hash-selected), AdamW
    step 1000 with m ~ |N(0,1e-3)|, v = N(0,1e-6)^2."""
    N, Nd = 1 << 28, 64
    tail = float(np.float32(1e-3 * 1e3))
    buf, res, so = _sampled_run(2, Nd, N, 1, HP_ADAMW_WIDE, zero.ZERO_BF16, 1e-3, kind=synth.HEAVY,
                                tail_sigma=tail, t0=999, m_kind=synth.ABS, v_kind=synth.SQUARE,
                                m_sigma=1e-3, v_sigma=1e-6, n_random=50_000,
                                extra=boundaries(N // Nd, N))
    assert res["step"] == 1000 and res["overflow"] == 0
    # E[g^2] for the mean of 64 replicas: (0.99 * 1e-6 + 0.01 * 1.0) / 64 per element
    expect = N * (0.99e-6 + 0.01) / 64
    assert abs(res["grad_sumsq"] / expect - 1) < 0.02
    del buf
    free()


def test_zero2_2p28_nd8_fused():
    N, Nd = 1 << 28, 8
    buf, res, so = _sampled_run(2, Nd, N, 2, HP_ADAMW_WIDE, zero.ZERO_BF16, 1e-3, n_random=50_000,
                                extra=boundaries(N // Nd, N))
    del buf
    free()


def test_zero3_llama7b_shaped_32_layers_nd8():
    """32 layers of q,k,v,o (4096x4096) + gate,up,down (4096x11008), bf16, Nd = 8; per layer:
    gather the full layer from 8 shards, reduce-scatter 8 bf16 grad replicas ~N(0,1e-3) into
    the fp32 gradient shard; then AdamW on the fp32 shards; 1 step.  Driven through the
    building blocks with fresh gradients per layer (seeded by layer), one layer buffer reused."""
    Nd, L, nl = 8, LLAMA7B_LAYER, 32
    N = L * nl
    S = oracle.partition(L, Nd)[0]
    hp = dict(HP_ADAMW_ZERO3)
    chp = zero.hparams(**hp)
    dev = "cuda"
    master = torch.zeros(N, device=dev)
    m = torch.zeros(N, device=dev)
    v = torch.zeros(N, device=dev)
    gsh = torch.zeros(N, device=dev)
    sh16 = torch.zeros(N, dtype=torch.bfloat16, device=dev)
    grads = [torch.zeros(L, dtype=torch.bfloat16, device=dev) for _ in range(Nd)]
    gathered = [torch.zeros(L, dtype=torch.bfloat16, device=dev) for _ in range(Nd)]
    ws = torch.zeros(zero.zero_workspace_bytes(), dtype=torch.uint8, device=dev)
    s = stream()
    fill(master, synth.NORMAL, synth.F32, synth.MASTER_STREAM, sigma=0.02)
    zero.zero_allgather(master.data_ptr(), [sh16.data_ptr()], 1, 0, N, zero.ZERO_GATE_ALWAYS,
                        None, s)
    zero.zero_workspace_init(ws.data_ptr(), 0, s)
    rng = np.random.default_rng(11)
    loc = np.unique(np.concatenate([rng.integers(0, L, 4000),
                                    np.array([0, L - 1] + boundaries(S, L))]))
    zero.zero_begin_step(ws.data_ptr(), s)
    samples = {}
    for l in range(nl):
        off = l * L
        shards = [sh16.data_ptr() + 2 * (off + r * S) for r in range(Nd)]
        zero.zero3_gather_layer(shards, Nd, L, [g.data_ptr() for g in gathered], s)
        want16 = oracle.f32_to_bf16(synth.values(synth.NORMAL, synth.F32, SEED,
                                                 synth.MASTER_STREAM, off + loc, 0.02))
        for r in (0, Nd - 1):
            assert at(gathered[r], loc).tobytes() == want16.tobytes(), "layer %d gather" % l
        for r in range(Nd):
            fill(grads[r], synth.NORMAL, synth.BF16, synth.grad_stream(1, r, l), sigma=1e-3)
        zero.zero_reduce_scatter([g.data_ptr() for g in grads], zero.ZERO_BF16, Nd, 0, L, chp,
                                 gsh.data_ptr() + 4 * off, ws.data_ptr(), s)
        samples[l] = grads_at(loc, Nd, synth.BF16, 1, 1e-3, layer=l)
    for l in range(nl):
        off = l * L
        zero.zero_adam_shard(master.data_ptr() + 4 * off, m.data_ptr() + 4 * off,
                             v.data_ptr() + 4 * off, gsh.data_ptr() + 4 * off, 0, L, chp,
                             sh16.data_ptr() + 2 * off, ws.data_ptr(), s)
    zero.zero_end_step(ws.data_ptr(), s)
    res = zero.zero_read_result(ws.data_ptr(), s)
    assert res["step"] == 1 and res["overflow"] == 0
    assert abs(res["grad_sumsq"] / (N * 1e-6 / 8) - 1) < 0.01
    for l in (0, 1, 17, 31):
        gidx = l * L + loc
        p0 = synth.values(synth.NORMAL, synth.F32, SEED, synth.MASTER_STREAM, gidx, 0.02)
        so = SampledOracle(gidx, Nd, oracle.BF16, p0, np.zeros_like(p0), np.zeros_like(p0), 0)
        g = so.step(samples[l], hp, False)
        assert_f32_close(at(gsh, gidx), g, "layer %d reduced grad" % l)
        assert_f32_close(at(master, gidx), so.p, "layer %d master" % l)
        assert_f32_close(at(m, gidx), so.m, "layer %d exp_avg" % l)
        assert_f32_close(at(v, gidx), so.v, "layer %d exp_avg_sq" % l)
        assert_bf16_close(at(sh16, gidx), so.out16, "layer %d bf16 shard" % l)
    del master, m, v, gsh, sh16, grads, gathered
    free()
