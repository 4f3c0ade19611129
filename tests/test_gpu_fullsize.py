"""Whole-vector parity at the workloads' full sizes (GPU, through the C ABI).

The sampled checks of test_gpu_parity.py compare tens of thousands of elements per workload;
here every element of the state, the weight shards or replicas and the gathered layers is
compared with the CPU oracle.  The oracle runs as it stands, one call per contiguous chunk of
the vector, on every host core: elements are independent, so a chunk's oracle step gives that
chunk's elements of the whole-vector step whenever the step is not skipped, and a skipped step
is decided by OR-ing the chunks' overflow flags from the oracle's own reduce-scatter.  The
inputs of each chunk are regenerated on the host by the seeded counter-based generator.

Workloads: two Llama-7B-shaped ZeRO-3 layers (2 x 202,375,168 elements, Nd = 8) through
zero_step(stage=3), two-phase and fused-layers, with an overflowing step; the wide fan-in step
(2^28 elements, Nd = 64, heavy-tailed bf16 gradients, AdamW step 1000 with prefilled m, v); ten
ZeRO-1 steps of GPT-2 small (124,439,808, Nd = 8); two steps at 2^28, Nd = 8 (the bench's
default workload); five bucketed fp16 steps of 1.3e9 elements at Nd = 16 with a skipped one.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
import synth
import zero_sharded_optimizer_03_b200 as zero
from _gpu import (HP_ADAMW_FP16_LS1024, HP_ADAMW_GPT2, HP_ADAMW_WIDE, HP_ADAMW_ZERO3, LLAMA7B_LAYER,
                  SEED, fill, free, u16)

pytestmark = pytest.mark.gpu

THREADS = max(1, min(32, len(os.sched_getaffinity(0))))
CHUNK = 1 << 20  # divides the Llama layer (193 x 2^20) and 2^28


def _pmap(fn, items):
    with ThreadPoolExecutor(max_workers=THREADS) as ex:
        return list(ex.map(fn, items))


def f32_err(got, want) -> float:
    """Max relative error |a-b|/max(|b|, 2^-126) of one chunk (0 when bit-identical); NaN
    positions must match."""
    if got.tobytes() == want.tobytes():
        return 0.0
    assert (np.isnan(got) == np.isnan(want)).all()
    fin = ~np.isnan(want)
    err = np.abs(got[fin].astype(np.float64) - want[fin]) / np.maximum(np.abs(want[fin]),
                                                                       2.0 ** -126)
    return float(err.max()) if err.size else 0.0


def bf16_ulps(got, want) -> int:
    """Max distance in bf16 ulps of one chunk (0 when bit-identical)."""
    if got.tobytes() == want.tobytes():
        return 0
    a, b = got.astype(np.int32), want.astype(np.int32)
    a = np.where(a & 0x8000, 0x8000 - (a & 0x7FFF), 0x8000 + a)
    b = np.where(b & 0x8000, 0x8000 - (b & 0x7FFF), 0x8000 + b)
    return int(np.abs(a - b).max())


def _grads_chunk(Nd, sdt, step, lo, n, sigma, layer=0, kind=synth.NORMAL, tail=0.0):
    return [synth.fill_host(kind, sdt, SEED, synth.grad_stream(step, r, layer), n, sigma=sigma,
                            tail_sigma=tail, first=lo) for r in range(Nd)]


# ----------------------------------------------------------------------------- ZeRO-3

@pytest.mark.parametrize("path", ["two-phase", "fused-layers"])
def test_zero3_two_llama_layers_every_element(path):
    """zero_step(stage=3) on two Llama-7B-shaped layers (q,k,v,o 4096x4096 + gate,up,down
    4096x11008 each, bf16, Nd = 8), per-layer gradient and gathered-weight buffers.  Step 1 has
    +inf in layer 1's gradient of rank 5 and must be skipped; step 2 is clean.  Checked against
    the oracle over the whole vector: the gathered layers of every rank after each step, the
    fp32 master / exp_avg / exp_avg_sq, the bf16 weight shards."""
    Nd, L, nl = 8, LLAMA7B_LAYER, 2
    N = L * nl
    flags = zero.ZERO_FUSED_LAYERS if path == "fused-layers" else 0
    hp = dict(HP_ADAMW_ZERO3)
    chp = zero.hparams(**hp)
    buf = zero.ZeroBuffers(3, Nd, N, layer_len=L, per_layer_buffers=True, flags=flags)
    assert buf.Np == N  # the layer length is a multiple of Nd: no padding
    fill(buf.master[0], synth.NORMAL, synth.F32, synth.MASTER_STREAM, n=N, sigma=0.02)
    buf.init_workspace(0)
    buf.sync_params_from_master()
    chunks = [(lo, CHUNK) for lo in range(0, N, CHUNK)]
    # initial weights and their bf16 cast (what every gather must deliver before the update)
    p0 = np.concatenate(_pmap(lambda c: synth.fill_host(synth.NORMAL, synth.F32, SEED,
                                                        synth.MASTER_STREAM, c[1], sigma=0.02,
                                                        first=c[0]), chunks))
    w0 = np.concatenate(_pmap(lambda c: oracle.f32_to_bf16(p0[c[0]:c[0] + c[1]]), chunks))
    inj_layer, inj_rank, inj_idx = 1, 5, 123_457  # index within the layer
    for k in (1, 2):
        for l in range(nl):
            for r in range(Nd):
                fill(buf.grads[r], synth.NORMAL, synth.BF16, synth.grad_stream(k, r, l), n=L,
                     sigma=1e-3, offset=l * L)
        if k == 1:
            buf.grads[inj_rank].view(torch.int16)[inj_layer * L + inj_idx] = 0x7F80
        buf.step(chp)
        res = buf.result()

        # the gathers ran before the update: every rank holds bf16(p0) of both layers
        for r in range(Nd):
            assert u16(buf.params[r]).tobytes() == w0.tobytes(), "step %d gather, rank %d" % (k, r)

        if k == 1:
            # the oracle's reduce-scatter decides the skip: OR of the chunks' overflow flags
            def rs_flag(c):
                lo, n = c
                l = lo // L
                g = _grads_chunk(Nd, synth.BF16, 1, lo - l * L, n, 1e-3, layer=l)
                if l == inj_layer and lo - l * L <= inj_idx < lo - l * L + n:
                    g[inj_rank][inj_idx - (lo - l * L)] = 0x7F80
                return oracle.reduce_scatter(Nd, n, oracle.BF16, g, hp)[1]
            assert any(_pmap(rs_flag, chunks)), "the oracle does not skip step 1"
            assert (res["overflow"], res["skipped"], res["step"]) == (1, 1, 0), res
            live = buf.live()
            assert live == 0
            assert buf.master[live].cpu().numpy().tobytes() == p0.tobytes()
            assert not buf.exp_avg[live].any() and not buf.exp_avg_sq[live].any()
            assert u16(buf.param_shard).tobytes() == w0.tobytes()
            continue

        assert (res["overflow"], res["skipped"], res["step"]) == (0, 1, 1), res
        live = buf.live()
        assert live == (1 if path == "fused-layers" else 0)
        got_p = buf.master[live].cpu().numpy()
        got_m = buf.exp_avg[live].cpu().numpy()
        got_v = buf.exp_avg_sq[live].cpu().numpy()
        got_w = u16(buf.param_shard)

        def check(c):
            lo, n = c
            l = lo // L
            g = _grads_chunk(Nd, synth.BF16, 2, lo - l * L, n, 1e-3, layer=l)
            p = p0[lo:lo + n].copy()
            m = np.zeros(n, np.float32)
            v = np.zeros(n, np.float32)
            reps = [np.zeros(n, np.uint16) for _ in range(Nd)]
            t, ovf, ss = oracle.zero12_step(Nd, n, 0, oracle.BF16, g, p, m, v, reps, hp, 0)
            assert (t, ovf) == (1, 0)
            return (f32_err(got_p[lo:lo + n], p), f32_err(got_m[lo:lo + n], m),
                    f32_err(got_v[lo:lo + n], v), bf16_ulps(got_w[lo:lo + n], reps[0]), ss)
        out = _pmap(check, chunks)
        worst = np.array([o[:4] for o in out], dtype=np.float64).max(axis=0)
        assert worst[0] <= 1e-6 and worst[1] <= 1e-6 and worst[2] <= 1e-6, worst
        assert worst[3] <= 1, worst
        ss = sum(o[4] for o in out)
        assert abs(res["grad_sumsq"] - ss) <= 1e-5 * ss
    del buf
    free()


# ----------------------------------------------------------------------------- wide fan-in

def test_wide_fan_in_2p28_nd64_every_element():
    """N = 2^28, Nd = 64, bf16 gradients ~N(0,1e-3) with 1% (hash-selected) at 1e3 times the
    scale, AdamW step 1000 with m ~ |N(0,1e-3)|, v = N(0,1e-6)^2 -- the fused step as zero_step
    runs it at this size (the TMA-pipelined kernel).  Every element of the fp32 state and of
    rank 0's bf16 replica is compared with the oracle; the other 63 replicas equal rank 0's."""
    N, Nd = 1 << 28, 64
    hp = dict(HP_ADAMW_WIDE)
    tail = float(np.float32(1e-3 * 1e3))
    buf = zero.ZeroBuffers(2, Nd, N)
    fill(buf.master[0], synth.NORMAL, synth.F32, synth.MASTER_STREAM, n=N, sigma=0.02)
    fill(buf.exp_avg[0], synth.ABS, synth.F32, synth.M_STREAM, n=N, sigma=1e-3)
    fill(buf.exp_avg_sq[0], synth.SQUARE, synth.F32, synth.V_STREAM, n=N, sigma=1e-6)
    buf.init_workspace(999)
    buf.sync_params_from_master()
    for r in range(Nd):
        fill(buf.grads[r], synth.HEAVY, synth.BF16, synth.grad_stream(1, r), sigma=1e-3,
             tail_sigma=tail)
    buf.step(zero.hparams(**hp))
    res = buf.result()
    assert (res["overflow"], res["step"]) == (0, 1000), res
    live = buf.live()
    assert live == 1
    for r in range(1, Nd):
        assert torch.equal(buf.params[r].view(torch.int16), buf.params[0].view(torch.int16))
    got_p = buf.master[live].cpu().numpy()
    got_m = buf.exp_avg[live].cpu().numpy()
    got_v = buf.exp_avg_sq[live].cpu().numpy()
    got_w = u16(buf.params[0])

    def check(c):
        lo, n = c
        g = _grads_chunk(Nd, synth.BF16, 1, lo, n, 1e-3, kind=synth.HEAVY, tail=tail)
        p = synth.fill_host(synth.NORMAL, synth.F32, SEED, synth.MASTER_STREAM, n, sigma=0.02,
                            first=lo)
        m = synth.fill_host(synth.ABS, synth.F32, SEED, synth.M_STREAM, n, sigma=1e-3, first=lo)
        v = synth.fill_host(synth.SQUARE, synth.F32, SEED, synth.V_STREAM, n, sigma=1e-6,
                            first=lo)
        reps = [np.zeros(n, np.uint16) for _ in range(Nd)]
        t, ovf, ss = oracle.zero12_step(Nd, n, 0, oracle.BF16, g, p, m, v, reps, hp, 999)
        assert (t, ovf) == (1000, 0)
        return (f32_err(got_p[lo:lo + n], p), f32_err(got_m[lo:lo + n], m),
                f32_err(got_v[lo:lo + n], v), bf16_ulps(got_w[lo:lo + n], reps[0]), ss)
    out = _pmap(check, [(lo, CHUNK) for lo in range(0, N, CHUNK)])
    worst = np.array([o[:4] for o in out], dtype=np.float64).max(axis=0)
    assert worst[0] <= 1e-6 and worst[1] <= 1e-6 and worst[2] <= 1e-6, worst
    assert worst[3] <= 1, worst
    ss = sum(o[4] for o in out)
    assert abs(res["grad_sumsq"] - ss) <= 1e-5 * ss
    del buf
    free()


# ----------------------------------------------------------------------------- ZeRO-1/2, several steps

def _zero12_every_element(stage, Nd, N, steps, hp, gdt, sigma, bucket=0, inject=None):
    """Run `steps` zero_step calls of stage 1/2 (fused path; bucketed if bucket) on the device,
    then compare the final fp32 state and rank 0's bf16 replica element by element with the
    oracle run over every chunk for the same steps (the other replicas must equal rank 0's).
    inject = (step, (rank, index)): +inf planted there; that step must be skipped."""
    sdt = synth.BF16 if gdt == zero.ZERO_BF16 else synth.FP16
    odt = oracle.BF16 if gdt == zero.ZERO_BF16 else oracle.FP16
    inf_bits = 0x7F80 if sdt == synth.BF16 else 0x7C00
    chp = zero.hparams(**hp)
    buf = zero.ZeroBuffers(stage, Nd, N, grad_dtype=gdt)
    assert buf.Np == N  # the workloads here are multiples of Nd: no padding
    fill(buf.master[0], synth.NORMAL, synth.F32, synth.MASTER_STREAM, n=N, sigma=0.02)
    buf.init_workspace(0)
    buf.sync_params_from_master()
    for k in range(1, steps + 1):
        for r in range(Nd):
            fill(buf.grads[r], synth.NORMAL, sdt, synth.grad_stream(k, r), sigma=sigma)
        if inject and k == inject[0]:
            buf.grads[inject[1][0]].view(torch.int16)[inject[1][1]] = inf_bits
        buf.step(chp, bucket=bucket)
    res = buf.result()
    skipped = {inject[0]} if inject else set()
    assert (res["step"], res["skipped"]) == (steps - len(skipped), len(skipped)), res
    live = buf.live()
    for r in range(1, Nd):
        assert torch.equal(buf.params[r].view(torch.int16), buf.params[0].view(torch.int16))
    got_p = buf.master[live].cpu().numpy()
    got_m = buf.exp_avg[live].cpu().numpy()
    got_v = buf.exp_avg_sq[live].cpu().numpy()
    got_w = u16(buf.params[0])
    del buf
    free()
    chunks = [(lo, min(CHUNK, N - lo)) for lo in range(0, N, CHUNK)]
    assert all(n % Nd == 0 for _, n in chunks)  # every chunk is its own unpadded partition

    def grads(k, lo, n):
        g = _grads_chunk(Nd, sdt, k, lo, n, sigma)
        if inject and k == inject[0]:
            rank, idx = inject[1]
            if lo <= idx < lo + n:
                g[rank][idx - lo] = inf_bits
        return g

    for k in sorted(skipped):  # the oracle's reduce-scatter decides the skip
        assert any(_pmap(lambda c: oracle.reduce_scatter(Nd, c[1], odt, grads(k, *c), hp)[1],
                         chunks)), "the oracle does not skip step %d" % k

    def check(c):
        lo, n = c
        p = synth.fill_host(synth.NORMAL, synth.F32, SEED, synth.MASTER_STREAM, n, sigma=0.02,
                            first=lo)
        m = np.zeros(n, np.float32)
        v = np.zeros(n, np.float32)
        reps = [np.zeros(n, np.uint16) for _ in range(Nd)]
        t, ss = 0, 0.0
        for k in range(1, steps + 1):
            if k in skipped:  # a skipped step changes nothing
                continue
            t, ovf, ss = oracle.zero12_step(Nd, n, 0, odt, grads(k, lo, n), p, m, v, reps, hp, t)
            assert ovf == 0
        return (f32_err(got_p[lo:lo + n], p), f32_err(got_m[lo:lo + n], m),
                f32_err(got_v[lo:lo + n], v), bf16_ulps(got_w[lo:lo + n], reps[0]), ss)
    out = _pmap(check, chunks)
    worst = np.array([o[:4] for o in out], dtype=np.float64).max(axis=0)
    assert worst[0] <= 1e-6 and worst[1] <= 1e-6 and worst[2] <= 1e-6, worst
    assert worst[3] <= 1, worst
    ss = sum(o[4] for o in out)  # the last step's sum of squares
    assert abs(res["grad_sumsq"] - ss) <= 1e-5 * ss


def test_zero1_gpt2_small_ten_steps_every_element():
    """N = 124,439,808 (GPT-2 small), Nd = 8, ZeRO-1, 10 AdamW steps (lr 6e-4, wd 0.01), fresh
    bf16 gradients ~N(0,1e-3) every step, bf16 weights all-gathered to 8 replicas each step."""
    _zero12_every_element(1, 8, 124_439_808, 10, dict(HP_ADAMW_GPT2), zero.ZERO_BF16, 1e-3)


def test_zero2_2p28_nd8_two_steps_every_element():
    """The default bench workload: N = 2^28, Nd = 8, bf16 gradients ~N(0,1e-3), AdamW (lr 1e-3,
    wd 0.01), two steps through the fused kernel."""
    _zero12_every_element(2, 8, 1 << 28, 2, dict(HP_ADAMW_WIDE), zero.ZERO_BF16, 1e-3)


def test_zero2_1p3b_fp16_buckets_overflow_every_element():
    """N = 1.3e9 in 25M-element buckets (52), Nd = 16, fp16 gradients ~N(0,1e-4)*1024 carrying
    loss scale 1024; +inf at the seeded (rank, index) on step 3, which must be skipped; 5 AdamW
    steps (the TMA-pipelined kernel at this fan-in)."""
    N, Nd = 1_300_000_000, 16
    site = synth.inject_site(SEED, Nd, N)
    _zero12_every_element(2, Nd, N, 5, dict(HP_ADAMW_FP16_LS1024), zero.ZERO_FP16, 1e-4 * 1024,
                          bucket=25_000_000, inject=(3, site))
