"""The workspace-free reduce-scatter (zero_reduce_scatter_noalloc).

Some callers cannot give the library a workspace: a plugin inside an application that owns all
device memory through its own arena has no buffer to spare, and a latency-critical caller cannot
call cudaMalloc because it may synchronize the device.  This entry point keeps its scratch in a
fixed array inside the library instead.  These tests check, through the C ABI, that its reduced
gradient equals the CPU oracle's bit for bit and its overflow flag and sum of squares match the
oracle's, on two calls in a row (the second call reuses the scratch left by the first), that it
agrees with the workspace-based zero_reduce_scatter, that it writes nothing outside its window,
and that oversized windows are refused.

This file is named so that pytest collects it after every other test file.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import zero_sharded_optimizer_03_b200 as zero

SEED = synth.SEED


def test_rejects_windows_beyond_the_scratch_limit():
    hp = zero.hparams(1e-3)
    with pytest.raises(zero.ZeroError) as e:
        zero.zero_reduce_scatter_noalloc([16] * 4, zero.ZERO_BF16, 4, 0,
                                         zero.ZERO_NOALLOC_MAX_WINDOW + 1, hp, 16, 16)
    assert e.value.code == zero.ZERO_ENOMEM
    assert "33554432" in str(e.value)


@pytest.mark.gpu
@pytest.mark.parametrize("gdt,Nd,N,windows", [
    (zero.ZERO_BF16, 8, 5_000_011, [(0, 5_000_011), (123, 4_000_000)]),
    (zero.ZERO_FP16, 16, 1 << 25, [(0, 1 << 25), (1 << 24, (1 << 25) - 5)]),
])
def test_noalloc_matches_oracle_and_workspace_reduce_scatter_twice(gdt, Nd, N, windows):
    stream = torch.cuda.current_stream().cuda_stream
    sdt = synth.BF16 if gdt == zero.ZERO_BF16 else synth.FP16
    odt = oracle.BF16 if gdt == zero.ZERO_BF16 else oracle.FP16
    tdt = torch.bfloat16 if gdt == zero.ZERO_BF16 else torch.float16
    hpd = dict(lr=1e-3, loss_scale=1024.0 if gdt == zero.ZERO_FP16 else 1.0)
    hp = zero.hparams(**hpd)
    sigma = 0.1024 if gdt == zero.ZERO_FP16 else 1e-3
    inf_bits = 0x7C00 if sdt == synth.FP16 else 0x7F80
    grads = [torch.empty(N, dtype=tdt, device="cuda") for _ in range(Nd)]
    ptrs = [g.data_ptr() for g in grads]
    ws = torch.zeros(zero.zero_workspace_bytes(), dtype=torch.uint8, device="cuda")
    ref = torch.zeros(N, device="cuda")
    got = torch.empty(N, device="cuda")
    summary = torch.zeros(2, dtype=torch.float64, device="cuda")  # zero_rs_summary_t, 16 bytes
    nan_bits = np.float32(np.nan).view(np.uint32)
    for call, (lo, hi) in enumerate(windows):
        hgrads = [synth.fill_host(synth.NORMAL, sdt, SEED, synth.grad_stream(50 + call, r), N,
                                  sigma=sigma) for r in range(Nd)]
        for r in range(Nd):
            synth.fill_device(ptrs[r], synth.NORMAL, sdt, SEED, synth.grad_stream(50 + call, r), N,
                              sigma, cuda_stream=stream)
        if call == 1:  # an overflow in the second call's window must be reported
            grads[Nd - 1].view(torch.int16)[hi - 1] = inf_bits
            hgrads[Nd - 1][hi - 1] = inf_bits
        want, want_flag, want_ss = oracle.reduce_scatter(Nd, N, odt, hgrads, hpd, lo, hi)
        got.fill_(float("nan"))
        zero.zero_reduce_scatter_noalloc(ptrs, gdt, Nd, lo, hi, hp, got.data_ptr(),
                                         summary.data_ptr(), False, stream)
        zero.zero_workspace_init(ws.data_ptr(), 0, stream)
        zero.zero_reduce_scatter(ptrs, gdt, Nd, lo, hi, hp, ref.data_ptr(), ws.data_ptr(), stream)
        res = zero.zero_read_result(ws.data_ptr(), stream)
        torch.cuda.synchronize()
        g = got.cpu().numpy()
        # bit for bit the oracle's reduced gradient (rank-order fp32 sum, one rounding per op)
        assert g[lo:hi].tobytes() == want[lo:hi].tobytes(), "call %d: reduced gradient" % call
        # and the workspace-based entry point's
        assert torch.equal(got[lo:hi].view(torch.int32), ref[lo:hi].view(torch.int32))
        # nothing written outside the window
        assert (g[:lo].view(np.uint32) == nan_bits).all() and (g[hi:].view(np.uint32) == nan_bits).all()
        flag = int(summary.view(torch.int32)[0].item())
        sumsq = float(summary[1].item())
        assert flag == want_flag == res["pending_overflow"] == (1 if call == 1 else 0)
        if call == 0:
            assert abs(sumsq - want_ss) <= 1e-5 * want_ss
            assert abs(sumsq - res["pending_sumsq"]) <= 1e-5 * want_ss
    # accumulate mode: two halves of a window combine into the whole window's summary
    lo, hi = windows[0]
    mid = (lo + hi) // 2
    hgrads = [synth.fill_host(synth.NORMAL, sdt, SEED, synth.grad_stream(50 + 1, r), N,
                              sigma=sigma) for r in range(Nd)]
    hgrads[Nd - 1][windows[1][1] - 1] = inf_bits  # the device replicas still hold call 1's inf
    want, want_flag, want_ss = oracle.reduce_scatter(Nd, N, odt, hgrads, hpd, lo, hi)
    got.fill_(float("nan"))
    zero.zero_reduce_scatter_noalloc(ptrs, gdt, Nd, lo, mid, hp, got.data_ptr(),
                                     summary.data_ptr(), False, stream)
    zero.zero_reduce_scatter_noalloc(ptrs, gdt, Nd, mid, hi, hp, got.data_ptr(),
                                     summary.data_ptr(), True, stream)
    torch.cuda.synchronize()
    assert int(summary.view(torch.int32)[0].item()) == want_flag == 1
    assert got[lo:hi].cpu().numpy().tobytes() == want[lo:hi].tobytes()
