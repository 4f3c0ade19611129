"""The workspace-free reduce-scatter (zero_reduce_scatter_noalloc).

Some callers cannot give the library a workspace: a plugin inside an application that owns all
device memory through its own arena has no buffer to spare, and a latency-critical caller cannot
call cudaMalloc because it may synchronize the device.  This entry point keeps its scratch in a
fixed array inside the library instead.  These tests check, through the C ABI, that it produces
what the workspace-based zero_reduce_scatter produces, on two calls in a row (the second call
reuses the scratch left by the first), and that oversized windows are refused.

This file is named so that pytest collects it after every other test file.
"""
import numpy as np
import pytest
import torch

import synth
import zero_sharded_optimizer_03_b200 as zero

SEED = synth.SEED


def test_rejects_windows_beyond_the_scratch_limit():
    hp = zero.hparams(1e-3)
    with pytest.raises(zero.ZeroError) as e:
        zero.zero_reduce_scatter_noalloc([16] * 4, zero.ZERO_BF16, 4, 0,
                                         zero.ZERO_NOALLOC_MAX_WINDOW + 1, hp, 16, 16)
    assert e.value.code == zero.ZERO_EINVAL
    assert "33554432" in str(e.value)


@pytest.mark.gpu
@pytest.mark.parametrize("gdt,Nd,N,windows", [
    (zero.ZERO_BF16, 8, 5_000_011, [(0, 5_000_011), (123, 4_000_000)]),
    (zero.ZERO_FP16, 16, 1 << 25, [(0, 1 << 25), (1 << 24, (1 << 25) - 5)]),
])
def test_noalloc_matches_workspace_reduce_scatter_twice(gdt, Nd, N, windows):
    stream = torch.cuda.current_stream().cuda_stream
    sdt = synth.BF16 if gdt == zero.ZERO_BF16 else synth.FP16
    tdt = torch.bfloat16 if gdt == zero.ZERO_BF16 else torch.float16
    hp = zero.hparams(1e-3, loss_scale=1024.0 if gdt == zero.ZERO_FP16 else 1.0)
    sigma = 0.1024 if gdt == zero.ZERO_FP16 else 1e-3
    grads = [torch.empty(N, dtype=tdt, device="cuda") for _ in range(Nd)]
    ptrs = [g.data_ptr() for g in grads]
    ws = torch.zeros(zero.zero_workspace_bytes(), dtype=torch.uint8, device="cuda")
    ref = torch.zeros(N, device="cuda")
    got = torch.full((N,), float("nan"), device="cuda")
    summary = torch.zeros(2, dtype=torch.float64, device="cuda")  # zero_rs_summary_t, 16 bytes
    for call, (lo, hi) in enumerate(windows):
        for r in range(Nd):
            synth.fill_device(ptrs[r], synth.NORMAL, sdt, SEED, synth.grad_stream(50 + call, r), N,
                              sigma, cuda_stream=stream)
        if call == 1:  # an overflow in the second call's window must be reported by both
            grads[Nd - 1].view(torch.int16)[hi - 1] = 0x7C00 if sdt == synth.FP16 else 0x7F80
        zero.zero_workspace_init(ws.data_ptr(), 0, stream)
        zero.zero_reduce_scatter(ptrs, gdt, Nd, lo, hi, hp, ref.data_ptr(), ws.data_ptr(), stream)
        want = zero.zero_read_result(ws.data_ptr(), stream)
        zero.zero_reduce_scatter_noalloc(ptrs, gdt, Nd, lo, hi, hp, got.data_ptr(),
                                         summary.data_ptr(), False, stream)
        torch.cuda.synchronize()
        a = got[lo:hi].cpu().numpy()
        b = ref[lo:hi].cpu().numpy()
        fin = np.isfinite(b)
        assert (np.isfinite(a) == fin).all()
        err = np.abs(a[fin].astype(np.float64) - b[fin]) / np.maximum(np.abs(b[fin]), 2.0 ** -126)
        assert err.max() <= 1e-6, "call %d: max rel err %g" % (call, err.max())
        flag = int(summary.view(torch.int32)[0].item())
        sumsq = float(summary[1].item())
        assert flag == want["pending_overflow"] == (1 if call == 1 else 0)
        if call == 0:
            assert abs(sumsq - want["pending_sumsq"]) <= 1e-5 * want["pending_sumsq"]
    # accumulate mode: two halves of a window combine into the whole window's summary
    lo, hi = windows[0]
    mid = (lo + hi) // 2
    zero.zero_reduce_scatter_noalloc(ptrs, gdt, Nd, lo, mid, hp, got.data_ptr(),
                                     summary.data_ptr(), False, stream)
    zero.zero_reduce_scatter_noalloc(ptrs, gdt, Nd, mid, hi, hp, got.data_ptr(),
                                     summary.data_ptr(), True, stream)
    zero.zero_workspace_init(ws.data_ptr(), 0, stream)
    zero.zero_reduce_scatter(ptrs, gdt, Nd, lo, hi, hp, ref.data_ptr(), ws.data_ptr(), stream)
    want = zero.zero_read_result(ws.data_ptr(), stream)
    torch.cuda.synchronize()
    assert int(summary.view(torch.int32)[0].item()) == want["pending_overflow"]
    if not want["pending_overflow"]:
        assert abs(float(summary[1].item()) - want["pending_sumsq"]) <= 1e-5 * want["pending_sumsq"]
    assert torch.equal(got[lo:hi], ref[lo:hi])
