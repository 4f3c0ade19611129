"""Pins of the oracle's dynamic loss scaler and global-norm clipping (no GPU).

The pages only name mixed precision; the readings (backoff/growth loss scaling, clipping by
the global 2-norm) are pinned to library routines that implement the same rules:
torch._amp_update_scale_ (the update inside torch.cuda.amp.GradScaler, which runs on CPU) and
torch.nn.utils.clip_grad_norm_ followed by torch.optim.AdamW; plus a closed form of clipping.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

RNG = np.random.default_rng(99)


@pytest.mark.parametrize("growth,backoff,interval", [(2.0, 0.5, 1), (2.0, 0.5, 3), (4.0, 0.25, 7)])
def test_scaler_matches_torch_amp_update_scale(growth, backoff, interval):
    flags = RNG.random(400) < 0.15
    s_t = torch.tensor([65536.0], dtype=torch.float32)
    g_t = torch.tensor([0], dtype=torch.int32)
    scale, good = 65536.0, 0
    for f in flags:
        torch._amp_update_scale_(s_t, g_t, torch.tensor([1.0 if f else 0.0]), growth, backoff,
                                 interval)
        scale, good = oracle.scaler_update(scale, good, bool(f), growth, backoff, interval)
        assert scale == float(s_t.item()) and good == int(g_t.item())


def test_clip_coefficient_closed_form():
    g = RNG.normal(0, 1e-3, 10_000).astype(np.float32)
    ss = float((g.astype(np.float64) ** 2).sum())
    norm = np.sqrt(ss)
    for max_norm in (norm / 10, norm / 2, norm * 0.999):
        c = oracle.clip_coef(ss, max_norm)
        clipped = g * np.float32(c)
        # ||g * max_norm / (||g|| + 1e-6)|| = max_norm * ||g|| / (||g|| + 1e-6)
        want = max_norm * norm / (norm + 1e-6)
        assert np.sqrt((clipped.astype(np.float64) ** 2).sum()) == pytest.approx(want, rel=1e-6)
    assert oracle.clip_coef(ss, norm * 2) == 1.0  # below the bound: untouched
    assert oracle.clip_coef(ss, 0.0) == 1.0        # clipping off


def _grads(Nd, N, dtype, sigma, step=1):
    return [synth.fill_host(synth.NORMAL, dtype, synth.SEED, synth.grad_stream(step, r), N,
                            sigma=sigma) for r in range(Nd)]


def test_clipped_step_matches_torch_clip_then_adamw():
    """Nd = 1, unit loss scale: the step is clip_grad_norm_ then AdamW on the fp32 gradient."""
    N = 5000
    hp = dict(lr=1e-3, weight_decay=0.01, loss_scale=1.0, max_grad_norm=0.01)
    p0 = synth.fill_host(synth.NORMAL, synth.F32, synth.SEED, 1, N, sigma=0.02)
    master, m, v = p0.copy(), np.zeros(N, np.float32), np.zeros(N, np.float32)
    reps = [np.zeros(N, np.uint16)]
    tp = torch.nn.Parameter(torch.from_numpy(p0.copy()))
    opt = torch.optim.AdamW([tp], lr=1e-3, weight_decay=0.01, foreach=False, fused=False)
    t = 0
    for k in range(1, 4):
        g16 = _grads(1, N, synth.BF16, 1e-3, k)
        t, ovf, ss, _, _ = oracle.zero12_step_ex(1, N, 0, oracle.BF16, g16, master, m, v, reps,
                                                 hp, t)
        assert ovf == 0 and np.sqrt(ss) > hp["max_grad_norm"]  # clipping is active
        tp.grad = torch.from_numpy(oracle.bf16_to_f32(g16[0]))
        torch.nn.utils.clip_grad_norm_([tp], hp["max_grad_norm"])
        opt.step()
    want = tp.detach().numpy()
    assert np.max(np.abs(master.astype(np.float64) - want)) / np.max(np.abs(want)) < 1e-6


def test_extended_step_reduces_to_the_base_step():
    Nd, N = 3, 777
    S, Np, _ = oracle.partition(N, Nd)
    hp = dict(lr=1e-3, weight_decay=0.01, loss_scale=1.0)
    init = np.zeros(Np, np.float32)
    init[:N] = synth.fill_host(synth.NORMAL, synth.F32, synth.SEED, 1, N, sigma=0.02)
    a = [init.copy(), np.zeros(Np, np.float32), np.zeros(Np, np.float32)]
    b = [init.copy(), np.zeros(Np, np.float32), np.zeros(Np, np.float32)]
    ra = [np.zeros(N, np.uint16) for _ in range(Nd)]
    rb = [np.zeros(N, np.uint16) for _ in range(Nd)]
    ta = tb = 0
    for k in range(1, 4):
        g = _grads(Nd, N, synth.BF16, 1e-3, k)
        ta, oa, sa = oracle.zero12_step(Nd, N, 0, oracle.BF16, g, *a, ra, hp, ta)
        tb, ob, sb, _, _ = oracle.zero12_step_ex(Nd, N, 0, oracle.BF16, g, *b, rb, hp, tb)
        assert (ta, oa, sa) == (tb, ob, sb)
    assert all(x.tobytes() == y.tobytes() for x, y in zip(a, b))


def test_dynamic_scale_equals_static_scale_and_backs_off():
    """With a dynamic scale S the step equals the static-scale step with loss_scale = S; an
    overflow halves S and skips; `interval` clean steps double it."""
    Nd, N = 2, 600
    S_, Np, _ = oracle.partition(N, Nd)
    hp_dyn = dict(lr=1e-3, weight_decay=0.01, dynamic_scale=True, scale_interval=2)
    init = np.zeros(Np, np.float32)
    init[:N] = synth.fill_host(synth.NORMAL, synth.F32, synth.SEED, 1, N, sigma=0.02)
    dyn = [init.copy(), np.zeros(Np, np.float32), np.zeros(Np, np.float32)]
    sta = [init.copy(), np.zeros(Np, np.float32), np.zeros(Np, np.float32)]
    rd = [np.zeros(N, np.uint16) for _ in range(Nd)]
    rs = [np.zeros(N, np.uint16) for _ in range(Nd)]
    scale, good, td, ts = 1024.0, 0, 0, 0
    scales = []
    for k in range(1, 7):
        g = [synth.fill_host(synth.NORMAL, synth.FP16, synth.SEED, synth.grad_stream(k, r), N,
                             sigma=1e-4 * scale) for r in range(Nd)]
        if k == 3:
            g[1][5] = 0x7C00  # +inf in fp16
        used = scale
        td, ovf, _, scale, good = oracle.zero12_step_ex(Nd, N, 0, oracle.FP16, g, *dyn, rd, hp_dyn,
                                                        td, scale, good)
        ts, ovf2, _ = oracle.zero12_step(Nd, N, 0, oracle.FP16, g, *sta, rs,
                                         dict(lr=1e-3, weight_decay=0.01, loss_scale=used), ts)
        assert ovf == ovf2 == (1 if k == 3 else 0)
        scales.append(scale)
    assert all(x.tobytes() == y.tobytes() for x, y in zip(dyn, sta))
    assert scales == [1024.0, 2048.0, 1024.0, 1024.0, 2048.0, 2048.0]


def test_bf16_kept_gradient_equals_rounding_then_update():
    """The bf16-kept reduced gradient variant equals: reduce-scatter (pinned), round to bf16
    (pinned), then the pinned Adam on the rounded values, with the norm of the rounded values."""
    Nd, N = 4, 1001
    S, Np, _ = oracle.partition(N, Nd)
    hp = dict(lr=1e-3, weight_decay=0.01, loss_scale=1.0, bf16_grad=True, max_grad_norm=0.02)
    init = np.zeros(Np, np.float32)
    init[:N] = synth.fill_host(synth.NORMAL, synth.F32, synth.SEED, 1, N, sigma=0.02)
    g16 = _grads(Nd, N, synth.BF16, 1e-3)
    p, m, v = init.copy(), np.zeros(Np, np.float32), np.zeros(Np, np.float32)
    reps = [np.zeros(N, np.uint16) for _ in range(Nd)]
    t, ovf, ss, _, _ = oracle.zero12_step_ex(Nd, N, 0, oracle.BF16, g16, p, m, v, reps, hp, 0)
    g, _, _ = oracle.reduce_scatter(Nd, N, oracle.BF16, g16, hp)
    gr = oracle.bf16_to_f32(oracle.f32_to_bf16(g))
    assert ss == float((gr[:N].astype(np.float64) ** 2).sum())
    gr = (gr * np.float32(oracle.clip_coef(ss, 0.02))).astype(np.float32)
    q, qm, qv = init.copy(), np.zeros(Np, np.float32), np.zeros(Np, np.float32)
    oracle.adam(q[:N], qm[:N], qv[:N], gr[:N], hp, Nd, 1)
    assert ovf == 0 and t == 1 and p.tobytes() == q.tobytes() and m.tobytes() == qm.tobytes()
