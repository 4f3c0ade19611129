"""Pins of the CPU oracle against things other than itself (no GPU).

Each test ties one part of the oracle to a fact fixed outside it: brute force over tiny
sizes, exact integer arithmetic, a hand-worked rounding case, a closed form of the first
Adam step, or a library routine (numpy / torch conversions, torch.optim.AdamW) in a special
case.  A plausible slip in the oracle (a dropped term, a swapped beta, a wrong shard bound,
a wrong rounding direction, a reordered sum) fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth

RNG = np.random.default_rng(1234)


# ----------------------------------------------------------------------------- partition

@pytest.mark.parametrize("Nd", range(1, 9))
def test_partition_brute_force(Nd):
    for N in range(0, 65):
        S, Np, pad = oracle.partition(N, Nd)
        s_bf = 0
        while s_bf * Nd < N:  # smallest shard length covering N
            s_bf += 1
        assert S == s_bf and Np == Nd * s_bf and pad == Nd * s_bf - N
        owners = []
        for i in range(N):
            hits = [r for r in range(Nd) if r * S <= i < min((r + 1) * S, N)]
            assert len(hits) == 1
            owners.append(hits[0])
            if S:
                assert oracle.owner(i, S) == hits[0]
        assert owners == sorted(owners)  # shards are contiguous and in rank order


def test_partition_rejects_bad_args():
    with pytest.raises(ValueError):
        oracle.partition(-1, 4)
    with pytest.raises(ValueError):
        oracle.partition(10, 0)


def test_partition_config_sizes():
    # shard lengths of the workloads (ceil(N/Nd)), worked by hand
    assert oracle.partition(1_000_003, 4) == (250_001, 1_000_004, 1)
    assert oracle.partition(124_439_808, 8) == (15_554_976, 124_439_808, 0)
    assert oracle.partition(1_300_000_000, 16) == (81_250_000, 1_300_000_000, 0)
    assert oracle.partition(202_375_168, 8) == (25_296_896, 202_375_168, 0)
    assert oracle.partition(1 << 28, 64) == (1 << 22, 1 << 28, 0)
    assert oracle.partition(5, 4) == (2, 8, 3)  # rank 3 holds only padding


# ----------------------------------------------------------------------------- formats

def test_bf16_decode_all_patterns_vs_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.bf16_to_f32(bits)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).float().numpy()
    same = (ours.view(np.uint32) == ref.view(np.uint32)) | (np.isnan(ours) & np.isnan(ref))
    assert same.all()


def test_f16_decode_all_patterns_vs_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.f16_to_f32(bits)
    ref = bits.view(np.float16).astype(np.float32)
    same = (ours.view(np.uint32) == ref.view(np.uint32)) | (np.isnan(ours) & np.isnan(ref))
    assert same.all()


def test_bf16_rne_hand_cases():
    # bf16 keeps 8 significant bits; at 1.0 its ulp is 2^-7.
    one = 1.0
    cases = [
        (one, 0x3F80),
        (one + 2.0 ** -8, 0x3F80),          # exact tie, kept LSB even -> down
        (one + 3 * 2.0 ** -8, 0x3F82),      # exact tie, kept LSB odd -> up to even
        (one + 2.0 ** -8 + 2.0 ** -20, 0x3F81),  # just above the tie -> up
        (one + 2.0 ** -8 - 2.0 ** -20, 0x3F80),  # just below the tie -> down
        (-(one + 3 * 2.0 ** -8), 0xBF82),
        (3.3895313892515355e38, 0x7F7F),    # largest bf16 stays finite
        (float(np.float32(3.4028234663852886e38)), 0x7F80),  # fp32 max rounds up to inf
        (float("inf"), 0x7F80),
        (0.0, 0x0000),
        (-0.0, 0x8000),
    ]
    for x, want in cases:
        got = int(oracle.f32_to_bf16(np.array([x], dtype=np.float32))[0])
        assert got == want, (x, hex(got), hex(want))
    assert np.isnan(oracle.bf16_to_f32(oracle.f32_to_bf16(np.array([np.nan], np.float32))))[0]


def test_bf16_rne_random_vs_torch():
    bits = RNG.integers(0, 2 ** 32, size=1 << 20, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    ours = oracle.f32_to_bf16(x)
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    nan = np.isnan(x)
    assert (ours[~nan] == ref[~nan]).all()
    assert np.isnan(oracle.bf16_to_f32(ours[nan])).all()


# ----------------------------------------------------------------------------- reduce-scatter

def _bf16(vals):
    return oracle.f32_to_bf16(np.asarray(vals, dtype=np.float32))


def test_reduce_is_in_rank_order():
    # fp32: 2^24 + 1 rounds to 2^24 (tie to even), so rank order gives 2^24 + 0 = 2^24;
    # the reverse order (1 + 1 + 2^24) would give 2^24 + 2.
    grads = [_bf16([2.0 ** 24]), _bf16([1.0]), _bf16([1.0])]
    hp = dict(lr=1e-3, loss_scale=1.0, grad_average=False)
    g, ovf, _ = oracle.reduce_scatter(3, 1, oracle.BF16, grads, hp)
    assert ovf == 0 and g[0] == np.float32(2.0 ** 24)


@pytest.mark.parametrize("Nd", [1, 2, 3, 4])
def test_reduce_scatter_small_integers_exact(Nd):
    for N in range(1, 65):
        ints = RNG.integers(-100, 101, size=(Nd, N))
        grads = [_bf16(ints[q]) for q in range(Nd)]  # |x| <= 100 is exact in bf16
        hp = dict(lr=1e-3, loss_scale=1.0, grad_average=False)
        g, ovf, ss = oracle.reduce_scatter(Nd, N, oracle.BF16, grads, hp)
        S, Np, pad = oracle.partition(N, Nd)
        exact = ints.sum(axis=0)
        assert ovf == 0
        assert (g[:N] == exact.astype(np.float32)).all()
        assert (g[N:] == 0).all()
        assert ss == float((exact.astype(np.int64) ** 2).sum())


def test_reduce_mean_and_loss_scale():
    # mean over 4 ranks with loss scale 1024: inv = 1/4096 is a power of two, so exact
    ints = RNG.integers(-50, 51, size=(4, 37))
    grads = [_bf16(ints[q]) for q in range(4)]
    hp = dict(lr=1e-3, loss_scale=1024.0, grad_average=True)
    g, _, _ = oracle.reduce_scatter(4, 37, oracle.BF16, grads, hp)
    assert (g[:37] == (ints.sum(axis=0) / 4096.0).astype(np.float32)).all()


def test_fp16_gradients_decode():
    vals = np.array([0.5, -0.25, 65504.0, 6.1035156e-05, 5.96e-08], dtype=np.float16)
    grads = [vals.view(np.uint16).copy()]
    hp = dict(lr=1e-3, loss_scale=1.0, grad_average=True)
    g, ovf, _ = oracle.reduce_scatter(1, 5, oracle.FP16, grads, hp)
    assert ovf == 0 and (g[:5] == vals.astype(np.float32)).all()


# ----------------------------------------------------------------------------- Adam

def test_first_step_closed_form():
    """Step 1 from m = v = 0 without decay: m_hat = g and v_hat = g^2 exactly, so
    p1 = p0 - lr * g / (|g| + eps) (Kingma & Ba, 2015, section 2)."""
    lr, eps = 1e-3, 1e-8
    g = np.concatenate([RNG.normal(0, 1e-3, 2000), RNG.normal(0, 1e-9, 200),
                        np.logspace(-11, -1, 50), -np.logspace(-11, -1, 50)]).astype(np.float32)
    p0 = RNG.normal(0, 0.02, g.size).astype(np.float32)
    p, m, v = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
    oracle.adam(p, m, v, g, dict(lr=lr, eps=eps, weight_decay=0.0), Nd=1, t=1)
    g64 = g.astype(np.float64)
    closed = p0.astype(np.float64) - lr * g64 / (np.abs(g64) + eps)
    ulp = np.spacing(np.abs(closed).astype(np.float32)).astype(np.float64)
    assert (np.abs(p - closed) <= 1e-6 * lr + ulp).all()
    assert (np.abs(p - p0) <= lr * (1 + 1e-6)).all()  # |step| <= lr on step 1


def _torch_adamw(p0, m0, v0, grads, lr, betas, eps, wd, step0):
    p = torch.nn.Parameter(torch.from_numpy(p0.copy()))
    opt = torch.optim.AdamW([p], lr=lr, betas=betas, eps=eps, weight_decay=wd, foreach=False,
                            fused=False)
    st = opt.state[p]
    st["step"] = torch.tensor(float(step0))
    st["exp_avg"] = torch.from_numpy(m0.copy())
    st["exp_avg_sq"] = torch.from_numpy(v0.copy())
    for g in grads:
        p.grad = torch.from_numpy(g.copy())
        opt.step()
    return p.detach().numpy(), st["exp_avg"].numpy(), st["exp_avg_sq"].numpy()


@pytest.mark.parametrize("wd,lr,step0", [(0.0, 1e-3, 0), (0.01, 6e-4, 0), (0.01, 1e-3, 999)])
def test_adam_matches_torch_adamw(wd, lr, step0):
    """Nd = 1 with unit loss scale is plain AdamW; torch.optim.AdamW (single-tensor path)
    evaluates the same rule with a different rounding order, so agreement is to a few ulps."""
    n = 4096
    p0 = RNG.normal(0, 0.02, n).astype(np.float32)
    if step0:
        m0 = np.abs(RNG.normal(0, 1e-3, n)).astype(np.float32)
        v0 = (RNG.normal(0, 1e-6, n) ** 2).astype(np.float32)
    else:
        m0 = np.zeros(n, np.float32)
        v0 = np.zeros(n, np.float32)
    grads = [RNG.normal(0, 1e-3, n).astype(np.float32) for _ in range(5)]
    p, m, v = p0.copy(), m0.copy(), v0.copy()
    hp = dict(lr=lr, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=wd)
    for k, g in enumerate(grads):
        oracle.adam(p, m, v, g, hp, Nd=1, t=step0 + k + 1)
    tp, tm, tv = _torch_adamw(p0, m0, v0, grads, lr, (0.9, 0.999), 1e-8, wd, step0)

    def normwise(a, b):  # max error relative to the vector's scale (terms cancel near 0)
        return np.max(np.abs(a.astype(np.float64) - b)) / np.max(np.abs(b))
    assert normwise(p, tp) < 1e-6
    assert normwise(m, tm) < 1e-6
    assert normwise(v, tv) < 1e-6


# ----------------------------------------------------------------------------- full steps

def _rand_grads(Nd, N, dtype, scale=1e-3):
    out = []
    for q in range(Nd):
        x = RNG.normal(0, scale, N).astype(np.float32)
        out.append(synth.to_dtype_bits(x, synth.BF16 if dtype == oracle.BF16 else synth.FP16))
    return out


def _state(N, Np):
    master = np.zeros(Np, np.float32)
    master[:N] = RNG.normal(0, 0.02, N)
    m = np.zeros(Np, np.float32)
    v = np.zeros(Np, np.float32)
    return master, m, v


HP = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, loss_scale=1.0)


@pytest.mark.parametrize("dtype", [oracle.BF16, oracle.FP16])
def test_sharded_equals_data_parallel_bit_exact(dtype):
    """ZeRO changes where state lives, not the arithmetic ([P3] comparisons): every N <= 64,
    Nd <= 4, three steps, sharded ZeRO-1/2 == unsharded all-reduce + Adam, bit for bit."""
    for Nd in range(1, 5):
        for N in range(0, 65):
            S, Np, pad = oracle.partition(N, Nd)
            ms, mm, mv = _state(N, Np)
            ds, dm, dv = ms[:N].copy(), mm[:N].copy(), mv[:N].copy()
            reps_s = [np.zeros(N, np.uint16) for _ in range(Nd)]
            reps_d = [np.zeros(N, np.uint16) for _ in range(Nd)]
            ts = td = 0
            for step in range(3):
                grads = _rand_grads(Nd, N, dtype)
                ts, ovs, sss = oracle.zero12_step(Nd, N, 0, dtype, grads, ms, mm, mv, reps_s, HP,
                                                  ts)
                td, ovd, ssd = oracle.dp_step(Nd, N, dtype, grads, ds, dm, dv, reps_d, HP, td)
                assert (ts, ovs) == (td, ovd) and sss == ssd
            assert ms[:N].tobytes() == ds.tobytes()
            assert mm[:N].tobytes() == dm.tobytes() and mv[:N].tobytes() == dv.tobytes()
            assert (ms[N:] == 0).all() and (mm[N:] == 0).all() and (mv[N:] == 0).all()
            for q in range(Nd):
                assert reps_s[q].tobytes() == reps_d[q].tobytes()
                assert reps_s[q].tobytes() == oracle.f32_to_bf16(ds).tobytes()


def test_bucketed_equals_unbucketed():
    for Nd, N in [(4, 61), (3, 50), (2, 17), (1, 9)]:
        S, Np, _ = oracle.partition(N, Nd)
        grads = _rand_grads(Nd, N, oracle.BF16)
        init = _state(N, Np)
        ref = None
        for bucket in [0, 1, 3, 7, 8, N, Np + 5]:
            master, m, v = (a.copy() for a in init)
            reps = [np.zeros(N, np.uint16) for _ in range(Nd)]
            t, ovf, ss = oracle.zero12_step(Nd, N, bucket, oracle.BF16, grads, master, m, v, reps,
                                            HP, 0)
            got = (master.tobytes(), m.tobytes(), v.tobytes(), t, ovf, ss)
            if ref is None:
                ref = got
            assert got == ref


@pytest.mark.parametrize("bad", [np.inf, -np.inf, np.nan, "inf-inf"])
def test_overflow_skips_whole_step(bad):
    Nd, N = 4, 53
    S, Np, _ = oracle.partition(N, Nd)
    master, m, v = _state(N, Np)
    m[:N] = 1e-4
    v[:N] = 1e-8
    reps = [oracle.f32_to_bf16(master[:N]) for _ in range(Nd)]
    grads = _rand_grads(Nd, N, oracle.BF16)
    if bad == "inf-inf":
        grads[1][7] = 0x7F80  # +inf
        grads[2][7] = 0xFF80  # -inf: the sum is NaN
    else:
        grads[3][N - 1] = oracle.f32_to_bf16(np.array([bad], np.float32))[0]
    snap = [master.tobytes(), m.tobytes(), v.tobytes()] + [r.tobytes() for r in reps]
    t, ovf, ss = oracle.zero12_step(Nd, N, 0, oracle.BF16, grads, master, m, v, reps, HP, 41)
    assert ovf == 1 and t == 41
    assert [master.tobytes(), m.tobytes(), v.tobytes()] + [r.tobytes() for r in reps] == snap


def test_one_bad_bucket_skips_all_buckets():
    Nd, N = 2, 40
    S, Np, _ = oracle.partition(N, Nd)
    master, m, v = _state(N, Np)
    snap = master.tobytes()
    grads = _rand_grads(Nd, N, oracle.FP16)
    grads[0][33] = 0x7C00  # fp16 +inf in the last bucket
    reps = [np.zeros(N, np.uint16) for _ in range(Nd)]
    t, ovf, _ = oracle.zero12_step(Nd, N, 8, oracle.FP16, grads, master, m, v, reps, HP, 0)
    assert ovf == 1 and t == 0 and master.tobytes() == snap


# ----------------------------------------------------------------------------- ZeRO-3

def test_zero3_gather_inverts_partition():
    for Nd in range(1, 6):
        for L in range(0, 40):
            full = RNG.integers(0, 65536, L).astype(np.uint16)
            S, Np, _ = oracle.partition(L, Nd)
            padded = np.zeros(Np, np.uint16)
            padded[:L] = full
            shards = [padded[r * S:(r + 1) * S].copy() for r in range(Nd)]
            assert (oracle.zero3_gather(Nd, L, shards) == full).all()


def test_zero3_equals_data_parallel_per_layer():
    Nd = 4
    layer_len = [13, 40, 1, 27]
    sizes = [oracle.partition(L, Nd) for L in layer_len]
    total = sum(s[1] for s in sizes)
    master = np.zeros(total, np.float32)
    m = np.zeros(total, np.float32)
    v = np.zeros(total, np.float32)
    off = 0
    flat_idx = []
    for L, (S, Np, _) in zip(layer_len, sizes):
        master[off:off + L] = RNG.normal(0, 0.02, L)
        flat_idx.extend(range(off, off + L))
        off += Np
    flat_idx = np.array(flat_idx)
    shard16 = oracle.f32_to_bf16(master)
    N = sum(layer_len)
    dp = [master[flat_idx].copy(), np.zeros(N, np.float32), np.zeros(N, np.float32)]
    t3 = tdp = 0
    for step in range(3):
        grads, gathered, dp_grads = [], [], [np.zeros(0, np.uint16)] * Nd
        per_layer = [_rand_grads(Nd, L, oracle.BF16) for L in layer_len]
        for lg in per_layer:
            grads.extend(lg)
        gathered = [np.zeros(L, np.uint16) for L in layer_len for _ in range(Nd)]
        old16 = shard16.copy()
        t3, ovf, ss3 = oracle.zero3_step(Nd, layer_len, oracle.BF16, grads, master, m, v, shard16,
                                         gathered, HP, t3)
        dp_grads = [np.concatenate([per_layer[l][q] for l in range(len(layer_len))])
                    for q in range(Nd)]
        reps = [np.zeros(N, np.uint16) for _ in range(Nd)]
        tdp, ovd, ssd = oracle.dp_step(Nd, N, oracle.BF16, dp_grads, dp[0], dp[1], dp[2], reps,
                                       HP, tdp)
        assert (t3, ovf) == (tdp, ovd)
        assert math.isclose(ss3, ssd, rel_tol=1e-12)
        assert master[flat_idx].tobytes() == dp[0].tobytes()
        assert m[flat_idx].tobytes() == dp[1].tobytes()
        assert shard16[flat_idx].tobytes() == reps[0].tobytes()
        # the just-in-time gather saw the previous step's weights, in every rank's buffer
        off = 0
        for li, (L, (S, Np, _)) in enumerate(zip(layer_len, sizes)):
            for dst in range(Nd):
                assert (gathered[li * Nd + dst] == old16[off:off + L]).all()
            off += Np


def test_update_elements_matches_full_step():
    Nd, N = 3, 29
    S, Np, _ = oracle.partition(N, Nd)
    master, m, v = _state(N, Np)
    p_e, m_e, v_e = master[:N].copy(), m[:N].copy(), v[:N].copy()
    grads = _rand_grads(Nd, N, oracle.BF16)
    reps = [np.zeros(N, np.uint16) for _ in range(Nd)]
    t, _, _ = oracle.zero12_step(Nd, N, 0, oracle.BF16, grads, master, m, v, reps, HP, 4)
    g_en = np.stack(grads, axis=1)
    out16, _ = oracle.update_elements(Nd, oracle.BF16, g_en, p_e, m_e, v_e, HP, t, skip=False)
    assert p_e.tobytes() == master[:N].tobytes() and (out16 == reps[0]).all()


def test_update_elements_on_a_skipped_step_change_nothing():
    """A skipped step (an overflow anywhere) leaves the sampled elements' state as it was and
    reports the unchanged weights, as the full step does."""
    Nd, N = 3, 29
    S, Np, _ = oracle.partition(N, Nd)
    master, m, v = _state(N, Np)
    grads = _rand_grads(Nd, N, oracle.BF16)
    p0, m0, v0 = master[:N].copy(), m[:N].copy(), v[:N].copy()
    p_e, m_e, v_e = p0.copy(), m0.copy(), v0.copy()
    out16, g = oracle.update_elements(Nd, oracle.BF16, np.stack(grads, axis=1), p_e, m_e, v_e, HP,
                                      5, skip=True, want_grad=True)
    assert (p_e.tobytes(), m_e.tobytes(), v_e.tobytes()) == (p0.tobytes(), m0.tobytes(),
                                                             v0.tobytes())
    assert (out16 == oracle.f32_to_bf16(p0)).all()
    # the clipping variant of the per-element driver skips the same way
    p_x, m_x, v_x = p0.copy(), m0.copy(), v0.copy()
    out16x = oracle.update_elements_ex(Nd, oracle.BF16, np.stack(grads, axis=1), p_x, m_x, v_x,
                                       HP, 5, True, np.float32(0.5))
    assert (p_x.tobytes(), m_x.tobytes(), v_x.tobytes()) == (p0.tobytes(), m0.tobytes(),
                                                             v0.tobytes())
    assert (out16x == oracle.f32_to_bf16(p0)).all()
    # the reduced gradient is still reported (rank-order mean), skip or not
    want = np.zeros(N, np.float32)
    for r in range(Nd):
        want = want + oracle.bf16_to_f32(grads[r])
    assert g.tobytes() == (want * np.float32(1.0 / Nd)).tobytes()
