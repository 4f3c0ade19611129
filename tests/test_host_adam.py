"""The CPU half of ZeRO-Offload (zero_host_adam, product code that runs on the host) against the
CPU oracle: bit-identical state and bf16 weights for any thread count, clipping factor and step."""

import numpy as np
import pytest

import oracle
import synth
import zero_sharded_optimizer_03_b200 as zero


def _p(a):
    return a.ctypes.data


@pytest.mark.parametrize("nthreads", [1, 3, 0])
@pytest.mark.parametrize("t,wd,coef", [(1, 0.0, 1.0), (7, 0.01, 1.0), (1000, 0.01, 0.37)])
def test_host_adam_matches_oracle(nthreads, t, wd, coef):
    n = 300_001  # several 64K blocks and a ragged tail
    hp = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=wd)
    p = synth.fill_host(synth.NORMAL, synth.F32, synth.SEED, 1, n, sigma=0.02)
    m = synth.fill_host(synth.ABS, synth.F32, synth.SEED, 2, n, sigma=1e-3) if t > 1 else \
        np.zeros(n, np.float32)
    v = synth.fill_host(synth.SQUARE, synth.F32, synth.SEED, 3, n, sigma=1e-6) if t > 1 else \
        np.zeros(n, np.float32)
    g = synth.fill_host(synth.HEAVY, synth.F32, synth.SEED, 4, n, sigma=1e-3, tail_sigma=1.0)
    op, om, ov = p.copy(), m.copy(), v.copy()
    og = (g * np.float32(coef)).astype(np.float32)  # the oracle applies the factor to g first
    oracle.adam(op, om, ov, og, hp, Nd=1, t=t)
    out16 = np.zeros(n, np.uint16)
    zero.zero_host_adam(_p(p), _p(m), _p(v), _p(g), n, zero.hparams(**hp), t, coef, _p(out16),
                        nthreads)
    assert p.tobytes() == op.tobytes()
    assert m.tobytes() == om.tobytes() and v.tobytes() == ov.tobytes()
    assert out16.tobytes() == oracle.f32_to_bf16(op).tobytes()


def test_host_adam_rejects_bad_arguments():
    hp = zero.hparams(1e-3)
    a = np.zeros(16, np.float32)
    for args in [(16, hp, 0, 1.0), (16, hp, 1, 0.0), (16, hp, 1, 1.5), (-1, hp, 1, 1.0)]:
        with pytest.raises(zero.ZeroError):
            zero.zero_host_adam(_p(a), _p(a), _p(a), _p(a), args[0], args[1], args[2], args[3])
    with pytest.raises(zero.ZeroError):
        zero.zero_host_adam(None, _p(a), _p(a), _p(a), 16, hp, 1, 1.0)
