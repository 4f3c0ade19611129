"""The seeded input generator (host side; its device twin is checked in the GPU tests)."""
import numpy as np

import synth


def test_unit_normal_moments_and_range():
    z = synth.unit_normal(synth.SEED, 7, np.arange(1 << 20))
    assert z.dtype == np.float32 and np.abs(z).max() < 6.0
    assert abs(float(z.mean())) < 5e-3 and abs(float(z.var()) - 1.0) < 5e-3
    # Irwin-Hall(12): kurtosis 3 - 1.2/12 = 2.9
    k = float(((z - z.mean()) ** 4).mean() / z.var() ** 2)
    assert abs(k - 2.9) < 0.03


def test_counter_based_index_addressing():
    a = synth.fill_host(synth.NORMAL, synth.F32, 1, 2, 5000, sigma=0.02)
    b = synth.values(synth.NORMAL, synth.F32, 1, 2, np.array([4999, 0, 1234]), sigma=0.02)
    assert (a[[4999, 0, 1234]] == b).all()
    c = synth.fill_host_numpy(synth.NORMAL, synth.F32, 1, 2, 3000, sigma=0.02, first=2000, chunk=777)
    assert (c == a[2000:]).all()
    assert not (synth.fill_host(synth.NORMAL, synth.F32, 1, 3, 100) == a[:100]).all()


def test_kinds():
    idx = np.arange(200000)
    x = synth.values_f32(synth.NORMAL, 5, 9, idx, sigma=1e-3)
    assert (synth.values_f32(synth.ABS, 5, 9, idx, sigma=1e-3) == np.abs(x)).all()
    assert (synth.values_f32(synth.SQUARE, 5, 9, idx, sigma=1e-3) == x * x).all()
    h = synth.values_f32(synth.HEAVY, 5, 9, idx, sigma=1e-3, tail_sigma=1.0, tail_mod=100)
    tail = synth.tail_mask(5, 9, idx, 100)
    assert abs(tail.mean() - 0.01) < 1e-3
    assert (h[~tail] == x[~tail]).all() and (np.abs(h[tail]) >= np.abs(x[tail])).all()
    assert (synth.values_f32(synth.ZERO, 5, 9, idx) == 0).all()


def test_output_types():
    x = synth.values_f32(synth.NORMAL, 5, 9, np.arange(1000), sigma=0.1)
    f16 = synth.to_dtype_bits(x, synth.FP16).view(np.float16)
    assert (f16 == x.astype(np.float16)).all()
    b16 = synth.to_dtype_bits(x, synth.BF16)
    back = (b16.astype(np.uint32) << 16).view(np.float32)
    assert (np.abs(back) <= np.abs(x)).all() and (np.abs(back - x) <= np.abs(x) * 2.0 ** -7).all()


def test_c_and_numpy_implementations_agree():
    for kind in (synth.NORMAL, synth.ABS, synth.SQUARE, synth.HEAVY, synth.ZERO):
        for dtype in (synth.BF16, synth.FP16, synth.F32):
            a = synth.fill_host(kind, dtype, 3, 41, 20_000, sigma=1e-3, tail_sigma=1.0,
                                first=999)
            b = synth.fill_host_numpy(kind, dtype, 3, 41, 20_000, sigma=1e-3, tail_sigma=1.0,
                                      first=999)
            assert a.tobytes() == b.tobytes(), (kind, dtype)


def test_inject_site_in_range():
    r, i = synth.inject_site(synth.SEED, 16, 1_300_000_000)
    assert 0 <= r < 16 and 0 <= i < 1_300_000_000
