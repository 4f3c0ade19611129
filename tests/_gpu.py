"""Helpers of the GPU parity tests: device buffers filled by the seeded generator, reads of
sampled elements, and a sampled-element oracle driver (each sampled element is evaluated by
the CPU oracle on its own; the global overflow decision is passed in)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth
import zero_sharded_optimizer_03_b200 as zero

SEED = synth.SEED

# Hyperparameters of the workloads (torch AdamW defaults where a workload states none).
HP_ADAM_LR1E3 = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, loss_scale=1.0)
HP_ADAMW_GPT2 = dict(lr=6e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, loss_scale=1.0)
HP_ADAMW_FP16_LS1024 = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, loss_scale=1024.0)
HP_ADAMW_ZERO3 = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, loss_scale=1.0)
HP_ADAMW_WIDE = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, loss_scale=1.0)

LLAMA7B_LAYER = 4 * 4096 * 4096 + 3 * 4096 * 11008  # q,k,v,o + gate,up,down = 202,375,168


def stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def u16(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def f32(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy() if t.dtype != torch.float32 else t.cpu().numpy()


def at(t: torch.Tensor, idx: np.ndarray) -> np.ndarray:
    sel = t[torch.from_numpy(idx).to(t.device)]
    return u16(sel) if t.dtype in (torch.bfloat16, torch.float16) else sel.cpu().numpy()


def fill(t: torch.Tensor, kind: int, dtype: int, stream_id: int, n: int | None = None,
         sigma: float = 1.0, tail_sigma: float = 0.0, tail_mod: int = 100, first: int = 0,
         offset: int = 0) -> None:
    n = t.numel() - offset if n is None else n
    synth.fill_device(t.data_ptr() + offset * t.element_size(), kind, dtype, SEED, stream_id, n,
                      sigma, tail_sigma, tail_mod, first, stream())


def put_bits(t: torch.Tensor, index: int, bits: int) -> None:
    """Plant one 16-bit pattern (e.g. +inf) in a device tensor (host-made fault injection)."""
    t.view(torch.int16)[index] = torch.tensor(np.array([bits], np.uint16).view(np.int16)[0])


def free() -> None:
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def sample_indices(N: int, n_random: int, extra=(), seed: int = 7) -> np.ndarray:
    rng = np.random.default_rng(seed)
    idx = [rng.integers(0, N, n_random)] if N > 0 else []
    edge = [0, 1, 7, 8, 9, N - 9, N - 8, N - 1, N - 2]
    idx.append(np.array([i for i in list(edge) + list(extra) if 0 <= i < N], dtype=np.int64))
    return np.unique(np.concatenate(idx).astype(np.int64))


def boundaries(period: int, N: int, count: int = 64) -> list:
    out = []
    k = 1
    while k * period < N and len(out) < 3 * count:
        out += [k * period - 1, k * period, k * period + 1]
        k += 1
    return out


class SampledOracle:
    """Tracks sampled elements through steps with the CPU oracle."""

    def __init__(self, idx, Nd, dtype, p, m, v, t0=0):
        self.idx, self.Nd, self.dtype = idx, Nd, dtype
        self.p, self.m, self.v = (np.ascontiguousarray(a, dtype=np.float32).copy()
                                  for a in (p, m, v))
        self.t = t0
        self.out16 = oracle.f32_to_bf16(self.p)

    def step(self, grads_en: np.ndarray, hp: dict, skip: bool) -> np.ndarray:
        """grads_en: uint16 [n, Nd].  Returns the reduced gradient at the samples."""
        out16, g = oracle.update_elements(self.Nd, self.dtype, grads_en, self.p, self.m, self.v,
                                          hp, self.t + 1, skip, want_grad=True)
        if not skip:
            self.t += 1
            self.out16 = out16
        return g


def grads_at(idx, Nd, dtype, step, sigma, kind=synth.NORMAL, tail_sigma=0.0, layer=0):
    cols = [synth.values(kind, dtype, SEED, synth.grad_stream(step, r, layer), idx, sigma,
                         tail_sigma) for r in range(Nd)]
    return np.stack(cols, axis=1)


def assert_f32_close(got: np.ndarray, want: np.ndarray, what: str, rel: float = 1e-6):
    """Max relative error |a-b|/max(|b|, 2^-126) <= rel (expected 0: same operation order)."""
    got = got.astype(np.float32)
    want = want.astype(np.float32)
    nan_ok = np.isnan(got) == np.isnan(want)
    assert nan_ok.all(), "%s: NaN mismatch" % what
    fin = ~np.isnan(want)
    err = np.abs(got[fin].astype(np.float64) - want[fin]) / np.maximum(np.abs(want[fin]),
                                                                       2.0 ** -126)
    assert err.size == 0 or err.max() <= rel, "%s: max rel err %.3g (%d of %d differ)" % (
        what, err.max(), int((err > 0).sum()), err.size)


def assert_bf16_close(got: np.ndarray, want: np.ndarray, what: str, ulps: int = 1):
    """Within `ulps` units in the last place of bf16 (expected 0)."""
    a = got.astype(np.int32)
    b = want.astype(np.int32)
    # map sign-magnitude bit patterns to a monotone integer line
    a = np.where(a & 0x8000, 0x8000 - (a & 0x7FFF), 0x8000 + a)
    b = np.where(b & 0x8000, 0x8000 - (b & 0x7FFF), 0x8000 + b)
    d = np.abs(a - b)
    assert d.size == 0 or d.max() <= ulps, "%s: %d elements differ by > %d ulp" % (
        what, int((d > ulps).sum()), ulps)


def exact_count(got: np.ndarray, want: np.ndarray) -> int:
    return int((got.view(np.uint32 if got.dtype == np.float32 else np.uint16)
                != want.view(np.uint32 if want.dtype == np.float32 else np.uint16)).sum())
