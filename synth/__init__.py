"""Seeded synthetic inputs for the ZeRO step: one counter-based generator, three implementations.

This module holds no part of the optimizer's arithmetic.  It serves both the CPU oracle and
the CUDA path: the tests and the benchmark draw every input (gradient replicas, master
weights, moments) from it, either on the host or directly in device memory, all from the
same definition, bit for bit.

Definition (SplitMix64, Steele, Lea & Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014, with the finalizer "variant 13" of Stafford's mix functions):

    GAMMA   = 0x9E3779B97F4A7C15
    mix(z)  = z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27; z *= 0x94D049BB133111EB;
              z ^= z >> 31                                              (mod 2^64)
    out(s, k) = mix(s + (k + 1) * GAMMA)                 k-th output of a generator with state s
    sub(seed, stream) = out(seed, stream)                state of an independent sub-stream

An approximately normal variate with index k of (seed, stream) sums the twelve 16-bit fields
of out(s, 3k), out(s, 3k+1), out(s, 3k+2) (s = sub(seed, stream)) -- an Irwin-Hall(12) sum of
discrete uniforms -- and centres it:  z = (sum - 393210) * 2^-16, exact in fp32, |z| < 6,
mean 0, variance 1 - 2^-32.  The value kinds are (every product one fp32 multiply):

    NORMAL  z * sigma
    ABS     |z * sigma|
    SQUARE  (z * sigma) * (z * sigma)
    HEAVY   z * sigma, except z * tail_sigma where out(sub(seed, stream ^ TAIL), k) % tail_mod == 0
    ZERO    0

and the output is stored as fp32, as fp16 (round to nearest even) or as bf16 (the upper 16
bits of the fp32 value, i.e. rounded toward zero).

Three implementations of this one definition: ``values`` (numpy, the readable reference, used
for sampled indices), ``fill_host`` (C, synth_host.c, for large host arrays) and
``fill_device`` (CUDA, synth.cu).  Tests check that all three agree bit for bit.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
M1 = 0xBF58476D1CE4E5B9
M2 = 0x94D049BB133111EB
TAIL = 1 << 62
MASK = (1 << 64) - 1

# value kinds
NORMAL, ABS, SQUARE, HEAVY, ZERO = 0, 1, 2, 3, 4
# output dtypes (same codes as the library's gradient dtypes; F32 is extra)
BF16, FP16, F32 = 0, 1, 2

SEED = 20261202

_HERE = os.path.dirname(os.path.abspath(__file__))


# ----------------------------------------------------------------------------- host side

def _mix(z: np.ndarray) -> np.ndarray:
    z = z ^ (z >> np.uint64(30))
    z = z * np.uint64(M1)
    z = z ^ (z >> np.uint64(27))
    z = z * np.uint64(M2)
    return z ^ (z >> np.uint64(31))


def _mix_int(z: int) -> int:
    z &= MASK
    z ^= z >> 30
    z = (z * M1) & MASK
    z ^= z >> 27
    z = (z * M2) & MASK
    return z ^ (z >> 31)


def sub_seed(seed: int, stream: int) -> int:
    return _mix_int((seed & MASK) + ((stream + 1) * GAMMA))


def _out(s: int, k: np.ndarray) -> np.ndarray:
    # s + (k+1)*GAMMA mod 2^64, with numpy's wrapping uint64 arithmetic
    kk = k.astype(np.uint64) + np.uint64(1)
    return _mix(np.uint64(s) + kk * np.uint64(GAMMA))


def _fields16(h: np.ndarray) -> np.ndarray:
    m = np.uint64(0xFFFF)
    return ((h & m) + ((h >> np.uint64(16)) & m) + ((h >> np.uint64(32)) & m)
            + (h >> np.uint64(48)))


def unit_normal(seed: int, stream: int, idx: np.ndarray) -> np.ndarray:
    """z for indices idx (int64 array), float32, exact."""
    idx = np.asarray(idx, dtype=np.int64)
    s = sub_seed(seed, stream)
    k3 = idx.astype(np.uint64) * np.uint64(3)
    total = (_fields16(_out(s, k3)) + _fields16(_out(s, k3 + np.uint64(1)))
             + _fields16(_out(s, k3 + np.uint64(2))))
    zi = total.astype(np.int64) - 393210
    return (zi.astype(np.float32) * np.float32(2.0 ** -16)).astype(np.float32)


def tail_mask(seed: int, stream: int, idx: np.ndarray, tail_mod: int) -> np.ndarray:
    s = sub_seed(seed, stream ^ TAIL)
    h = _out(s, np.asarray(idx, dtype=np.int64).astype(np.uint64))
    return (h % np.uint64(tail_mod)) == 0


def values_f32(kind: int, seed: int, stream: int, idx, sigma: float = 1.0,
               tail_sigma: float = 0.0, tail_mod: int = 100) -> np.ndarray:
    """fp32 values of the given kind at indices idx."""
    idx = np.asarray(idx, dtype=np.int64)
    if kind == ZERO:
        return np.zeros(idx.shape, dtype=np.float32)
    z = unit_normal(seed, stream, idx)
    sg = np.float32(sigma)
    if kind == HEAVY:
        scale = np.where(tail_mask(seed, stream, idx, tail_mod), np.float32(tail_sigma), sg)
        return (z * scale.astype(np.float32)).astype(np.float32)
    x = (z * sg).astype(np.float32)
    if kind == NORMAL:
        return x
    if kind == ABS:
        return np.abs(x)
    if kind == SQUARE:
        return (x * x).astype(np.float32)
    raise ValueError("unknown kind %r" % kind)


def to_dtype_bits(x: np.ndarray, dtype: int) -> np.ndarray:
    """Store fp32 values as the generator's output type: uint16 bit patterns for fp16 (round to
    nearest even) and bf16 (upper half of the fp32 word), float32 for F32."""
    if dtype == F32:
        return x.astype(np.float32)
    if dtype == FP16:
        return x.astype(np.float16).view(np.uint16)
    if dtype == BF16:
        return (np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)
    raise ValueError("unknown dtype %r" % dtype)


def values(kind: int, dtype: int, seed: int, stream: int, idx, sigma: float = 1.0,
           tail_sigma: float = 0.0, tail_mod: int = 100) -> np.ndarray:
    return to_dtype_bits(values_f32(kind, seed, stream, idx, sigma, tail_sigma, tail_mod), dtype)


def fill_host_numpy(kind, dtype, seed, stream, n, sigma=1.0, tail_sigma=0.0, tail_mod=100,
                    first=0, chunk=1 << 22) -> np.ndarray:
    """Values for indices first .. first+n-1 with the numpy implementation (slow)."""
    out = np.empty(n, dtype=np.float32 if dtype == F32 else np.uint16)
    for lo in range(0, n, chunk):
        hi = min(n, lo + chunk)
        out[lo:hi] = values(kind, dtype, seed, stream, np.arange(first + lo, first + hi,
                                                                  dtype=np.int64),
                            sigma, tail_sigma, tail_mod)
    return out


def fill_host(kind, dtype, seed, stream, n, sigma=1.0, tail_sigma=0.0, tail_mod=100,
              first=0) -> np.ndarray:
    """Values for indices first .. first+n-1 with the C implementation."""
    out = np.empty(n, dtype=np.float32 if dtype == F32 else np.uint16)
    rc = _host_lib().synth_fill_host(out.ctypes.data, dtype, kind, seed & MASK, stream & MASK,
                                     first, n, float(np.float32(sigma)),
                                     float(np.float32(tail_sigma)), tail_mod)
    if rc != 0:
        raise ValueError("synth_fill_host rejected its arguments")
    return out


# ----------------------------------------------------------------------------- stream ids

def grad_stream(step: int, rank: int, layer: int = 0) -> int:
    """Stream of rank `rank`'s gradient replica at call `step` (layer `layer` for ZeRO-3)."""
    return (step << 32) | (layer << 16) | (rank + 256)


MASTER_STREAM, M_STREAM, V_STREAM = 1, 2, 3


def inject_site(seed: int, Nd: int, N: int):
    """(rank, index) where an overflow is planted: out(sub(seed, 0xC3), 0/1) mod Nd / N."""
    s = sub_seed(seed, 0xC3)
    h = _out(s, np.array([0, 1], dtype=np.int64))
    return int(h[0] % np.uint64(Nd)), int(h[1] % np.uint64(N))


# ----------------------------------------------------------------------------- device side

_SRC = os.path.join(_HERE, "synth.cu")
_SO = os.path.join(_HERE, "libzsynth.so")
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared", "-fmad=false"]


_HOST_SRC = os.path.join(_HERE, "synth_host.c")
_HOST_SO = os.path.join(_HERE, "libzsynth_host.so")


def build(force: bool = False) -> str:
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp.%d" % os.getpid()
        nvcc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
        subprocess.run([nvcc, *NVCC_FLAGS, _SRC, "-o", tmp], check=True)
        os.replace(tmp, _SO)
    if (force or not os.path.exists(_HOST_SO)
            or os.path.getmtime(_HOST_SO) < os.path.getmtime(_HOST_SRC)):
        tmp = _HOST_SO + ".tmp.%d" % os.getpid()
        subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-std=c11", "-fPIC", "-shared",
                        _HOST_SRC, "-o", tmp], check=True)
        os.replace(tmp, _HOST_SO)
    return _SO


_host = None


def _host_lib():
    global _host
    if _host is None:
        if not os.path.exists(_HOST_SO):
            build()
        L = ctypes.CDLL(_HOST_SO)
        L.synth_fill_host.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64,
                                      ctypes.c_int64, ctypes.c_float, ctypes.c_float,
                                      ctypes.c_uint32]
        L.synth_fill_host.restype = ctypes.c_int
        _host = L
    return _host


_dev = None


def _device_lib():
    global _dev
    if _dev is None:
        if not os.path.exists(_SO):
            raise RuntimeError("synth/libzsynth.so is not built; run __graft_entry__.build()")
        L = ctypes.CDLL(_SO)
        L.synth_fill.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_uint64,
                                 ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64,
                                 ctypes.c_float, ctypes.c_float, ctypes.c_uint32,
                                 ctypes.c_void_p]
        L.synth_fill.restype = ctypes.c_int
        _dev = L
    return _dev


def fill_device(ptr: int, kind: int, dtype: int, seed: int, stream: int, n: int,
                sigma: float = 1.0, tail_sigma: float = 0.0, tail_mod: int = 100,
                first: int = 0, cuda_stream: int = 0) -> None:
    """Write values first .. first+n-1 into device memory at ptr (asynchronous)."""
    rc = _device_lib().synth_fill(ptr, dtype, kind, seed & MASK, stream & MASK, first, n,
                                  float(np.float32(sigma)), float(np.float32(tail_sigma)),
                                  tail_mod, cuda_stream)
    if rc != 0:
        raise RuntimeError("synth_fill failed with code %d" % rc)
