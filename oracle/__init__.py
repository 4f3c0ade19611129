"""CPU oracle for the sharded mixed-precision Adam step (ZeRO-1/2/3).

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  Only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` leg of ``bench.py`` may import this package.  The CUDA library
(``zero_sharded_optimizer_03_b200``) never imports or links it, and the two share no code.

The arithmetic lives in ``zero_oracle.c`` (plain single-threaded C, one element per loop
iteration, fp32 round-to-nearest with no contraction); this module only compiles it with gcc
and marshals numpy arrays.  The source comments cite the pages each function follows and
list the readings taken where the pages are silent.

Sources: [P1] "ZeRO 优化器的三个阶段深度对比：显存节省与通信开销的量化分析" (wmrh.cn),
[P2] "ZeRO 优化器：把显存“分”着用" (5688vip.com course note), [P3] "ZeRO Optimization（零冗余优化）"
(ai-master.cc glossary).

Parity status: every function here is pinned by ``tests/test_oracle_*.py`` against values
the pages print, closed forms, brute force or a library special case, except the exact fp32
operation order of the update, which the pages do not fix (it is pinned to within a few
ulps by ``torch.optim.AdamW``; the exact order is the reading stated in ``zero_oracle.c``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "zero_oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")

BF16 = 0
FP16 = 1

CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-Wall", "-Wextra",
          "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile zero_oracle.c into liboracle.so next to it (gcc, no GPU needed)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp.%d" % os.getpid()
        subprocess.run(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _SO)
    return _SO


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        P = ctypes.c_void_p
        i64, i32, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        L.oracle_partition.argtypes = [i64, i32, P]
        L.oracle_partition.restype = i32
        L.oracle_owner.argtypes = [i64, i64]
        L.oracle_owner.restype = i64
        L.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        L.oracle_f32_to_bf16.restype = ctypes.c_uint16
        L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_f32.restype = ctypes.c_float
        L.oracle_f16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_f16_to_f32.restype = ctypes.c_float
        for fn in ("oracle_bf16_array_to_f32", "oracle_f16_array_to_f32",
                   "oracle_f32_array_to_bf16"):
            getattr(L, fn).argtypes = [P, P, i64]
            getattr(L, fn).restype = None
        L.oracle_scalars.argtypes = [P, i32, i64, P]
        L.oracle_scalars.restype = None
        L.oracle_reduce_scatter_window.argtypes = [i32, i64, i32, P, ctypes.c_float, i64, i64,
                                                   P, P, P]
        L.oracle_reduce_scatter_window.restype = None
        L.oracle_adam.argtypes = [P, P, P, P, i64, P]
        L.oracle_adam.restype = None
        L.oracle_allgather.argtypes = [i32, i64, P, P]
        L.oracle_allgather.restype = None
        L.oracle_zero12_step.argtypes = [i32, i64, i64, i32, P, P, P, P, P, P, P, P, P]
        L.oracle_zero12_step.restype = i32
        L.oracle_dp_step.argtypes = [i32, i64, i32, P, P, P, P, P, P, P, P, P]
        L.oracle_dp_step.restype = i32
        L.oracle_zero3_gather.argtypes = [i32, i64, P, P]
        L.oracle_zero3_gather.restype = None
        L.oracle_zero3_step.argtypes = [i32, i32, P, i32, P, P, P, P, P, P, P, P, P, P]
        L.oracle_zero3_step.restype = i32
        L.oracle_update_elements.argtypes = [i32, i64, i32, P, P, P, P, P, P, P, i64, i32]
        L.oracle_update_elements.restype = None
        L.oracle_scaler_update.argtypes = [P, P, i32, dbl, dbl, i64]
        L.oracle_scaler_update.restype = None
        L.oracle_clip_coef.argtypes = [dbl, dbl]
        L.oracle_clip_coef.restype = ctypes.c_float
        L.oracle_zero12_step_ex.argtypes = [i32, i64, i64, i32, P, P, P, P, P, P, P, P, P, P, P]
        L.oracle_zero12_step_ex.restype = i32
        L.oracle_update_elements_ex.argtypes = [i32, i64, i32, P, P, P, P, P, P, i64, i32,
                                                ctypes.c_float]
        L.oracle_update_elements_ex.restype = None
        L.oracle_memory_estimate.argtypes = [dbl, i32, i32, i32, P]
        L.oracle_memory_estimate.restype = None
        L.oracle_comm_volume.argtypes = [i32, dbl, i32]
        L.oracle_comm_volume.restype = dbl
        _lib = L
    return _lib


# ----------------------------------------------------------------------------- helpers

def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _ptr_array(arrays) -> ctypes.Array:
    arr = (ctypes.c_void_p * max(1, len(arrays)))()
    for k, a in enumerate(arrays):
        arr[k] = _ptr(a)
    return arr


def _hp(hp: dict) -> np.ndarray:
    return np.array([hp["lr"], hp.get("beta1", 0.9), hp.get("beta2", 0.999),
                     hp.get("eps", 1e-8), hp.get("weight_decay", 0.0),
                     hp.get("loss_scale", 1.0), 1.0 if hp.get("grad_average", True) else 0.0],
                    dtype=np.float64)


class _Scalars(ctypes.Structure):
    _fields_ = [("inv", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("omb1", ctypes.c_float), ("omb2", ctypes.c_float), ("eps", ctypes.c_float),
                ("decay", ctypes.c_float), ("step_size", ctypes.c_float),
                ("sbc2", ctypes.c_float), ("apply_decay", ctypes.c_int)]


class _Mem(ctypes.Structure):
    _fields_ = [("optimizer_states", ctypes.c_double), ("gradients", ctypes.c_double),
                ("parameters", ctypes.c_double), ("total", ctypes.c_double)]


# ----------------------------------------------------------------------------- API

def partition(N: int, Nd: int):
    """(S, Np, pad): shard length ceil(N/Nd), padded length Nd*S, pad count."""
    out = np.zeros(3, dtype=np.int64)
    if lib().oracle_partition(N, Nd, _ptr(out)) != 0:
        raise ValueError("bad partition arguments N=%r Nd=%r" % (N, Nd))
    return int(out[0]), int(out[1]), int(out[2])


def owner(i: int, S: int) -> int:
    return int(lib().oracle_owner(i, S))


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.uint16)
    out = np.empty(a.shape, dtype=np.float32)
    lib().oracle_bf16_array_to_f32(_ptr(a), _ptr(out), a.size)
    return out


def f16_to_f32(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.uint16)
    out = np.empty(a.shape, dtype=np.float32)
    lib().oracle_f16_array_to_f32(_ptr(a), _ptr(out), a.size)
    return out


def f32_to_bf16(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty(a.shape, dtype=np.uint16)
    lib().oracle_f32_array_to_bf16(_ptr(a), _ptr(out), a.size)
    return out


def scalars(hp: dict, Nd: int, t: int) -> dict:
    s = _Scalars()
    h = _hp(hp)
    lib().oracle_scalars(_ptr(h), Nd, t, ctypes.addressof(s))
    return {name: getattr(s, name) for name, _ in _Scalars._fields_}


def reduce_scatter(Nd: int, N: int, dtype: int, grads, hp: dict, lo: int = 0, hi=None):
    """Reduced fp32 gradient shards (Nd*S floats), overflow flag and sum of squares."""
    S, Np, _ = partition(N, Nd)
    out = np.zeros(Np, dtype=np.float32)
    ovf = ctypes.c_int(0)
    ss = ctypes.c_double(0.0)
    inv = scalars(hp, Nd, 1)["inv"]
    lib().oracle_reduce_scatter_window(Nd, N, dtype, _ptr_array(grads), inv, lo,
                                       Np if hi is None else hi, _ptr(out),
                                       ctypes.byref(ovf), ctypes.byref(ss))
    return out, ovf.value, ss.value


def adam(p, m, v, g, hp: dict, Nd: int, t: int):
    """One in-place update of float32 arrays p, m, v with gradient g at step t."""
    s = _Scalars()
    lib().oracle_scalars(_ptr(_hp(hp)), Nd, t, ctypes.addressof(s))
    lib().oracle_adam(_ptr(p), _ptr(m), _ptr(v), _ptr(g), p.size, ctypes.addressof(s))


def allgather(Nd: int, N: int, master: np.ndarray, replicas) -> None:
    lib().oracle_allgather(Nd, N, _ptr(master), _ptr_array(replicas))


def zero12_step(Nd, N, bucket, dtype, grads, master, m, v, replicas, hp, t):
    """ZeRO-1/2 step in place.  Returns (t, overflow, sumsq)."""
    tt = ctypes.c_int64(t)
    ovf = ctypes.c_int(0)
    ss = ctypes.c_double(0.0)
    rc = lib().oracle_zero12_step(Nd, N, bucket, dtype, _ptr_array(grads), _ptr(master),
                                  _ptr(m), _ptr(v), _ptr_array(replicas), _ptr(_hp(hp)),
                                  ctypes.byref(tt), ctypes.byref(ovf), ctypes.byref(ss))
    if rc != 0:
        raise ValueError("oracle_zero12_step failed")
    return tt.value, ovf.value, ss.value


def dp_step(Nd, N, dtype, grads, master, m, v, replicas, hp, t):
    """Unsharded data-parallel step in place.  Returns (t, overflow, sumsq)."""
    tt = ctypes.c_int64(t)
    ovf = ctypes.c_int(0)
    ss = ctypes.c_double(0.0)
    rc = lib().oracle_dp_step(Nd, N, dtype, _ptr_array(grads), _ptr(master), _ptr(m), _ptr(v),
                              _ptr_array(replicas), _ptr(_hp(hp)), ctypes.byref(tt),
                              ctypes.byref(ovf), ctypes.byref(ss))
    if rc != 0:
        raise ValueError("oracle_dp_step failed")
    return tt.value, ovf.value, ss.value


def zero3_gather(Nd: int, L: int, shards) -> np.ndarray:
    full = np.zeros(L, dtype=np.uint16)
    lib().oracle_zero3_gather(Nd, L, _ptr_array(shards), _ptr(full))
    return full


def zero3_step(Nd, layer_len, dtype, grads, master, m, v, shard16, gathered, hp, t):
    """ZeRO-3 step in place.  grads / gathered: flat lists, layer-major, Nd per layer
    (gathered may be None).  Returns (t, overflow, sumsq)."""
    ll = np.ascontiguousarray(layer_len, dtype=np.int64)
    tt = ctypes.c_int64(t)
    ovf = ctypes.c_int(0)
    ss = ctypes.c_double(0.0)
    gptr = None if gathered is None else _ptr_array(gathered)
    rc = lib().oracle_zero3_step(Nd, len(ll), _ptr(ll), dtype, _ptr_array(grads), _ptr(master),
                                 _ptr(m), _ptr(v), _ptr(shard16), gptr, _ptr(_hp(hp)),
                                 ctypes.byref(tt), ctypes.byref(ovf), ctypes.byref(ss))
    if rc != 0:
        raise ValueError("oracle_zero3_step failed")
    return tt.value, ovf.value, ss.value


def update_elements(Nd, dtype, grads_en, p, m, v, hp, t_new, skip, want_grad=False):
    """Element-wise step for independent sampled elements.  grads_en: uint16 [n, Nd];
    p, m, v: float32 [n] updated in place.  Returns (bf16 weights [n], reduced grad or None)."""
    g = np.ascontiguousarray(grads_en, dtype=np.uint16)
    n = p.size
    out16 = np.empty(n, dtype=np.uint16)
    gout = np.empty(n, dtype=np.float32) if want_grad else None
    lib().oracle_update_elements(Nd, n, dtype, _ptr(g), _ptr(p), _ptr(m), _ptr(v), _ptr(out16),
                                 None if gout is None else _ptr(gout), _ptr(_hp(hp)), t_new,
                                 1 if skip else 0)
    return out16, gout


def scaler_update(scale: float, good: int, overflow: bool, growth: float = 2.0,
                  backoff: float = 0.5, interval: int = 2000):
    """One dynamic loss-scale update.  Returns (scale, good)."""
    sc = ctypes.c_double(scale)
    gd = ctypes.c_int64(good)
    lib().oracle_scaler_update(ctypes.byref(sc), ctypes.byref(gd), 1 if overflow else 0, growth,
                               backoff, interval)
    return sc.value, gd.value


def clip_coef(sumsq: float, max_norm: float) -> float:
    return float(lib().oracle_clip_coef(sumsq, max_norm))


def _hpx(hp: dict) -> np.ndarray:
    return np.concatenate([_hp(hp), np.array(
        [hp.get("max_grad_norm", 0.0), hp.get("scale_growth", 2.0), hp.get("scale_backoff", 0.5),
         float(hp.get("scale_interval", 2000)), 1.0 if hp.get("dynamic_scale", False) else 0.0,
         1.0 if hp.get("bf16_grad", False) else 0.0], dtype=np.float64)])


def zero12_step_ex(Nd, N, bucket, dtype, grads, master, m, v, replicas, hp, t, scale=None, good=0):
    """ZeRO-1/2 step with clipping (hp['max_grad_norm']), the bf16-kept reduced gradient
    (hp['bf16_grad']) and, if hp['dynamic_scale'], the dynamic loss scale `scale` / `good`.
    Returns (t, overflow, sumsq, scale, good)."""
    tt = ctypes.c_int64(t)
    ovf = ctypes.c_int(0)
    ss = ctypes.c_double(0.0)
    sc = ctypes.c_double(hp.get("loss_scale", 1.0) if scale is None else scale)
    gd = ctypes.c_int64(good)
    rc = lib().oracle_zero12_step_ex(Nd, N, bucket, dtype, _ptr_array(grads), _ptr(master), _ptr(m),
                                     _ptr(v), _ptr_array(replicas), _ptr(_hpx(hp)),
                                     ctypes.byref(tt), ctypes.byref(sc), ctypes.byref(gd),
                                     ctypes.byref(ovf), ctypes.byref(ss))
    if rc != 0:
        raise ValueError("oracle_zero12_step_ex failed")
    return tt.value, ovf.value, ss.value, sc.value, gd.value


def update_elements_ex(Nd, dtype, grads_en, p, m, v, hp, t_new, skip, coef):
    g = np.ascontiguousarray(grads_en, dtype=np.uint16)
    out16 = np.empty(p.size, dtype=np.uint16)
    lib().oracle_update_elements_ex(Nd, p.size, dtype, _ptr(g), _ptr(p), _ptr(m), _ptr(v),
                                    _ptr(out16), _ptr(_hp(hp)), t_new, 1 if skip else 0, coef)
    return out16


STAGES = ("DP", "ZeRO-1", "ZeRO-2", "ZeRO-3")


def memory_estimate(N: float, Nd: int, bytes_per_param: int = 2, bytes_per_opt_state: int = 12):
    """Per-GPU model-state memory in GiB, keyed DP / ZeRO-1 / ZeRO-2 / ZeRO-3."""
    out = (_Mem * 4)()
    lib().oracle_memory_estimate(float(N), Nd, bytes_per_param, bytes_per_opt_state, out)
    return {STAGES[s]: {k: getattr(out[s], k) for k, _ in _Mem._fields_} for s in range(4)}


def comm_volume(stage: int, N: float, Nd: int) -> float:
    return float(lib().oracle_comm_volume(stage, float(N), Nd))
