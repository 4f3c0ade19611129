"""Python binding of libzero.so, the B200 sharded mixed-precision Adam step (ZeRO-1/2/3).

Argument marshalling only: every function forwards to the C entry point of the same name in
``include/zero.h`` (device pointers as ints, the CUDA stream as an int handle).  All device
work runs in the library's sm_100a kernels.  If libzero.so has not been built, importing this
package raises ImportError: there is no fallback implementation.

``ZeroBuffers`` is plumbing for callers that hold their state in torch tensors: it allocates
the caller-owned buffers the C API expects (with torch) and fills a ``zero_state_t``.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "ZeroError", "ZeroTimeout", "zero_partition", "zero_workspace_bytes", "zero_workspace_init",
    "zero_read_result", "zero_begin_step", "zero_reduce_scatter", "zero_adam_shard",
    "zero_allgather", "zero_end_step", "zero3_gather_layer", "zero_step",
    "zero_memory_estimate", "zero_comm_volume", "zero_version", "zero_profile_events",
    "zero_test_inject_stall", "zero_loss_scaler_init", "zero_host_adam", "zero_offload_step",
    "zero_fused_window", "zero_end_step_flip", "zero_repair_window",
    "ZeroOffloadBuffers",
    "zero_reduce_scatter_noalloc", "ZERO_NOALLOC_MAX_WINDOW", "hparams", "ZeroBuffers",
    "LIB_PATH", "ZERO_BF16", "ZERO_FP16", "ZERO_FUSED", "ZERO_TWO_PASS", "ZERO_NO_TMA",
    "ZERO_FORCE_TMA", "ZERO_BF16_GRAD_SHARD", "ZERO_FUSED_LAYERS",
    "ZERO_GATE_ALWAYS",
    "ZERO_GATE_NO_OVERFLOW", "ZERO_MAX_ND", "ZERO_OK", "ZERO_EINVAL", "ZERO_ECUDA",
    "ZERO_ENOMEM", "ZERO_ETIMEOUT",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libzero.so")

ZERO_OK, ZERO_EINVAL, ZERO_ECUDA, ZERO_ENOMEM, ZERO_ETIMEOUT = 0, -1, -2, -3, -4
ZERO_MAX_ND = 64
ZERO_BF16, ZERO_FP16 = 0, 1
ZERO_FUSED, ZERO_TWO_PASS, ZERO_NO_TMA, ZERO_FORCE_TMA, ZERO_BF16_GRAD_SHARD = 0, 1, 2, 4, 8
ZERO_FUSED_LAYERS = 16
ZERO_GATE_ALWAYS, ZERO_GATE_NO_OVERFLOW = 0, 1

_i64, _i32, _dbl, _P = ctypes.c_int64, ctypes.c_int32, ctypes.c_double, ctypes.c_void_p


class zero_partition_t(ctypes.Structure):
    _fields_ = [("N", _i64), ("Nd", _i32), ("reserved", _i32), ("S", _i64), ("Np", _i64),
                ("pad", _i64)]


class zero_hparams_t(ctypes.Structure):
    _fields_ = [("lr", _dbl), ("beta1", _dbl), ("beta2", _dbl), ("eps", _dbl),
                ("weight_decay", _dbl), ("loss_scale", _dbl), ("grad_average", _i32),
                ("reserved", _i32), ("max_grad_norm", _dbl)]


class zero_step_result_t(ctypes.Structure):
    _fields_ = [("step", _i64), ("skipped", _i64), ("overflow", _i32), ("live", _i32),
                ("grad_sumsq", _dbl), ("pending_overflow", _i32), ("reserved", _i32),
                ("pending_sumsq", _dbl), ("error", _i32), ("reserved2", _i32),
                ("loss_scale", _dbl), ("good_steps", _i64), ("dynamic_scale", _i32),
                ("reserved3", _i32)]


class zero_state_t(ctypes.Structure):
    _fields_ = [("grad_dtype", _i32), ("flags", _i32),
                ("grads", _P * ZERO_MAX_ND), ("params", _P * ZERO_MAX_ND),
                ("master", _P * 2), ("exp_avg", _P * 2), ("exp_avg_sq", _P * 2),
                ("grad_shard", _P), ("param_shard", _P),
                ("grad_layer_stride", _i64), ("param_layer_stride", _i64),
                ("workspace", _P)]


class zero_rs_summary_t(ctypes.Structure):
    _fields_ = [("overflow", _i32), ("reserved", _i32), ("sumsq", _dbl)]


ZERO_NOALLOC_MAX_CTAS = 16384
ZERO_NOALLOC_MAX_WINDOW = ZERO_NOALLOC_MAX_CTAS * 2048


class zero_offload_state_t(ctypes.Structure):
    _fields_ = [("grad_dtype", _i32), ("host_threads", _i32),
                ("grads", _P * ZERO_MAX_ND), ("params", _P * ZERO_MAX_ND),
                ("grad_dev", _P), ("param_dev", _P), ("grad_host", _P), ("param_host", _P),
                ("master_host", _P), ("exp_avg_host", _P), ("exp_avg_sq_host", _P),
                ("workspace", _P), ("upload_stream", _P)]


class zero_mem_t(ctypes.Structure):
    _fields_ = [("optimizer_states", _dbl), ("gradients", _dbl), ("parameters", _dbl),
                ("total", _dbl)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError("libzero.so is not built (expected at %s); run "
                          "`python -m zero_sharded_optimizer_03_b200.build` or "
                          "__graft_entry__.build()" % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    sig = {
        "zero_last_error": ([], ctypes.c_char_p),
        "zero_version": ([], ctypes.c_char_p),
        "zero_partition": ([_i64, ctypes.c_int, ctypes.POINTER(zero_partition_t)], ctypes.c_int),
        "zero_workspace_bytes": ([], ctypes.c_size_t),
        "zero_workspace_init": ([_P, _i64, _P], ctypes.c_int),
        "zero_read_result": ([_P, ctypes.POINTER(zero_step_result_t), _P], ctypes.c_int),
        "zero_begin_step": ([_P, _P], ctypes.c_int),
        "zero_reduce_scatter": ([_P, ctypes.c_int, ctypes.c_int, _i64, _i64,
                                 ctypes.POINTER(zero_hparams_t), _P, _P, _P], ctypes.c_int),
        "zero_adam_shard": ([_P, _P, _P, _P, _i64, _i64, ctypes.POINTER(zero_hparams_t), _P,
                             _P, _P], ctypes.c_int),
        "zero_allgather": ([_P, _P, ctypes.c_int, _i64, _i64, ctypes.c_int, _P, _P],
                           ctypes.c_int),
        "zero_end_step": ([_P, _P], ctypes.c_int),
        "zero3_gather_layer": ([_P, ctypes.c_int, _i64, _P, ctypes.c_int, _P], ctypes.c_int),
        "zero_step": ([ctypes.c_int, ctypes.c_int, _i64, _i64, ctypes.POINTER(zero_state_t),
                       ctypes.POINTER(zero_hparams_t), _P], ctypes.c_int),
        "zero_memory_estimate": ([_dbl, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                  ctypes.POINTER(zero_mem_t)], ctypes.c_int),
        "zero_comm_volume": ([ctypes.c_int, _dbl, ctypes.c_int], _dbl),
        "zero_profile_events": ([_P, _P], ctypes.c_int),
        "zero_test_inject_stall": ([_i64], ctypes.c_int),
        "zero_loss_scaler_init": ([_P, _dbl, _dbl, _dbl, _i64, _P], ctypes.c_int),
        "zero_fused_window": ([ctypes.c_int, _i64, _i64, ctypes.POINTER(zero_state_t),
                               ctypes.POINTER(zero_hparams_t), ctypes.c_int, _P], ctypes.c_int),
        "zero_end_step_flip": ([_P, _P], ctypes.c_int),
        "zero_repair_window": ([ctypes.c_int, _i64, _i64, ctypes.POINTER(zero_state_t), _P],
                               ctypes.c_int),
        "zero_host_adam": ([_P, _P, _P, _P, _i64, ctypes.POINTER(zero_hparams_t), _i64,
                            ctypes.c_float, _P, ctypes.c_int], ctypes.c_int),
        "zero_offload_step": ([ctypes.c_int, _i64, _i64, ctypes.POINTER(zero_offload_state_t),
                               ctypes.POINTER(zero_hparams_t), _P], ctypes.c_int),
        "zero_reduce_scatter_noalloc": ([_P, ctypes.c_int, ctypes.c_int, _i64, _i64,
                                         ctypes.POINTER(zero_hparams_t), _P, _P, ctypes.c_int,
                                         _P], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    return L


lib = _load()


class ZeroError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__("libzero error %d: %s" % (code, msg))
        self.code = code


class ZeroTimeout(ZeroError):
    """ZERO_ETIMEOUT from zero_read_result: a kernel gave up a bounded wait in an earlier step
    (that step was skipped).  `result` holds the bookkeeping the call still filled in."""

    def __init__(self, code: int, msg: str, result: dict):
        super().__init__(code, msg)
        self.result = result


def _check(rc: int) -> None:
    if rc != ZERO_OK:
        raise ZeroError(rc, lib.zero_last_error().decode())


def _ptrs(ptrs) -> ctypes.Array:
    arr = (_P * max(1, len(ptrs)))()
    for k, p in enumerate(ptrs):
        arr[k] = int(p)
    return arr


def hparams(lr, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, loss_scale=1.0,
            grad_average=True, max_grad_norm=0.0) -> zero_hparams_t:
    return zero_hparams_t(lr, beta1, beta2, eps, weight_decay, loss_scale,
                          1 if grad_average else 0, 0, max_grad_norm)


# ----------------------------------------------------------------------------- entry points

def zero_version() -> str:
    return lib.zero_version().decode()


def zero_partition(N: int, Nd: int) -> zero_partition_t:
    out = zero_partition_t()
    _check(lib.zero_partition(N, Nd, ctypes.byref(out)))
    return out


def zero_workspace_bytes() -> int:
    return int(lib.zero_workspace_bytes())


def zero_workspace_init(ws: int, t: int = 0, stream: int = 0) -> None:
    _check(lib.zero_workspace_init(ws, t, stream))


def zero_read_result(ws: int, stream: int = 0) -> dict:
    """The workspace bookkeeping as a dict.  Raises ZeroTimeout (carrying the dict) while the
    workspace error word is set."""
    out = zero_step_result_t()
    rc = lib.zero_read_result(ws, ctypes.byref(out), stream)
    res = {k: getattr(out, k) for k, _ in zero_step_result_t._fields_
           if not k.startswith("reserved")}
    if rc == ZERO_ETIMEOUT:
        raise ZeroTimeout(rc, lib.zero_last_error().decode(), res)
    _check(rc)
    return res


def zero_begin_step(ws: int, stream: int = 0) -> None:
    _check(lib.zero_begin_step(ws, stream))


def zero_reduce_scatter(grads, dtype: int, Nd: int, lo: int, hi: int, hp: zero_hparams_t,
                        grad_out: int, ws: int, stream: int = 0) -> None:
    _check(lib.zero_reduce_scatter(_ptrs(grads), dtype, Nd, lo, hi, ctypes.byref(hp), grad_out,
                                   ws, stream))


def zero_adam_shard(master: int, exp_avg: int, exp_avg_sq: int, grad: int, lo: int, hi: int,
                    hp: zero_hparams_t, param_out: int | None, ws: int, stream: int = 0) -> None:
    _check(lib.zero_adam_shard(master, exp_avg, exp_avg_sq, grad, lo, hi, ctypes.byref(hp),
                               param_out, ws, stream))


def zero_allgather(master: int, replicas, Nd: int, lo: int, hi: int,
                   gate: int = ZERO_GATE_ALWAYS, ws: int | None = None, stream: int = 0) -> None:
    _check(lib.zero_allgather(master, _ptrs(replicas), Nd, lo, hi, gate, ws, stream))


def zero_reduce_scatter_noalloc(grads, dtype: int, Nd: int, lo: int, hi: int,
                                hp: zero_hparams_t, grad_out: int, summary: int,
                                accumulate: bool = False, stream: int = 0) -> None:
    """Workspace-free reduce-scatter (see include/zero.h): `summary` is a device pointer to a
    zero_rs_summary_t (16 bytes) that receives the window's overflow flag and sum of squares."""
    _check(lib.zero_reduce_scatter_noalloc(_ptrs(grads), dtype, Nd, lo, hi, ctypes.byref(hp),
                                           grad_out, summary, 1 if accumulate else 0, stream))


def zero_fused_window(Nd: int, lo: int, hi: int, state: zero_state_t, hp: zero_hparams_t,
                      finalize: bool = False, stream: int = 0) -> None:
    _check(lib.zero_fused_window(Nd, lo, hi, ctypes.byref(state), ctypes.byref(hp),
                                 1 if finalize else 0, stream))


def zero_end_step_flip(ws: int, stream: int = 0) -> None:
    _check(lib.zero_end_step_flip(ws, stream))


def zero_repair_window(Nd: int, lo: int, hi: int, state: zero_state_t, stream: int = 0) -> None:
    _check(lib.zero_repair_window(Nd, lo, hi, ctypes.byref(state), stream))


def zero_host_adam(master: int, exp_avg: int, exp_avg_sq: int, grad: int, n: int,
                   hp: zero_hparams_t, t: int, clip_coef: float = 1.0,
                   param_out: int | None = None, nthreads: int = 0) -> None:
    """AdamW on host memory (pointers into host arrays), bit-identical to the device kernels."""
    _check(lib.zero_host_adam(master, exp_avg, exp_avg_sq, grad, n, ctypes.byref(hp), t,
                              clip_coef, param_out, nthreads))


def zero_offload_step(Nd: int, N: int, chunk: int, state: zero_offload_state_t,
                      hp: zero_hparams_t, stream: int = 0) -> None:
    _check(lib.zero_offload_step(Nd, N, chunk, ctypes.byref(state), ctypes.byref(hp), stream))


def zero_loss_scaler_init(ws: int, init_scale: float = 65536.0, growth_factor: float = 2.0,
                          backoff_factor: float = 0.5, growth_interval: int = 2000,
                          stream: int = 0) -> None:
    _check(lib.zero_loss_scaler_init(ws, init_scale, growth_factor, backoff_factor,
                                     growth_interval, stream))


def zero_test_inject_stall(unit: int) -> None:
    _check(lib.zero_test_inject_stall(unit))


def zero_profile_events(start_event: int | None, stop_event: int | None) -> None:
    _check(lib.zero_profile_events(start_event, stop_event))


def zero_end_step(ws: int, stream: int = 0) -> None:
    _check(lib.zero_end_step(ws, stream))


def zero3_gather_layer(shards, Nd: int, L: int, out, stream: int = 0) -> None:
    _check(lib.zero3_gather_layer(_ptrs(shards), Nd, L, _ptrs(out), len(out), stream))


def zero_step(stage: int, Nd: int, N: int, bucket: int, state: zero_state_t, hp: zero_hparams_t,
              stream: int = 0) -> None:
    _check(lib.zero_step(stage, Nd, N, bucket, ctypes.byref(state), ctypes.byref(hp), stream))


STAGES = ("DP", "ZeRO-1", "ZeRO-2", "ZeRO-3")


def zero_memory_estimate(N: float, Nd: int, bytes_per_param: int = 2,
                         bytes_per_opt_state: int = 12) -> dict:
    out = (zero_mem_t * 4)()
    _check(lib.zero_memory_estimate(float(N), Nd, bytes_per_param, bytes_per_opt_state, out))
    return {STAGES[s]: {k: getattr(out[s], k) for k, _ in zero_mem_t._fields_} for s in range(4)}


def zero_comm_volume(stage: int, N: float, Nd: int) -> float:
    return float(lib.zero_comm_volume(stage, float(N), Nd))


# ----------------------------------------------------------------------------- torch plumbing

class ZeroBuffers:
    """Caller-owned device buffers of one simulated ZeRO job, allocated with torch.

    stage 1/2: Nd gradient replicas and Nd bf16 weight replicas of N elements; two padded
    copies of master/exp_avg/exp_avg_sq (ZERO_FUSED ping-pongs between them) or one copy plus
    an fp32 gradient shard (ZERO_TWO_PASS).
    stage 3: `layers` layers of `layer_len` elements (the last may be shorter), every layer
    padded to a multiple of Nd; one layer-sized gradient buffer and one gathered-weight
    buffer per rank (reused for every layer unless per_layer_buffers is set); one fp32 state
    copy and a reduced-gradient shard, or, with ZERO_FUSED_LAYERS, two state copies and no
    gradient shard.
    """

    def __init__(self, stage: int, Nd: int, N: int, grad_dtype: int = ZERO_BF16,
                 flags: int = ZERO_FUSED, layer_len: int = 0, per_layer_buffers: bool = False,
                 device: str = "cuda"):
        import torch
        self.torch = torch
        self.stage, self.Nd, self.N, self.flags = stage, Nd, N, flags
        self.grad_dtype = grad_dtype
        gdt = torch.bfloat16 if grad_dtype == ZERO_BF16 else torch.float16
        f32 = dict(dtype=torch.float32, device=device)
        self.ws = torch.zeros(zero_workspace_bytes(), dtype=torch.uint8, device=device)
        st = zero_state_t()
        st.grad_dtype = grad_dtype
        st.flags = flags
        st.workspace = self.ws.data_ptr()
        if stage in (1, 2):
            part = zero_partition(N, Nd)
            self.Np = part.Np
            self.layer_len, self.layers, self.layer_padded = N, 1, [part.Np]
            self.grads = [torch.zeros(N, dtype=gdt, device=device) for _ in range(Nd)]
            self.params = [torch.zeros(N, dtype=torch.bfloat16, device=device)
                           for _ in range(Nd)]
            copies = 1 if flags & ZERO_TWO_PASS else 2
            self.master = [torch.zeros(self.Np, **f32) for _ in range(copies)]
            self.exp_avg = [torch.zeros(self.Np, **f32) for _ in range(copies)]
            self.exp_avg_sq = [torch.zeros(self.Np, **f32) for _ in range(copies)]
            gs_dt = torch.bfloat16 if flags & ZERO_BF16_GRAD_SHARD else torch.float32
            self.grad_shard = (torch.zeros(self.Np, dtype=gs_dt, device=device)
                               if flags & ZERO_TWO_PASS else None)
            self.param_shard = None
        elif stage == 3:
            L = layer_len if layer_len > 0 else N
            self.layer_len = L
            self.layers = (N + L - 1) // L if N > 0 else 0
            self.layer_sizes = [min(L, N - l * L) for l in range(self.layers)]
            self.layer_padded = [zero_partition(x, Nd).Np for x in self.layer_sizes]
            self.Np = sum(self.layer_padded)
            nbuf = N if per_layer_buffers else L
            stride = L if per_layer_buffers else 0
            self.grads = [torch.zeros(max(nbuf, 1), dtype=gdt, device=device) for _ in range(Nd)]
            self.params = [torch.zeros(max(nbuf, 1), dtype=torch.bfloat16, device=device)
                           for _ in range(Nd)]
            fused = bool(flags & ZERO_FUSED_LAYERS)  # two state copies, no gradient shard
            copies = 2 if fused else 1
            self.master = [torch.zeros(self.Np, **f32) for _ in range(copies)]
            self.exp_avg = [torch.zeros(self.Np, **f32) for _ in range(copies)]
            self.exp_avg_sq = [torch.zeros(self.Np, **f32) for _ in range(copies)]
            gs_dt = torch.bfloat16 if flags & ZERO_BF16_GRAD_SHARD else torch.float32
            self.grad_shard = None if fused else torch.zeros(self.Np, dtype=gs_dt, device=device)
            self.param_shard = torch.zeros(self.Np, dtype=torch.bfloat16, device=device)
            st.grad_layer_stride = stride
            st.param_layer_stride = stride
        else:
            raise ValueError("stage must be 1, 2 or 3")
        for r in range(Nd):
            st.grads[r] = self.grads[r].data_ptr()
            st.params[r] = self.params[r].data_ptr()
        for k in range(len(self.master)):
            st.master[k] = self.master[k].data_ptr()
            st.exp_avg[k] = self.exp_avg[k].data_ptr()
            st.exp_avg_sq[k] = self.exp_avg_sq[k].data_ptr()
        if self.grad_shard is not None:
            st.grad_shard = self.grad_shard.data_ptr()
        if self.param_shard is not None:
            st.param_shard = self.param_shard.data_ptr()
        self.state = st

    def stream(self) -> int:
        return self.torch.cuda.current_stream().cuda_stream

    def init_workspace(self, t: int = 0) -> None:
        zero_workspace_init(self.ws.data_ptr(), t, self.stream())

    def step(self, hp: zero_hparams_t, bucket: int = 0) -> None:
        b = bucket if self.stage in (1, 2) else self.layer_len
        zero_step(self.stage, self.Nd, self.N, b, self.state, hp, self.stream())

    def result(self) -> dict:
        return zero_read_result(self.ws.data_ptr(), self.stream())

    def live(self) -> int:
        """Index of the state copy holding the current state (0 on the in-place paths)."""
        if self.stage in (1, 2):
            fused = not (self.flags & ZERO_TWO_PASS)
        else:
            fused = bool(self.flags & ZERO_FUSED_LAYERS)
        return self.result()["live"] if fused else 0

    def sync_params_from_master(self) -> None:
        """Write bf16(master) into every weight replica (stage 1/2) or the bf16 shards
        (stage 3): the all-gather of the initial weights."""
        live = self.live()
        if self.stage in (1, 2):
            zero_allgather(self.master[live].data_ptr(), [p.data_ptr() for p in self.params],
                           self.Nd, 0, self.N, ZERO_GATE_ALWAYS, None, self.stream())
        else:
            zero_allgather(self.master[live].data_ptr(), [self.param_shard.data_ptr()], 1, 0,
                           self.Np, ZERO_GATE_ALWAYS, None, self.stream())


class ZeroOffloadBuffers:
    """Caller-owned buffers of a ZeRO-Offload job, allocated with torch: the Nd device gradient
    and weight replicas, device staging buffers, pinned host staging buffers and the fp32
    optimizer state in (pinned) host memory."""

    def __init__(self, Nd: int, N: int, grad_dtype: int = ZERO_BF16, chunk: int = 1 << 24,
                 host_threads: int = 0, device: str = "cuda"):
        import torch
        self.torch = torch
        self.Nd, self.N, self.chunk = Nd, N, chunk
        gdt = torch.bfloat16 if grad_dtype == ZERO_BF16 else torch.float16
        n = max(N, 1)
        self.ws = torch.zeros(zero_workspace_bytes(), dtype=torch.uint8, device=device)
        self.grads = [torch.zeros(n, dtype=gdt, device=device) for _ in range(Nd)]
        self.params = [torch.zeros(n, dtype=torch.bfloat16, device=device) for _ in range(Nd)]
        self.grad_dev = torch.zeros(n, dtype=torch.float32, device=device)
        self.param_dev = torch.zeros(n, dtype=torch.bfloat16, device=device)
        pin = dict(pin_memory=True)
        self.grad_host = torch.zeros(n, dtype=torch.float32, **pin)
        self.param_host = torch.zeros(n, dtype=torch.bfloat16, **pin)
        self.master = torch.zeros(n, dtype=torch.float32, **pin)
        self.exp_avg = torch.zeros(n, dtype=torch.float32, **pin)
        self.exp_avg_sq = torch.zeros(n, dtype=torch.float32, **pin)
        self.upload = torch.cuda.Stream()
        st = zero_offload_state_t()
        st.grad_dtype = grad_dtype
        st.host_threads = host_threads
        for r in range(Nd):
            st.grads[r] = self.grads[r].data_ptr()
            st.params[r] = self.params[r].data_ptr()
        st.grad_dev = self.grad_dev.data_ptr()
        st.param_dev = self.param_dev.data_ptr()
        st.grad_host = self.grad_host.data_ptr()
        st.param_host = self.param_host.data_ptr()
        st.master_host = self.master.data_ptr()
        st.exp_avg_host = self.exp_avg.data_ptr()
        st.exp_avg_sq_host = self.exp_avg_sq.data_ptr()
        st.workspace = self.ws.data_ptr()
        st.upload_stream = self.upload.cuda_stream
        self.state = st

    def stream(self) -> int:
        return self.torch.cuda.current_stream().cuda_stream

    def init_workspace(self, t: int = 0) -> None:
        zero_workspace_init(self.ws.data_ptr(), t, self.stream())

    def sync_params_from_master(self) -> None:
        """Upload bf16(master) into every device weight replica (the initial all-gather)."""
        staging = self.master.to(self.grad_dev.device, non_blocking=False)
        zero_allgather(staging.data_ptr(), [p.data_ptr() for p in self.params], self.Nd, 0,
                       self.N, ZERO_GATE_ALWAYS, None, self.stream())
        self.torch.cuda.current_stream().synchronize()

    def step(self, hp: zero_hparams_t) -> None:
        zero_offload_step(self.Nd, self.N, self.chunk, self.state, hp, self.stream())

    def result(self) -> dict:
        return zero_read_result(self.ws.data_ptr(), self.stream())
