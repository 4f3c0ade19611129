"""Sharded Adam step over real GPUs: one process per GPU, data-parallel rank r owns shard r.

The simulated path (zero_step) keeps all Nd ranks in one GPU.  Here the Nd ranks are the
processes of a torch.distributed process group (NCCL), one per GPU ([P1] §二: each rank updates
the parameters it holds and the updated parameters are all-gathered; [P3] core operations:
ReduceScatter of gradients, AllGather of parameters).  Gradient and weight buffers are allocated
in symmetric memory, so every rank holds the peer-mapped addresses of every rank's buffers; the
library's fused kernel (zero_fused_window) then, for this rank's shard only, reads the Nd
gradient replicas over NVLink and sums them in rank order (the reduce-scatter), updates the
shard's fp32 state, and stores the new bf16 weights into every rank's replica (the all-gather)
-- one kernel, compute and collective together over peer memory.  NCCL combines the ranks'
overflow flags (MAX) and sums of squares (SUM) inside the workspace, on the stream, so that
every rank commits or skips the step alike; the same arithmetic as the single-GPU path, so the
results are bit-identical to it.

This module is host plumbing (buffer set-up and the order of the calls); every step of the
path runs in the library's kernels and in NCCL.  Multicast objects are not used (the kernels do
plain peer loads and stores).
"""
from __future__ import annotations

import os

os.environ.setdefault("TORCH_SYMM_MEM_DISABLE_MULTICAST", "1")
os.environ.setdefault("NCCL_NVLS_ENABLE", "0")

from . import (ZERO_BF16, ZERO_FUSED, ZERO_GATE_ALWAYS, ZERO_NO_TMA,  # noqa: E402
               zero_allgather, zero_end_step_flip, zero_fused_window, zero_partition,
               zero_read_result, zero_repair_window, zero_state_t, zero_workspace_bytes,
               zero_workspace_init)

# byte offsets of the pending overflow flag (int32) and sum of squares (double) in the workspace
PENDING_FLAG_OFFSET = 4
PENDING_SUMSQ_OFFSET = 8


def rank_window(N: int, world: int, rank: int):
    """[lo, hi) of the parameters rank `rank` owns, and the shard length S = ceil(N/world)."""
    S = zero_partition(N, world).S
    lo = min(rank * S, N)
    hi = min(lo + S, N)
    return lo, hi, S


def shard_state(S: int, lo: int, device, torch):
    """This rank's fp32 state: two copies each of master / exp_avg / exp_avg_sq for a shard of S
    elements that starts at global index lo, zero-filled.  Returns (views, bases): views[name][k]
    is copy k's S-element tensor; bases[name][k] is the device address of global element 0, so
    bases + 4*lo addresses the shard's first element (the library indexes the state by global
    position).  Each copy is allocated 3 floats longer and viewed from offset lo % 4, which
    makes every base 16-byte aligned whatever lo is, so the kernels' 16-byte vector path runs
    on every rank's window."""
    off = lo % 4
    views, bases = {}, {}
    for name in ("master", "exp_avg", "exp_avg_sq"):
        views[name], bases[name] = [], []
        for _ in range(2):
            t = torch.zeros(max(S, 1) + 3, dtype=torch.float32, device=device)
            v = t[off:off + max(S, 1)]
            views[name].append(v)
            bases[name].append(v.data_ptr() - 4 * lo)
    return views, bases


def combine_step_totals(flag, sumsq, group=None) -> None:
    """Combine the ranks' pending overflow flags (MAX) and sums of squares (SUM) in place."""
    import torch.distributed as dist
    dist.all_reduce(flag, op=dist.ReduceOp.MAX, group=group)
    dist.all_reduce(sumsq, op=dist.ReduceOp.SUM, group=group)


class DistZero:
    """One rank of a data-parallel job of N parameters over the GPUs of `group`.

    grad  : this rank's full gradient replica (N elements, bf16 or fp16), written by backward
    param : this rank's full bf16 weight replica (N elements), rewritten by every step
    master, exp_avg, exp_avg_sq : this rank's fp32 shard [lo, hi), two copies (the fused pass
            writes the other copy and the end of the step makes it live unless the step
            overflowed)
    """

    def __init__(self, N: int, group=None, grad_dtype: int = ZERO_BF16, device=None,
                 symm=None):
        """device: this rank's GPU (default: the current CUDA device).  symm: the module that
        allocates the peer-mapped buffers (default torch.distributed._symmetric_memory; its
        `empty` and `rendezvous` are all that is used)."""
        import torch
        import torch.distributed as dist
        if symm is None:
            import torch.distributed._symmetric_memory as symm
        self.torch, self.dist, self.group = torch, dist, group
        self.N = N
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.lo, self.hi, self.S = rank_window(N, self.world, self.rank)
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        self.device = torch.device(dev)
        gdt = torch.bfloat16 if grad_dtype == ZERO_BF16 else torch.float16
        n = max(N, 1)
        self.grad = symm.empty(n, dtype=gdt, device=dev)
        self.param = symm.empty(n, dtype=torch.bfloat16, device=dev)
        gname = (group or dist.group.WORLD).group_name
        self._hg = symm.rendezvous(self.grad, gname)
        self._hp = symm.rendezvous(self.param, gname)
        views, bases = shard_state(self.S, self.lo, dev, torch)
        self.master, self.exp_avg, self.exp_avg_sq = (views[k] for k in
                                                      ("master", "exp_avg", "exp_avg_sq"))
        self.ws = torch.zeros(zero_workspace_bytes(), dtype=torch.uint8, device=dev)
        self.flag = self.ws[PENDING_FLAG_OFFSET:PENDING_FLAG_OFFSET + 4].view(torch.int32)
        self.sumsq = self.ws[PENDING_SUMSQ_OFFSET:PENDING_SUMSQ_OFFSET + 8].view(torch.float64)
        self._sync = torch.zeros(1, dtype=torch.int32, device=dev)
        st = zero_state_t()
        st.grad_dtype = grad_dtype
        st.flags = ZERO_FUSED | ZERO_NO_TMA  # plain peer loads / stores
        for q in range(self.world):
            st.grads[q] = int(self._hg.buffer_ptrs[q])
            st.params[q] = int(self._hp.buffer_ptrs[q])
        for k in range(2):  # state indexed by global position: base + lo is its first element
            st.master[k] = bases["master"][k]
            st.exp_avg[k] = bases["exp_avg"][k]
            st.exp_avg_sq[k] = bases["exp_avg_sq"][k]
        st.workspace = self.ws.data_ptr()
        self.state = st

    def stream(self) -> int:
        if self.device.type != "cuda":
            return 0
        return self.torch.cuda.current_stream().cuda_stream

    def init(self, t: int = 0) -> None:
        zero_workspace_init(self.ws.data_ptr(), t, self.stream())

    def publish_weights(self) -> None:
        """Write bf16(master) of this rank's shard into every rank's weight replica (the
        all-gather of the initial weights); every rank calls it."""
        live = self.live()
        base = self.master[live].data_ptr() - 4 * self.lo
        self.barrier()
        zero_allgather(base, [self.state.params[q] for q in range(self.world)], self.world,
                       self.lo, self.hi, ZERO_GATE_ALWAYS, None, self.stream())
        self.barrier()

    def barrier(self) -> None:
        """Stream-ordered barrier: every rank's queued work precedes every rank's next work."""
        self.dist.all_reduce(self._sync, group=self.group)

    def step(self, hp) -> None:
        """One ZeRO step of the whole job (every rank calls it, in the same order)."""
        s = self.stream()
        self.barrier()  # every rank's gradients are complete before peers read them
        zero_fused_window(self.world, self.lo, self.hi, self.state, hp, False, s)
        combine_step_totals(self.flag, self.sumsq, self.group)
        zero_end_step_flip(self.ws.data_ptr(), s)
        zero_repair_window(self.world, self.lo, self.hi, self.state, s)
        self.barrier()  # every rank's stores into the replicas are complete before use

    def result(self) -> dict:
        return zero_read_result(self.ws.data_ptr(), self.stream())

    def live(self) -> int:
        return self.result()["live"]

    def close(self) -> None:
        """Release the symmetric-memory handles (call before destroy_process_group)."""
        self._hg = self._hp = None
