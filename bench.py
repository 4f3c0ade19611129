#!/usr/bin/env python
"""Benchmark of the sharded mixed-precision Adam step (ZeRO) on B200.

One step = one ``zero_step`` call through the C ABI: the reduce-scatter of Nd gradient
replicas, the fp16/bf16 unscale and overflow check, Adam/AdamW on every rank's fp32 shard,
and the bf16 all-gather to the Nd weight replicas, all Nd simulated ranks in this GPU's memory.

Default workload: the fused reduce-scatter + AdamW + all-gather step on N = 2^28 parameters
with Nd = 8 simulated ranks, bf16 gradients ~N(0,1e-3), AdamW (lr 1e-3, wd 0.01).  Inputs are
synthetic, generated on the device by the seeded generator before the timed region (distinct
gradients per step, cycling through as many sets as fit a memory budget); every step reads more
than the 126 MB L2.

Prints one JSON line (rank 0).  Under torchrun (N > 1 GPUs) the ranks are real data-parallel
ranks, one per GPU: rank r owns shard r of the workload's parameters and the fused kernel reads
the peers' gradients and writes every peer's weights over NVLink (zero_sharded_optimizer_03_b200
.dist); the total work is fixed (strong scaling).  Workloads the real-rank path does not cover
(ZeRO-3 layers, offload) run one independent replica per GPU instead (weak scaling).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "params updated/s and achieved HBM GB/s (% of B200 peak) per ZeRO step"

# name -> workload.  bytes_per_param: algorithmic HBM traffic of one step per parameter.
WORKLOADS = {
    "zero1-gpt2-small": dict(
        desc="ZeRO-1 flat N=124,439,808 (GPT-2 small), Nd=8, bf16 grads ~N(0,1e-3), AdamW "
             "lr 6e-4 wd 0.01, bf16 weights all-gathered to 8 replicas",
        stage=1, Nd=8, N=124_439_808, bucket=0, gdt="bf16", sigma=1e-3, kind="normal",
        hp=dict(lr=6e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, loss_scale=1.0)),
    "zero2-2p28-nd8": dict(
        desc="ZeRO-2 flat N=2^28, Nd=8, bf16 grads ~N(0,1e-3), AdamW lr 1e-3 wd 0.01",
        stage=2, Nd=8, N=1 << 28, bucket=0, gdt="bf16", sigma=1e-3, kind="normal",
        hp=dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, loss_scale=1.0)),
    "zero2-1m-nd4": dict(
        desc="ZeRO-2 N=1,000,003 (padded to ceil(N/4)), Nd=4, bf16 grads ~N(0,1e-3), Adam lr 1e-3",
        stage=2, Nd=4, N=1_000_003, bucket=0, gdt="bf16", sigma=1e-3, kind="normal",
        hp=dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, loss_scale=1.0)),
    "zero2-fp16-bucketed": dict(
        desc="ZeRO-2 N=1.3e9 in 25M-element buckets, Nd=16, fp16 grads ~N(0,1e-4)*1024 "
             "(loss scale 1024), AdamW lr 1e-3 wd 0.01",
        stage=2, Nd=16, N=1_300_000_000, bucket=25_000_000, gdt="fp16", sigma=1e-4 * 1024,
        kind="normal",
        hp=dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, loss_scale=1024.0)),
    "zero2-wide-fanin-nd64": dict(
        desc="ZeRO-2 flat N=2^28, Nd=64, bf16 grads ~N(0,1e-3) with 1% x1e3, AdamW step 1000 "
             "with m,v prefilled",
        stage=2, Nd=64, N=1 << 28, bucket=0, gdt="bf16", sigma=1e-3, kind="heavy", t0=999,
        hp=dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, loss_scale=1.0)),
    "zero2-offload-gpt2-small": dict(
        desc="ZeRO-Offload: N=124,439,808 (GPT-2 small), Nd=8, bf16 grads ~N(0,1e-3); "
             "reduce-scatter on the GPU, AdamW (lr 6e-4 wd 0.01) on fp32 state in pinned host "
             "memory, bf16 weights back to 8 replicas, 16M-element chunks",
        stage=2, offload=True, chunk=1 << 24, Nd=8, N=124_439_808, bucket=0, gdt="bf16",
        sigma=1e-3, kind="normal",
        hp=dict(lr=6e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, loss_scale=1.0)),
    "zero3-llama7b": dict(
        desc="ZeRO-3 Llama-7B-shaped: 32 layers of q,k,v,o 4096x4096 + gate,up,down 4096x11008 "
             "(202,375,168 each), Nd=8; per layer gather from 8 bf16 shards and reduce-scatter "
             "8 bf16 grad replicas ~N(0,1e-3) into the fp32 grad shard, then AdamW on the shards",
        stage=3, Nd=8, N=32 * 202_375_168, layer=202_375_168, bucket=202_375_168, gdt="bf16",
        sigma=1e-3, kind="normal",
        hp=dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, loss_scale=1.0)),
}
DEFAULT = "zero2-2p28-nd8"


def bytes_per_param(w, two_pass=False, g16=False, fused_layers=False) -> int:
    Nd = w["Nd"]
    gb = 2 if g16 else 4  # bytes of the kept reduced gradient
    if w["stage"] == 3 and fused_layers:
        # gather: 2 read + 2Nd written; fused pass: 2Nd + 12 read, 12 + 2 (bf16 shard) written
        return (2 + 2 * Nd) + (2 * Nd + 12 + 12 + 2)
    if w["stage"] == 3:
        # gather: 2 read + 2Nd written; RS: 2Nd read + gb written; Adam + cast: gb + 24 + 2
        return (2 + 2 * Nd) + (2 * Nd + gb) + (gb + 24 + 2)
    if two_pass:
        # RS: 2Nd read + gb written; Adam + cast + AG: gb + 24 read/written + 2Nd written
        return (2 * Nd + gb) + (gb + 24 + 2 * Nd)
    # fused step: Nd 2-byte gradient reads, fp32 master/m/v read + write, Nd 2-byte weight writes
    return 2 * Nd + 24 + 2 * Nd


L2_BYTES = 126e6  # B200 L2 capacity
SELF_REPAIR_MAX = 1 << 21  # longest step zero_step runs without an overflow-repair launch

# NVLink figures for the real-rank roofline: a peer copy measured between B200s of an NVSwitch
# node (per direction per GPU) and NVIDIA's nominal link rate, used when MEASURED_PEAKS.json has
# none.
NVLINK_PEER_COPY_GBS = 770.0
NVLINK_NOMINAL_GBS = 900.0


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def nvlink_peak():
    """(GB/s per direction per GPU, source) for NVLink: MEASURED_PEAKS.json if it has a figure,
    else the measured B200 peer copy."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        for key in ("nvlink_gbs", "nvlink_peer_gbs", "p2p_gbs"):
            if key in d:
                return float(d[key]), "measured (MEASURED_PEAKS.json %s)" % key
    return NVLINK_PEER_COPY_GBS, ("measured B200 peer copy, per direction (nominal %g)"
                                  % NVLINK_NOMINAL_GBS)


def traffic_record(kernel: str, workload: str):
    """ncu DRAM bytes per launch of `kernel` on `workload` (profiles/traffic.json), or None when
    no capture exists or a source file of the kernel has changed since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    for rec in json.load(open(path)).get("records", []):
        if rec.get("kernel") != kernel or rec.get("workload") != workload:
            continue
        for rel, sha in rec.get("sources", {}).items():
            if hashlib.sha256(open(os.path.join(ROOT, rel), "rb").read()).hexdigest() != sha:
                return None
        return rec
    return None


def optimizer_instances(stage: int, step_bytes: float) -> int:
    """Independent optimizer instances a workload cycles through so that a step finds none of
    its data in L2 from its previous run: enough that three L2 capacities of other steps' data
    pass between two runs of one instance (at most 64); 1 for steps that large already, and for
    ZeRO-3 (its steps are gigabytes)."""
    if stage == 3 or step_bytes >= 3 * L2_BYTES:
        return 1
    return int(min(64, -(-3 * L2_BYTES // step_bytes)))


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-i", self.gpu_id, "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- CPU baseline

def host_threads() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def cpu_baseline(w, target_s=10.0, steps=1, threads=1, max_bytes=6e9):
    """Time the CPU oracle as it stands on a bounded sample of the workload: the first n
    parameters, split into `threads` contiguous chunks of equal length; each thread runs the
    unmodified, single-threaded oracle step on its own chunk (elements are independent, and the
    sample has no overflow, so every chunk updates exactly as the whole vector would).  n is
    sized for about target_s seconds per step and at most max_bytes of host inputs.  Returns
    (n, [seconds of each step])."""
    from concurrent.futures import ThreadPoolExecutor

    import numpy as np

    import oracle
    import synth
    Nd = w["Nd"]
    odt = oracle.FP16 if w["gdt"] == "fp16" else oracle.BF16
    sdt = synth.FP16 if w["gdt"] == "fp16" else synth.BF16
    kind = synth.HEAVY if w["kind"] == "heavy" else synth.NORMAL
    tail = float(np.float32(w["sigma"] * 1e3)) if w["kind"] == "heavy" else 0.0
    t0 = w.get("t0", 0)

    def make(lo, n):  # inputs of elements lo .. lo+n-1 (n a multiple of Nd: no padding)
        grads = [synth.fill_host(kind, sdt, synth.SEED, synth.grad_stream(1, r), n,
                                 sigma=w["sigma"], tail_sigma=tail, first=lo) for r in range(Nd)]
        p = synth.fill_host(synth.NORMAL, synth.F32, synth.SEED, synth.MASTER_STREAM, n,
                            sigma=0.02, first=lo)
        if t0:
            m = synth.fill_host(synth.ABS, synth.F32, synth.SEED, synth.M_STREAM, n, sigma=1e-3,
                                first=lo)
            v = synth.fill_host(synth.SQUARE, synth.F32, synth.SEED, synth.V_STREAM, n,
                                sigma=1e-6, first=lo)
        else:
            m, v = np.zeros(n, np.float32), np.zeros(n, np.float32)
        return [grads, p, m, v, [np.zeros(n, np.uint16) for _ in range(Nd)]]

    def one_step(n, g, p, m, v, reps, t):
        if w["stage"] == 3:  # the sample is one layer: gather, reduce-scatter, Adam + cast
            sh16 = oracle.f32_to_bf16(p)
            gathered = [np.zeros(n, np.uint16) for _ in range(Nd)]
            return oracle.zero3_step(Nd, [n], odt, g, p, m, v, sh16, gathered, w["hp"], t)[0]
        bucket = min(w.get("bucket", 0), n)
        return oracle.zero12_step(Nd, n, bucket, odt, g, p, m, v, reps, w["hp"], t)[0]

    n0 = 1 << 16
    d0 = make(0, n0)
    tt = time.perf_counter()
    one_step(n0, *d0, t0)
    rate0 = n0 / (time.perf_counter() - tt)
    host_bytes = 4 * Nd + 12 + (2 if w["stage"] == 3 else 0)
    n = int(min(w["N"], rate0 * target_s * threads, max_bytes / host_bytes))
    unit = threads * Nd
    nc = max(1, n // unit) * Nd  # elements per thread
    with ThreadPoolExecutor(max_workers=threads) as ex:
        data = list(ex.map(lambda c: make(c * nc, nc), range(threads)))
        tcount = [t0] * threads
        times = []
        for _ in range(steps):
            tt = time.perf_counter()
            tcount = list(ex.map(lambda c: one_step(nc, *data[c], tcount[c]), range(threads)))
            times.append(time.perf_counter() - tt)
    return nc * threads, times


def cpu_baseline_record(w, target_s=10.0):
    """The cpu_baseline object of the bench line: the oracle on every host core (primary) and
    on one core, each on its own bounded sample of the workload."""
    ncores = host_threads()
    n1, t1 = cpu_baseline(w, target_s=target_s, threads=1)
    nA, tA = cpu_baseline(w, target_s=target_s / 2, threads=ncores)
    return {"value": nA / tA[0], "unit": "params/s", "cores": ncores, "kind": "oracle",
            "sample": "first %d of %d parameters, Nd=%d, one ZeRO step, %d contiguous chunks, "
                      "one oracle call per core (%.1f s)" % (nA, w["N"], w["Nd"], ncores, tA[0]),
            "single_core": {"value": n1 / t1[0], "unit": "params/s", "cores": 1,
                            "sample": "first %d of %d parameters, Nd=%d, one ZeRO step (%.1f s)"
                                      % (n1, w["N"], w["Nd"], t1[0])}}


# ----------------------------------------------------------------------------- ranks

def max_over_ranks(values, dist=None, device=None):
    """Element-wise maximum of a list of floats over all ranks (identity without dist).  Every
    rank must call it with the same number of values, in the same order."""
    if dist is None:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def whole_job_rate(units_per_rank, world, ms_per_step):
    """Units all ranks process per second when each rank processes units_per_rank per step and
    the slowest rank takes ms_per_step (replicas: per-GPU work is fixed)."""
    return world * units_per_rank / (ms_per_step / 1e3)


# ----------------------------------------------------------------------------- offload

def run_offload(args, w, world, rank, dist, dev, config):
    """ZeRO-Offload step: reduce-scatter on the GPU, AdamW on host memory, weights back."""
    import numpy as np
    import torch

    import synth
    import zero_sharded_optimizer_03_b200 as zero
    Nd, N = w["Nd"], w["N"]
    steps = min(args.steps, 20)  # host-bound steps of ~0.1 s: keep the timed region short
    s = torch.cuda.current_stream()
    sp = s.cuda_stream
    buf = zero.ZeroOffloadBuffers(Nd, N, chunk=w["chunk"], host_threads=0)
    buf.master.numpy()[:] = synth.fill_host(synth.NORMAL, synth.F32, synth.SEED,
                                            synth.MASTER_STREAM, N, sigma=0.02)
    buf.init_workspace(0)
    buf.sync_params_from_master()
    for r in range(Nd):
        synth.fill_device(buf.grads[r].data_ptr(), synth.NORMAL, synth.BF16, synth.SEED,
                          synth.grad_stream(1, r), N, w["sigma"], cuda_stream=sp)
    hp = zero.hparams(**w["hp"])
    for _ in range(args.warmup):
        buf.step(hp)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    wall = time.perf_counter()
    t0.record(s)
    for _ in range(steps):
        buf.step(hp)
    t1.record(s)
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall
    ms_total = max_over_ranks([t0.elapsed_time(t1)], dist, dev)[0]
    res = buf.result()
    assert res["overflow"] == 0 and res["skipped"] == 0, res
    ms = ms_total / steps
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_record(w)
    host_bytes = 30 * N  # grad 4 read, master/m/v 12 read + 12 written, bf16 weights 2 written
    pcie_bytes = 6 * N   # fp32 gradient down (4), bf16 weights up (2)
    if rank == 0:
        config["path"] = "offload"
        config["kernel"] = "reduce_scatter_kernel + host AdamW + gather_layer_kernel"
        config["host_threads"] = os.cpu_count()
        line = {"metric": METRIC, "value": whole_job_rate(N, world, ms), "unit": "params/s",
                "n_gpus": world, "steps": steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic", "config": config,
                "roofline": {"bound": "host", "achieved": host_bytes / (ms / 1e3) / 1e9,
                             "peak": None, "unit": "GB/s", "frac": None, "traffic": None,
                             "pcie_gbs": pcie_bytes / (ms / 1e3) / 1e9,
                             "note": "host-memory and PCIe bound; no measured host peak"},
                "cpu_baseline": cpu, "e2e": None, "clocks": None,
                "gpu_launches": steps * (-(-N // w["chunk"]) * 2 + 1),
                "wall_s": wall}
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


# ----------------------------------------------------------------------------- real ranks

def dist_roofline(S: int, world: int, hbm_gbs: float, link_gbs: float):
    """Per-rank bytes and ideal time of the real-rank fused step for a shard of S elements over
    `world` GPUs: HBM carries the rank's own gradient and weight replica windows and its fp32
    state (2 + 24 + 2 bytes per element); NVLink carries the peers' gradients in and the new
    weights out to the peers (2 + 2 bytes per element per peer).  Returns (hbm_bytes,
    link_bytes, bound, ideal_seconds): the slower of the two is the bound."""
    hbm_bytes = S * (2 + 24 + 2)
    link_bytes = S * 2 * (world - 1) * 2
    t_hbm = hbm_bytes / (hbm_gbs * 1e9)
    t_link = link_bytes / (link_gbs * 1e9)
    return hbm_bytes, link_bytes, ("nvlink" if t_link > t_hbm else "hbm"), max(t_hbm, t_link)


def run_dist(args, w, config):
    """Data parallelism over real GPUs (one process per GPU, torchrun): rank r owns shard r of
    the workload's N parameters and runs the fused kernel over peer memory (symmetric memory);
    Nd = the number of GPUs.  Total work is fixed: strong scaling."""
    import datetime

    import torch
    import torch.distributed as dist

    import synth
    import zero_sharded_optimizer_03_b200 as zero
    from zero_sharded_optimizer_03_b200.dist import DistZero
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29631")
    os.environ.setdefault("RANK", "0")
    os.environ.setdefault("WORLD_SIZE", "1")
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    rank, world = dist.get_rank(), dist.get_world_size()
    N = w["N"]
    dz = DistZero(N)
    sp = torch.cuda.current_stream().cuda_stream
    synth.fill_device(dz.master[0].data_ptr(), synth.NORMAL, synth.F32, synth.SEED,
                      synth.MASTER_STREAM, dz.hi - dz.lo, 0.02, first=dz.lo, cuda_stream=sp)
    synth.fill_device(dz.grad.data_ptr(), synth.NORMAL, synth.BF16, synth.SEED,
                      synth.grad_stream(1, rank), N, w["sigma"], cuda_stream=sp)
    dz.init(0)
    dz.publish_weights()
    hp = zero.hparams(**w["hp"])
    for _ in range(args.warmup):
        dz.step(hp)
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for a, b in kev:
        a.record()
        b.record()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    gpu_id = getattr(torch.cuda.get_device_properties(dev), "uuid", None)
    sampler = ClockSampler(("GPU-" + str(gpu_id)) if gpu_id else str(local))
    sampler.start()
    time.sleep(0.3)
    dist.barrier()
    torch.cuda.synchronize()
    t0.record()
    for k in range(args.steps):
        zero.zero_profile_events(kev[k][0].cuda_event, kev[k][1].cuda_event)
        dz.step(hp)
    t1.record()
    torch.cuda.synchronize()
    dist.barrier()
    clocks = sampler.stop()
    ms_total, kern_ms = max_over_ranks(
        [t0.elapsed_time(t1), sum(a.elapsed_time(b) for a, b in kev) / args.steps], dist, dev)
    res = dz.result()
    assert res["overflow"] == 0, res
    ms = ms_total / args.steps
    # end to end, host to host: this rank's gradient replica up from pinned host memory, the
    # step, this rank's updated bf16 weight replica back to pinned host memory
    e2e = None
    if not args.no_e2e:
        host_g = torch.empty(N, dtype=dz.grad.dtype, pin_memory=True)
        host_g.copy_(dz.grad)
        host_p = torch.empty(N, dtype=torch.bfloat16, pin_memory=True)
        torch.cuda.synchronize()
        e_start = torch.cuda.Event(enable_timing=True)
        e_stop = torch.cuda.Event(enable_timing=True)
        dist.barrier()
        torch.cuda.synchronize()
        e_start.record()
        for _ in range(args.e2e_steps):
            dz.grad.copy_(host_g, non_blocking=True)
            dz.step(hp)
            host_p.copy_(dz.param, non_blocking=True)
            res_e = dz.result()
            assert res_e["overflow"] == 0, res_e
        e_stop.record()
        torch.cuda.synchronize()
        e_ms = max_over_ranks([e_start.elapsed_time(e_stop)], dist, dev)[0]
        e2e = {"value": N / (e_ms / args.e2e_steps / 1e3), "unit": "params/s",
               "h2d_bytes_per_step": 2 * N * world, "d2h_bytes_per_step": (2 * N + 112) * world,
               "steps": args.e2e_steps, "result": "every rank's bf16 weight replica + step record"}
    hbm_peak, hbm_src = peaks()
    link_peak, link_src = nvlink_peak()
    hbm_bytes, link_bytes, bound, ideal = dist_roofline(dz.S, world, hbm_peak, link_peak)
    if rank == 0:
        config.update({"Nd": world, "path": "real ranks: fused kernel over peer memory + NCCL "
                       "step totals", "kernel": "fused_step_kernel (peer loads/stores)",
                       "parallelism": "dp%d (one rank per GPU)" % world,
                       "l2": "inputs larger than L2 (%.2f GB gradient replica per rank)"
                             % (2 * N / 1e9)})
        line = {"metric": METRIC, "value": N / (ms / 1e3), "unit": "params/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
                "dtype": "f32", "data": "synthetic", "config": config,
                "roofline": {"bound": bound, "achieved": (hbm_bytes if bound == "hbm" else
                                                          link_bytes) / (kern_ms / 1e3) / 1e9,
                             "peak": hbm_peak if bound == "hbm" else link_peak, "unit": "GB/s",
                             "frac": ideal / (kern_ms / 1e3), "traffic": None,
                             "peak_source": hbm_src if bound == "hbm" else link_src,
                             "hbm_peak": hbm_peak, "hbm_peak_source": hbm_src,
                             "nvlink_peak": link_peak, "nvlink_peak_source": link_src,
                             "kernel_ms": kern_ms, "hbm_bytes_per_rank": hbm_bytes,
                             "nvlink_bytes_per_rank": link_bytes},
                "cpu_baseline": None, "e2e": e2e, "clocks": clocks,
                "gpu_launches": 3 * args.steps}
        print(json.dumps(line), flush=True)
    dz.close()
    dist.barrier()
    dist.destroy_process_group()


# ----------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--dist", action="store_true",
                    help="real data parallelism: one rank per GPU owns one shard (Nd = GPUs)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--grad-sets-gb", type=float, default=24.0,
                    help="device memory budget for distinct per-step gradient sets")
    ap.add_argument("--no-tma", action="store_true",
                    help="fused path: always the register-pipelined kernel")
    ap.add_argument("--tma", action="store_true",
                    help="fused path: always the TMA-pipelined kernel")
    ap.add_argument("--bf16-grad-shard", action="store_true",
                    help="two-pass / stage 3: keep the reduced gradient as bf16")
    ap.add_argument("--two-pass", action="store_true",
                    help="stages 1/2: reduce-scatter into an fp32 shard, then Adam + all-gather; "
                         "stage 3: the two-phase step (gathers and reduce-scatters, then Adam)")
    ap.add_argument("--fused-layers", action="store_true",
                    help="stage 3: one speculative fused pass per layer carrying the layer's "
                         "gather (two fp32 state copies); the default for stage 3 unless "
                         "--two-pass or --bf16-grad-shard")
    ap.add_argument("--graph", action="store_true",
                    help="replay the timed steps from CUDA graphs (default for launch-bound steps)")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every timed step from the host, even a launch-bound one")
    ap.add_argument("--bucket-override", type=int, default=-1,
                    help="stages 1/2: run with a different bucket size (0 = one bucket)")
    ap.add_argument("--nd-override", type=int, default=0,
                    help="run the workload with a different number of simulated ranks")
    ap.add_argument("--layer-override", type=int, default=0,
                    help="stage 3: run with a different layer length")
    ap.add_argument("--n-override", type=int, default=0,
                    help="run the workload at a different N (small cases for profiling)")
    args = ap.parse_args()
    assert args.warmup >= 3, "at least 3 warm-up steps"
    w = dict(WORKLOADS[args.workload])
    if w["stage"] == 3 and not args.two_pass and not args.bf16_grad_shard:
        # the faster ZeRO-3 step (60 B/param against 68) whenever its second fp32 state copy fits
        # (the Llama-7B-shaped job: 155 GB of state + 6.5 GB of layer buffers of 180 GB)
        args.fused_layers = True
    if w["stage"] == 3 and args.two_pass:
        args.two_pass, args.fused_layers = False, False  # stage 3's two-phase step
    if args.n_override:
        w["N"] = args.n_override
        w["desc"] += " [N overridden to %d]" % args.n_override
    if args.nd_override:
        w["Nd"] = args.nd_override
        w["desc"] += " [Nd overridden to %d]" % args.nd_override
    if args.layer_override and w["stage"] == 3:
        w["layer"] = w["bucket"] = args.layer_override
        w["desc"] += " [layer overridden to %d]" % args.layer_override
    if args.bucket_override >= 0 and w["stage"] != 3:
        w["bucket"] = args.bucket_override
        w["desc"] += " [bucket overridden to %d]" % args.bucket_override

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    config = {"workload": w["desc"], "N": w["N"], "Nd": w["Nd"], "stage": w["stage"],
              "bucket": w["bucket"], "grad_dtype": w["gdt"], "state_dtype": "f32",
              "path": ("two-pass" if args.two_pass else
                       ("per-layer fused" if w["stage"] == 3 and args.fused_layers else
                        ("per-layer" if w["stage"] == 3 else "fused")))
              + (", bf16 gradient shard" if args.bf16_grad_shard else ""),
              "weights_dtype": "bf16", "parallelism": "replicas (%d simulated ranks per GPU)"
              % w["Nd"], "l2": "inputs larger than L2 (%.1f GB of gradients per step)"
              % (2 * w["Nd"] * w["N"] / 1e9)}

    # one rank per GPU: the real data-parallel path for flat ZeRO-1/2 workloads
    real_ranks = world > 1 and w["stage"] in (1, 2) and not w.get("offload")
    if (args.dist or real_ranks) and args.impl != "reference":
        return run_dist(args, w, config)

    if args.impl == "reference":
        if rank != 0:
            return
        # each step is a bounded sample of the workload, sized so that the whole run of
        # warmup + steps oracle steps takes about two minutes (at most 3 s per step); the
        # oracle runs on every host core, one contiguous chunk of the sample per core
        per_step = min(3.0, 120.0 / (args.warmup + args.steps))
        cores = host_threads()
        n, times = cpu_baseline(w, target_s=per_step, steps=args.warmup + args.steps,
                                threads=cores)
        timed = times[args.warmup:]
        ms = 1e3 * sum(timed) / len(timed)
        val = n / (ms / 1e3)
        line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "params/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": config,
                "cpu_baseline": {"value": val, "unit": "params/s", "cores": cores,
                                 "kind": "oracle",
                                 "sample": "first %d of %d parameters, Nd=%d, one step each, "
                                           "one contiguous chunk per core"
                                 % (n, w["N"], w["Nd"])},
                "e2e": {"value": val, "unit": "params/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch
    import synth
    import zero_sharded_optimizer_03_b200 as zero

    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if w.get("offload"):
        return run_offload(args, w, world, rank, dist, dev, config)
    s = torch.cuda.current_stream()
    sp = s.cuda_stream

    Nd, N, stage = w["Nd"], w["N"], w["stage"]
    gdt = zero.ZERO_FP16 if w["gdt"] == "fp16" else zero.ZERO_BF16
    sdt = synth.FP16 if w["gdt"] == "fp16" else synth.BF16
    kind = synth.HEAVY if w["kind"] == "heavy" else synth.NORMAL
    tail = float(__import__("numpy").float32(w["sigma"] * 1e3))
    hp = zero.hparams(**w["hp"])
    flags = zero.ZERO_TWO_PASS if args.two_pass else zero.ZERO_FUSED
    if args.no_tma:
        flags |= zero.ZERO_NO_TMA
    if args.tma:
        flags |= zero.ZERO_FORCE_TMA
    # which fused kernel zero_step picks (mirrors the library's rule)
    tma_path = (not args.two_pass and w["stage"] != 3 and not args.no_tma and
                (args.tma or (w["Nd"] >= 16 and (w["bucket"] or w["N"]) >= (1 << 24))))
    if w["stage"] == 3 and args.fused_layers:
        line_kernel = ("zero3 step: gather_layer_tma + fused_step kernels (per layer)" if args.tma
                       else "zero3 step: fused_step kernel with the layer gather (per layer)")
    elif w["stage"] == 3:
        line_kernel = "zero3 step: gather_layer + reduce_scatter + adam kernels"
    elif args.two_pass:
        line_kernel = "reduce_scatter + adam kernels (two-pass)"
    else:
        line_kernel = "fused_step_tma_kernel" if tma_path else "fused_step_kernel"
    config["kernel"] = line_kernel
    if args.bf16_grad_shard:
        flags |= zero.ZERO_BF16_GRAD_SHARD
    def make_buffers():
        if stage == 3:
            assert w["layer"] % Nd == 0 and N % w["layer"] == 0, "unpadded layers expected"
            b = zero.ZeroBuffers(3, Nd, N, grad_dtype=gdt, layer_len=w["layer"],
                                 flags=(zero.ZERO_BF16_GRAD_SHARD if args.bf16_grad_shard else 0)
                                 | (zero.ZERO_FORCE_TMA if args.tma else 0)
                                 | (zero.ZERO_FUSED_LAYERS if args.fused_layers else 0))
        else:
            b = zero.ZeroBuffers(stage, Nd, N, grad_dtype=gdt, flags=flags)
        synth.fill_device(b.master[0].data_ptr(), synth.NORMAL, synth.F32, synth.SEED,
                          synth.MASTER_STREAM, N, 0.02, cuda_stream=sp)
        if w.get("t0"):
            synth.fill_device(b.exp_avg[0].data_ptr(), synth.ABS, synth.F32, synth.SEED,
                              synth.M_STREAM, N, 1e-3, cuda_stream=sp)
            synth.fill_device(b.exp_avg_sq[0].data_ptr(), synth.SQUARE, synth.F32, synth.SEED,
                              synth.V_STREAM, N, 1e-6, cuda_stream=sp)
        b.init_workspace(w.get("t0", 0))
        b.sync_params_from_master()
        return b

    # A step smaller than a few L2 capacities would find its state and weights still in L2
    # from its previous run; such workloads cycle through independent optimizer instances (own
    # state, weights, workspace and gradients) so that every step's data comes from HBM.
    bpp = bytes_per_param(w, args.two_pass, args.bf16_grad_shard, args.fused_layers)
    ninst = optimizer_instances(stage, bpp * N)
    insts = [make_buffers() for _ in range(ninst)]
    buf = insts[0]
    glen = buf.grads[0].numel()  # N (stages 1/2) or one layer (stage 3, reused per layer)

    # distinct gradient sets (set 0 lives in buf.grads; with several instances, instance k's
    # own buf.grads is set k)
    set_bytes = 2 * Nd * glen
    if ninst > 1:
        nsets = ninst
        gsets = [b.grads for b in insts]
    else:
        nsets = int(max(1, min(args.warmup + args.steps, args.grad_sets_gb * 1e9 // set_bytes)))
        if stage == 3:
            nsets = 1
        gsets = [buf.grads] + [[torch.empty(glen, dtype=buf.grads[0].dtype, device=dev)
                                for _ in range(Nd)] for _ in range(nsets - 1)]
    states = []
    for k, gs in enumerate(gsets):
        for r in range(Nd):
            synth.fill_device(gs[r].data_ptr(), kind, sdt, synth.SEED,
                              synth.grad_stream(k + 1, r), glen, w["sigma"], tail, cuda_stream=sp)
        st = zero.zero_state_t.from_buffer_copy(insts[k].state if ninst > 1 else buf.state)
        for r in range(Nd):
            st.grads[r] = gs[r].data_ptr()
        states.append(st)
    if ninst > 1:
        config["l2"] = ("inputs larger than L2: %d independent optimizer instances cycled, "
                        "%.0f MB of step data between two runs of one instance"
                        % (ninst, ninst * bpp * N / 1e6))
    nb = 1 if w["bucket"] == 0 else -(-N // w["bucket"])
    if stage == 3 and args.fused_layers:
        # per layer: the fused gather + update kernel (+ a TMA gather kernel with --tma); the
        # overflow-repair check
        launches_per_step = (2 if args.tma else 1) * nb + 1
    elif stage == 3:
        launches_per_step = 3 * nb  # per layer: gather, reduce-scatter, Adam
    elif args.two_pass:
        launches_per_step = 2 * nb  # per bucket: reduce-scatter, Adam + all-gather
    elif nb == 1 and not tma_path and N <= SELF_REPAIR_MAX:
        launches_per_step = 1  # the fused kernel repairs a short step itself after a skip
    else:
        launches_per_step = nb + 1  # fused kernel per bucket + the overflow-repair check

    def step(k, ev=None):
        if ev is not None:
            zero.zero_profile_events(ev[0].cuda_event, ev[1].cuda_event)
        zero.zero_step(stage, Nd, N, w["bucket"], states[k % nsets], hp, sp)

    for k in range(args.warmup):
        step(k)
    torch.cuda.synchronize()

    # Launch-bound steps (the workloads that cycle optimizer instances: tens of microseconds per
    # step) are replayed from CUDA graphs of captured zero_step calls, as a training loop of
    # such a model would run them: the host cost of a Python call and two kernel launches per
    # step is then paid once at capture.  One graph holds one step of every instance in order;
    # single-step graphs make up a remainder, so exactly args.steps steps are timed.
    use_graph = (ninst > 1 and not args.no_graph) or args.graph
    graphs_all, graphs_one = None, []
    if use_graph:
        side = torch.cuda.Stream()
        side.wait_stream(s)
        for k in range(nsets):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                zero.zero_step(stage, Nd, N, w["bucket"], states[k], hp, side.cuda_stream)
            graphs_one.append(g)
        graphs_all = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graphs_all, stream=side):
            for k in range(nsets):
                zero.zero_step(stage, Nd, N, w["bucket"], states[k], hp, side.cuda_stream)
        s.wait_stream(side)
        for _ in range(2):  # warm replays (capture runs nothing)
            graphs_all.replay()
        torch.cuda.synchronize()
        config["launch"] = ("CUDA graphs of captured zero_step calls (%d steps per graph), "
                            "replayed" % nsets)

    def timed_steps():
        if not use_graph:
            for k in range(args.steps):
                step(args.warmup + k)
            return
        for _ in range(args.steps // nsets):
            graphs_all.replay()
        for k in range(args.steps % nsets):
            graphs_one[k].replay()

    # at least 100 evented steps, so that one slow step does not decide the average
    kev_steps = max(args.steps, 100)
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(kev_steps)]
    for a, b in kev:  # create the underlying CUDA events before handing them to the library
        a.record(s)
        b.record(s)
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    gpu_id = getattr(torch.cuda.get_device_properties(dev), "uuid", None)
    sampler = ClockSampler(("GPU-" + str(gpu_id)) if gpu_id else str(local))
    sampler.start()
    time.sleep(0.3)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t_start.record(s)
    timed_steps()
    t_stop.record(s)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    # more steps, each bracketed by CUDA events around its data kernels (the roofline's kernel
    # time); kept out of the loop above, whose time per step is the headline, because an event
    # record between two steps costs time on a microsecond step
    for k in range(kev_steps):
        step(args.warmup + args.steps + k, kev[k])
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms_total = t_start.elapsed_time(t_stop)
    kern_list = [a.elapsed_time(b) for a, b in kev]
    kern_ms = sum(kern_list) / kev_steps
    kern_median = statistics.median(kern_list)
    del graphs_all, graphs_one
    for b in insts:
        res = b.result()
        assert res["overflow"] == 0 and res["skipped"] == 0, res

    ms_total, kern_ms = max_over_ranks([ms_total, kern_ms], dist, dev)
    ms_step = ms_total / args.steps
    value = whole_job_rate(N, world, ms_step)
    achieved = bpp * N / (kern_ms / 1e3) / 1e9
    peak, peak_src = peaks()
    tr = None
    if not args.n_override and args.bucket_override < 0:
        tr = traffic_record(line_kernel, args.workload)
    traffic = tr["dram_bytes_per_launch"] if tr else None

    # end to end through the public API, host to host: every step copies the Nd gradient
    # replicas from pinned host memory to the device, runs the step, copies the step's product
    # -- the updated bf16 weights (rank 0's replica; for ZeRO-3 the weight shards, which hold
    # the whole vector) -- back to pinned host memory, and reads the step's bookkeeping
    # (zero_read_result: overflow / skip, 112 bytes, synchronizing)
    e2e = None
    if not args.no_e2e:
        host = [torch.empty(glen, dtype=buf.grads[0].dtype, pin_memory=True) for _ in range(Nd)]
        for r in range(Nd):
            host[r].copy_(buf.grads[r])
        result_dev = buf.param_shard if stage == 3 else buf.params[0]
        result_host = torch.empty(result_dev.numel(), dtype=result_dev.dtype, pin_memory=True)
        torch.cuda.synchronize()
        d2h = result_dev.numel() * result_dev.element_size() + 112
        e_start = torch.cuda.Event(enable_timing=True)
        e_stop = torch.cuda.Event(enable_timing=True)
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        e_start.record(s)
        for k in range(args.e2e_steps):
            # (ZeRO-3: the gradient buffers hold one layer, which every layer of the step reuses)
            for r in range(Nd):
                buf.grads[r].copy_(host[r], non_blocking=True)
            zero.zero_step(stage, Nd, N, w["bucket"], buf.state, hp, sp)
            result_host.copy_(result_dev, non_blocking=True)
            res_e = zero.zero_read_result(buf.ws.data_ptr(), sp)
            assert res_e["overflow"] == 0, res_e
        e_stop.record(s)
        torch.cuda.synchronize()
        e_ms = max_over_ranks([e_start.elapsed_time(e_stop)], dist, dev)[0]
        e2e = {"value": whole_job_rate(N, world, e_ms / args.e2e_steps), "unit": "params/s",
               "h2d_bytes_per_step": 2 * Nd * glen,
               "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
               "result": "bf16 weights (%s) + 112-byte step record" %
                         ("weight shards, N elements" if stage == 3 else "rank 0 replica, N elements")}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_record(w)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "params/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f32", "data": "synthetic", "config": config,
                "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak,
                             "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                             "peak_source": peak_src,
                             "kernel": line_kernel,
                             "bytes_per_param": bpp, "kernel_ms": kern_ms,
                             "kernel_ms_median": kern_median, "kernel_steps": kev_steps,
                             "frac_of_8TBs": achieved / 8000.0},
                "hbm_gbs_per_step": bpp * N / (ms_step / 1e3) / 1e9,
                "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
                "gpu_launches": launches_per_step * args.steps,
                "grad_sets": nsets, "instances": ninst}
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
