"""One rank of the multi-GPU ZeRO check (launched by tests/test_dist_gpu.py through torchrun).

Every rank owns a shard of N parameters; three steps, the second with an overflow planted in
rank 0's gradient; the rank's shard and its weight replica are compared with the CPU oracle
(Nd = world size).  Prints one JSON line per rank."""
import datetime
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

import oracle  # noqa: E402
import synth  # noqa: E402
import zero_sharded_optimizer_03_b200 as zero  # noqa: E402
from zero_sharded_optimizer_03_b200.dist import DistZero  # noqa: E402


def main():
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                            device_id=torch.device("cuda", local))
    N = int(os.environ.get("ZERO_DIST_N", "100003"))
    rank, world = dist.get_rank(), dist.get_world_size()
    dz = DistZero(N)
    hp = dict(lr=1e-3, weight_decay=0.01, loss_scale=1.0)
    master0 = synth.fill_host(synth.NORMAL, synth.F32, synth.SEED, synth.MASTER_STREAM, N,
                              sigma=0.02)
    dz.master[0][:dz.hi - dz.lo].copy_(torch.from_numpy(master0[dz.lo:dz.hi]))
    dz.init(0)
    dz.publish_weights()
    S, Np, _ = oracle.partition(N, world)
    om = np.zeros(Np, np.float32)
    om[:N] = master0
    mm = np.zeros(Np, np.float32)
    vm = np.zeros(Np, np.float32)
    oreps = [oracle.f32_to_bf16(master0) for _ in range(world)]
    t = 0
    flags = []
    for k in (1, 2, 3):
        synth.fill_device(dz.grad.data_ptr(), synth.NORMAL, synth.BF16, synth.SEED,
                          synth.grad_stream(k, rank), N, 1e-3,
                          cuda_stream=torch.cuda.current_stream().cuda_stream)
        hg = [synth.fill_host(synth.NORMAL, synth.BF16, synth.SEED, synth.grad_stream(k, q), N,
                              sigma=1e-3) for q in range(world)]
        if k == 2:
            if rank == 0:
                dz.grad.view(torch.int16)[7] = 0x7F80  # +inf in bf16
            hg[0][7] = 0x7F80
        dz.step(zero.hparams(**hp))
        t, ovf, ss = oracle.zero12_step(world, N, 0, oracle.BF16, hg, om, mm, vm, oreps, hp, t)
        res = dz.result()
        flags.append((res["overflow"], ovf, res["step"], t))
    torch.cuda.synchronize()
    live = dz.live()
    got_m = dz.master[live][:dz.hi - dz.lo].cpu().numpy()
    got_v = dz.exp_avg_sq[live][:dz.hi - dz.lo].cpu().numpy()
    got_p = dz.param.view(torch.int16).cpu().numpy().view(np.uint16)[:N]
    out = {
        "rank": rank, "world": world,
        "flags_ok": all(a == b and c == d for a, b, c, d in flags),
        "overflow_seq": [f[0] for f in flags],
        "master_exact": got_m.tobytes() == om[dz.lo:dz.hi].tobytes(),
        "exp_avg_sq_exact": got_v.tobytes() == vm[dz.lo:dz.hi].tobytes(),
        "replica_exact": got_p.tobytes() == oreps[rank].tobytes(),
        "sumsq_rel": abs(res["grad_sumsq"] - ss) / ss,
    }
    print(json.dumps(out), flush=True)
    dz.close()
    dist.barrier()
    dist.destroy_process_group()


if __name__ == "__main__":
    main()
