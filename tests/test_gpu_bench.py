"""bench.py on a B200: one run of the 1,000,003-element workload (CUDA-graph replay, optimizer
instances cycled, end-to-end leg, CPU baselines) prints one JSON line with the keys and the
consistency the benchmark line promises."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.gpu
def test_bench_line_on_the_short_workload():
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--workload",
                        "zero2-1m-nd4", "--steps", "40", "--warmup", "3"],
                       capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-3000:]
    lines = [x for x in p.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    N = 1_000_003
    assert d["unit"] == "params/s" and d["higher_is_better"] is True and d["n_gpus"] == 1
    assert (d["steps"], d["warmup"]) == (40, 3)
    assert abs(d["value"] - N / (d["ms_per_step"] / 1e3)) <= 1e-6 * d["value"]
    assert d["config"]["N"] == N and d["config"]["Nd"] == 4
    assert "CUDA graphs" in d["config"]["launch"] and d["instances"] == 10
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["bytes_per_param"] == 40
    assert abs(r["achieved"] - 40 * N / (r["kernel_ms"] / 1e3) / 1e9) <= 1e-6 * r["achieved"]
    assert abs(r["frac"] - r["achieved"] / r["peak"]) <= 1e-9 and 0 < r["frac"] < 1.2
    assert r["kernel_steps"] >= 100
    e = d["e2e"]
    assert e["h2d_bytes_per_step"] == 2 * 4 * N and e["d2h_bytes_per_step"] == 2 * N + 112
    assert 0 < e["value"] < d["value"]
    c = d["cpu_baseline"]
    assert c["kind"] == "oracle" and c["cores"] >= 1 and c["value"] > 0 and c["sample"]
    assert c["single_core"]["cores"] == 1 and c["single_core"]["value"] > 0
    assert d["gpu_launches"] == 40  # one fused pass per step (it repairs itself after a skip)
    assert d["clocks"] is None or d["clocks"]["sm_mhz"] > 0


@pytest.mark.gpu
def test_bench_real_rank_line_one_rank():
    """`bench.py --dist` under torchrun, one rank on one GPU (the real-rank path the bench takes
    on N GPUs): one JSON line, strong scaling, the rank's HBM bytes and no NVLink bytes."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    env = dict(os.environ, NCCL_NVLS_ENABLE="0", TORCH_SYMM_MEM_DISABLE_MULTICAST="1")
    cmd = ["timeout", "-k", "30", "600", sys.executable, "-m", "torch.distributed.run",
           "--nnodes", "1", "--nproc-per-node", "1", "--master-addr", "127.0.0.1",
           "--master-port", str(port), os.path.join(ROOT, "bench.py"), "--dist", "--workload",
           "zero1-gpt2-small", "--steps", "20", "--warmup", "5"]
    p = subprocess.run(cmd, capture_output=True, text=True, cwd=ROOT, env=env)
    assert p.returncode == 0, p.stderr[-3000:]
    lines = [x for x in p.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    N = 124_439_808
    assert d["scaling"] == "strong" and d["n_gpus"] == 1 and d["config"]["Nd"] == 1
    assert abs(d["value"] - N / (d["ms_per_step"] / 1e3)) <= 1e-6 * d["value"]
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["nvlink_bytes_per_rank"] == 0
    assert r["hbm_bytes_per_rank"] == 28 * N and 0 < r["frac"] < 1.2
    assert d["e2e"]["h2d_bytes_per_step"] == 2 * N and d["e2e"]["value"] > 0
