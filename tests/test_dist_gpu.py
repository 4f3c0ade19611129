"""Real data parallelism (one process per GPU, symmetric-memory peer buffers, NCCL for the step
totals), run through torchrun with one rank per available GPU (this check uses one GPU)."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.gpu
def test_dist_zero_matches_oracle_one_rank_per_gpu():
    nproc = 1  # ranks must not share a GPU: their kernels wait on one another
    env = dict(os.environ, ZERO_DIST_N="100003", NCCL_NVLS_ENABLE="0",
               TORCH_SYMM_MEM_DISABLE_MULTICAST="1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node",
           str(nproc), "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "tests", "_dist_worker.py")]
    res = subprocess.run(["timeout", "-k", "30", "300"] + cmd, env=env, capture_output=True,
                         text=True)
    assert res.returncode == 0, res.stdout[-2000:] + res.stderr[-4000:]
    lines = [json.loads(x) for x in res.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == nproc
    for r in lines:
        assert r["flags_ok"] and r["overflow_seq"] == [0, 1, 0], r
        assert r["master_exact"] and r["exp_avg_sq_exact"] and r["replica_exact"], r
        assert r["sumsq_rel"] <= 1e-5, r
