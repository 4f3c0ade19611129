"""Host helpers of bench.py that need no GPU: the algorithmic bytes per parameter behind every
roofline figure, and the rule that a stored DRAM-traffic record is reported only while the
kernel sources it was captured on are unchanged."""
import hashlib
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _w(stage, Nd):
    return dict(stage=stage, Nd=Nd)


@pytest.mark.parametrize("Nd,want", [(1, 28), (4, 40), (8, 56), (16, 88), (64, 280)])
def test_fused_step_bytes_per_param(Nd, want):
    # Nd 2-byte gradient reads + fp32 master/m/v read and written + Nd 2-byte weight writes
    assert bench.bytes_per_param(_w(2, Nd)) == want == 24 + 4 * Nd


def test_two_pass_and_zero3_bytes_per_param():
    # two-pass ZeRO-1/2 at Nd = 8: RS 16 read + 4 written, Adam 4 + 24 + 16 weight writes
    assert bench.bytes_per_param(_w(1, 8), two_pass=True) == 64
    assert bench.bytes_per_param(_w(1, 8), two_pass=True, g16=True) == 60
    # ZeRO-3 at Nd = 8: gather 2 + 16, RS 16 + 4, Adam 4 + 24 + 2 (bf16 shard)
    assert bench.bytes_per_param(_w(3, 8)) == 68
    assert bench.bytes_per_param(_w(3, 8), g16=True) == 64
    # fused layers: gather 2 + 16, fused pass 16 + 12 read, 12 + 2 written
    assert bench.bytes_per_param(_w(3, 8), fused_layers=True) == 60 == 28 + 4 * 8


def test_workloads_match_their_descriptions():
    w = bench.WORKLOADS
    assert (w["zero2-1m-nd4"]["N"], w["zero2-1m-nd4"]["Nd"]) == (1_000_003, 4)
    assert (w["zero1-gpt2-small"]["N"], w["zero1-gpt2-small"]["Nd"]) == (124_439_808, 8)
    assert w["zero2-fp16-bucketed"]["gdt"] == "fp16" and w["zero2-fp16-bucketed"]["Nd"] == 16
    assert (w["zero2-wide-fanin-nd64"]["N"], w["zero2-wide-fanin-nd64"]["Nd"]) == (1 << 28, 64)
    z3 = w["zero3-llama7b"]
    assert z3["layer"] == 4 * 4096 * 4096 + 3 * 4096 * 11008 and z3["N"] == 32 * z3["layer"]
    assert bench.DEFAULT == "zero2-2p28-nd8"
    assert (w[bench.DEFAULT]["N"], w[bench.DEFAULT]["Nd"], w[bench.DEFAULT]["bucket"]) == (1 << 28, 8, 0)


def test_cpu_baseline_record_has_the_all_core_and_single_core_legs():
    """The CPU baseline reports the oracle on every host core (one contiguous chunk per core) and
    on one core, each with its core count and sample."""
    w = dict(bench.WORKLOADS["zero2-1m-nd4"])
    rec = bench.cpu_baseline_record(w, target_s=0.2)
    assert rec["kind"] == "oracle" and rec["unit"] == "params/s" and rec["value"] > 0
    assert rec["cores"] == bench.host_threads() >= 1
    one = rec["single_core"]
    assert one["cores"] == 1 and one["value"] > 0 and one["sample"]
    n, times = bench.cpu_baseline(w, target_s=0.05, steps=2, threads=3)
    assert n % (3 * w["Nd"]) == 0 and 0 < n <= w["N"] and len(times) == 2


def test_traffic_record_follows_the_kernel_sources(tmp_path, monkeypatch):
    src = tmp_path / "k.cuh"
    src.write_bytes(b"// kernel v1\n")
    (tmp_path / "profiles").mkdir()
    rec = dict(kernel="fused_step_kernel", workload="zero1-gpt2-small",
               sources={"k.cuh": hashlib.sha256(b"// kernel v1\n").hexdigest()},
               dram_bytes_per_launch=123)
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"records": [rec]}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_record("fused_step_kernel", "zero1-gpt2-small")["dram_bytes_per_launch"] == 123
    assert bench.traffic_record("fused_step_kernel", "zero2-2p28-nd8") is None
    assert bench.traffic_record("fused_step_tma_kernel", "zero1-gpt2-small") is None
    src.write_bytes(b"// kernel v2\n")  # the kernel changed since the capture
    assert bench.traffic_record("fused_step_kernel", "zero1-gpt2-small") is None


def test_committed_traffic_records_are_consistent():
    """Every committed record's per-launch figure is the captured bytes scaled by the workload's
    N, and names sources that exist (a stale record is legal: bench.py then reports null)."""
    recs = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))["records"]
    assert recs
    for r in recs:
        for rel in r["sources"]:
            assert os.path.exists(os.path.join(ROOT, rel)), rel
        N = bench.WORKLOADS[r["workload"]]["N"]
        scaled = (r["captured_read_bytes"] + r["captured_write_bytes"]) * N / r["captured_n"]
        assert abs(r["dram_bytes_per_launch"] - scaled) <= 1
        # DRAM traffic within a few percent of the algorithmic bytes (no re-reads)
        assert 0.9 <= r["dram_bytes_per_launch"] / r["algorithmic_bytes_per_launch"] <= 1.05


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the CPU oracle timed on the host) prints one JSON line with
    the keys the benchmark contract asks of the reference arm."""
    import subprocess
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                       timeout=600, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [x for x in p.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["unit"] == "params/s" and d["higher_is_better"] is True and d["value"] > 0
    assert (d["steps"], d["warmup"], d["n_gpus"]) == (1, 3, 1)
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["config"]["workload"] == bench.WORKLOADS[bench.DEFAULT]["desc"]


def test_short_workloads_cycle_optimizer_instances():
    """A step smaller than three L2 capacities cycles independent optimizer instances so that its
    data comes from HBM: the 1M-element workload (40 B/param) takes 10, the large ones 1."""
    w = bench.WORKLOADS
    assert bench.optimizer_instances(2, 40 * w["zero2-1m-nd4"]["N"]) == 10
    assert bench.optimizer_instances(2, 56 * w["zero2-2p28-nd8"]["N"]) == 1
    assert bench.optimizer_instances(1, 56 * w["zero1-gpt2-small"]["N"]) == 1
    assert bench.optimizer_instances(3, 1000) == 1
    assert bench.optimizer_instances(2, 40 * 8192) == 64
    n = bench.optimizer_instances(2, 40 * 262_144)
    assert (n - 1) * 40 * 262_144 < 3 * bench.L2_BYTES <= n * 40 * 262_144


def test_real_rank_roofline_bytes_and_bound():
    """The real-rank step's roofline: one GPU moves only its HBM bytes; with peers each element
    of a rank's shard crosses NVLink once per peer in (gradient) and once out (weights), so at
    the measured 770 GB/s B200 peer copy against ~6.5 TB/s of HBM the step is NVLink-bound from 2 GPUs."""
    S = 1 << 25
    hbm, link, bound, ideal = bench.dist_roofline(S, 1, 6527.8, 770.0)
    assert (hbm, link, bound) == (28 * S, 0, "hbm") and ideal == 28 * S / 6527.8e9
    hbm, link, bound, ideal = bench.dist_roofline(S, 8, 6527.8, 770.0)
    assert (hbm, link, bound) == (28 * S, 4 * 7 * S, "nvlink") and ideal == 28 * S / 770e9
    assert bench.dist_roofline(S, 2, 6527.8, 770.0)[2] == "nvlink"
