"""Pins of the oracle's memory and communication closed forms (no GPU).

The figures come from tests/golden/pages_figures.json, which records numbers the pages print
with their source.  Exact values are recomputed here with rational arithmetic (fractions),
independently of the oracle's floating-point evaluation order.
"""
import json
import os
from fractions import Fraction

import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_figures.json")
FIG = {f["id"]: f for f in json.load(open(GOLDEN, encoding="utf-8"))["figures"]}
GiB = 2 ** 30


def test_fp16_params_of_175B_is_350GB():
    f = FIG["fp16_params_175B"]
    mem = oracle.memory_estimate(f["num_params"], 1)
    assert mem["DP"]["parameters"] * GiB == pytest.approx(f["bytes"], rel=1e-12)


def test_default_byte_accounting_is_2_2_12():
    f = FIG["mixed_precision_bytes"]
    assert (f["bytes_per_param"], f["bytes_per_opt_state"]) == (2, 12)
    mem = oracle.memory_estimate(1.0, 1)  # one parameter, one rank: bytes per parameter
    dp = mem["DP"]
    assert dp["parameters"] * GiB == pytest.approx(2)
    assert dp["gradients"] * GiB == pytest.approx(2)
    assert dp["optimizer_states"] * GiB == pytest.approx(12)
    assert dp["total"] * GiB == pytest.approx(16)


def test_example_call_175B_on_64_ranks_exact():
    f = FIG["example_call"]
    N, Nd = Fraction(int(f["num_params"])), f["dp_degree"]
    P = G = 2 * N
    O = 12 * N
    exact = {
        "DP": (O, G, P),
        "ZeRO-1": (O / Nd, G, P),
        "ZeRO-2": (O / Nd, G / Nd, P),
        "ZeRO-3": (O / Nd, G / Nd, P / Nd),
    }
    mem = oracle.memory_estimate(f["num_params"], Nd)
    for stage, (o, g, p) in exact.items():
        got = mem[stage]
        assert got["optimizer_states"] == pytest.approx(float(o / GiB), rel=1e-14)
        assert got["gradients"] == pytest.approx(float(g / GiB), rel=1e-14)
        assert got["parameters"] == pytest.approx(float(p / GiB), rel=1e-14)
        assert got["total"] == pytest.approx(float((o + g + p) / GiB), rel=1e-14)
    # the four totals, worked by hand to 2 decimals (GiB)
    assert round(mem["DP"]["total"], 2) == 2607.70
    assert round(mem["ZeRO-1"]["total"], 2) == 682.48
    assert round(mem["ZeRO-2"]["total"], 2) == 361.62
    assert round(mem["ZeRO-3"]["total"], 2) == 40.75
    # ZeRO-3 keeps (2 + 2 + 12) N / Nd bytes per GPU
    assert mem["ZeRO-3"]["total"] * GiB == pytest.approx(16 * 175e9 / 64, rel=1e-14)


def test_fp32_16_byte_breakdown():
    f = FIG["fp32_breakdown"]
    assert f["param"] + f["grad"] + f["momentum"] + f["variance"] == f["total"] == 16
    # fp32 weights and gradients (4 B), optimizer state momentum + variance (8 B)
    mem = oracle.memory_estimate(1.0, 1, bytes_per_param=4, bytes_per_opt_state=8)
    assert mem["DP"]["total"] * GiB == pytest.approx(f["total"])
    share = mem["DP"]["optimizer_states"] / mem["DP"]["total"]
    assert share == pytest.approx(f["optimizer_share"])


def test_stage1_7B_on_8_cards():
    f = FIG["stage1_7B_8cards"]
    per_param = f["opt_bytes_total"] / f["num_params"]  # 4 bytes of optimizer state
    mem = oracle.memory_estimate(f["num_params"], f["dp_degree"], bytes_per_param=2,
                                 bytes_per_opt_state=int(per_param))
    assert mem["DP"]["optimizer_states"] * GiB == pytest.approx(f["opt_bytes_total"])
    assert mem["ZeRO-1"]["optimizer_states"] * GiB == pytest.approx(f["opt_bytes_per_card"])


def test_memory_ratios_4x_8x_linear():
    f = FIG["memory_ratios"]
    big = oracle.memory_estimate(175e9, 10 ** 7)
    assert big["DP"]["total"] / big["ZeRO-1"]["total"] == pytest.approx(f["zero1_ratio"], rel=1e-5)
    assert big["DP"]["total"] / big["ZeRO-2"]["total"] == pytest.approx(f["zero2_ratio"], rel=1e-5)
    for Nd in (1, 2, 8, 64, 1000):
        mem = oracle.memory_estimate(175e9, Nd)
        assert mem["DP"]["total"] / mem["ZeRO-3"]["total"] == pytest.approx(Nd, rel=1e-12)
        # each stage saves at least as much as the one before
        assert (mem["DP"]["total"] >= mem["ZeRO-1"]["total"] >= mem["ZeRO-2"]["total"]
                >= mem["ZeRO-3"]["total"])
    one = oracle.memory_estimate(175e9, 1)
    assert one["DP"]["total"] == one["ZeRO-3"]["total"]  # no saving on a single rank ([P3])


@pytest.mark.parametrize("Nd", [2, 4, 8, 16, 64, 1024])
def test_comm_volume(Nd):
    f = FIG["comm_volume"]
    N = 1e9
    dp = oracle.comm_volume(0, N, Nd)
    assert oracle.comm_volume(1, N, Nd) == pytest.approx(f["zero12_vs_dp"] * dp)
    assert oracle.comm_volume(2, N, Nd) == pytest.approx(f["zero12_vs_dp"] * dp)
    assert oracle.comm_volume(3, N, Nd) / dp == pytest.approx(f["zero3_vs_dp"], rel=1e-15)
    # ring all-reduce: 2 (Nd-1)/Nd N elements per rank, about 2N for large Nd
    assert dp == pytest.approx(float(2 * Fraction(Nd - 1, Nd) * int(N)), rel=1e-15)
    if Nd >= 1024:
        assert dp / N == pytest.approx(f["zero12_elements_per_N"], rel=1e-3)
    assert oracle.comm_volume(1, N, 1) == 0.0  # a single rank sends nothing
