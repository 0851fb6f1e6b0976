"""bench.py's host arithmetic (no GPU): the per-call element and byte counts
of the workloads, the derived ALU bounds and the step statistics."""
import math
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_vim_small_bidir_counts():
    """B 64, L 197, D 768, N 16, fp32, two directions: elements B L D N x 2;
    bytes x, delta, z (each direction) and out, B and C per direction, and
    A, D, delta_bias per direction."""
    w = bench.workload_info(1)
    B, L, D, N = 64, 197, 768, 16
    assert w["elems"] == B * L * D * N * 2 == 309_854_208
    assert w["bytes"] == B * L * D * 4 * 5 + B * L * N * 4 * 4 + 2 * (D * N + 2 * D) * 4 == 196_997_120


def test_ssd_counts():
    """Mamba2 SSD B 4, L 8192, H 32, P 64, N 128, bf16: x, z, y (B L H P),
    B and C (B L N), delta (B L H) and three fp32 scalars per head."""
    w = bench.workload_info(4)
    assert w["elems"] == 4 * 8192 * 32 * 64 * 128
    assert w["bytes"] == 3 * 4 * 8192 * 32 * 64 * 2 + 2 * 4 * 8192 * 128 * 2 + 4 * 8192 * 32 * 2 + 32 * 12


def test_alu_bounds():
    # forward: 64/3 elements per clock per SM; backward: 256/43
    assert bench.alu_peak_elems(1965.0) == pytest.approx(148 * 1965e6 * 64 / 3)
    assert bench.alu_peak_elems(1965.0) / 1e9 == pytest.approx(6204.16, abs=0.01)
    assert bench.bwd_alu_peak_elems(1965.0) / 1e9 == pytest.approx(1731.39, abs=0.01)
    # the balance the backward bound rests on: x exps on the MUFU (16 / clk)
    # take as long as 19 + 8 (3 - x) FMA-pipe operations (128 / clk)
    x = 43 / 16
    assert x / 16 == pytest.approx((19 + 8 * (3 - x)) / 128)


def test_step_stats_and_throughput():
    s = bench.step_stats([float(v) for v in range(1, 11)])
    assert s["median"] == 5.5 and s["p10"] == pytest.approx(1.9) and s["p90"] == pytest.approx(9.1)
    assert bench.step_stats([2.0]) == {"median": 2.0, "p10": 2.0, "p90": 2.0}
    # units of every rank over the max-over-ranks job time
    assert bench.job_throughput(1e6, 4, 10, 20.0) == pytest.approx(4e6 * 10 / 0.02)
    assert math.isfinite(bench.job_throughput(1.0, 1, 1, 1e-3))
