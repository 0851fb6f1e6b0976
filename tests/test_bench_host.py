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


def test_roofline_frac_is_the_hbm_fraction():
    """Every workload is graded on HBM bytes: frac = algorithmic bytes /
    time / HBM peak; the derived on-chip bounds sit in their own fields."""
    peaks, _ = bench.load_peaks()
    for cfg in range(5):
        info = bench.workload_info(cfg)
        r = bench.roofline(info, 1e-4, None)
        assert r["bound"] == "hbm" and r["unit"] == "GB/s"
        assert r["achieved"] == pytest.approx(info["bytes"] / 1e-4 / 1e9)
        assert r["frac"] == pytest.approx(r["achieved"] / peaks["hbm_gbs"])
        if info["kind"] == "s6":
            mhz = peaks.get("sm_max_mhz", 1965.0)
            assert r["mufu_frac"] == pytest.approx(info["elems"] / 1e-4 / (148 * mhz * 1e6 * 16))
            assert r["alu_frac"] == pytest.approx(r["mufu_frac"] * 16 / (64 / 3))
        else:
            t = r["tensor_pipe_est"]
            assert t["sms_used"] == 128
            assert t["all_sms"] == pytest.approx(t["over_sms_used"] * 128 / 148)


def test_reference_arm_prints_the_same_config():
    for cfg in range(5):
        info = bench.workload_info(cfg)
        a = bench.config_dict(info, cfg, "scan", 1)
        assert a["config_index"] == cfg and a["algorithmic_bytes_per_step"] == info["bytes"]
        assert a == bench.config_dict(bench.workload_info(cfg), cfg, "scan", 1)


def test_output_columns_and_error_measure():
    """Column c of an S6 output is (b, d) = divmod(c, D); of an SSD output
    (b, h, p) with c = (b H + h) P + p; the error measure divides by
    max(|o|, rms(o))."""
    import numpy as np
    s6 = {"kind": "s6", "dim": 5}
    out = np.arange(2 * 3 * 5).reshape(2, 3, 5)
    g = bench.output_columns(out, s6, [0, 7])
    assert (g[0] == out[0, :, 0]).all() and (g[1] == out[1, :, 2]).all()
    ssd = {"kind": "ssd", "nheads": 3, "headdim": 4}
    out = np.arange(2 * 6 * 3 * 4).reshape(2, 6, 3, 4)
    g = bench.output_columns(out, ssd, [(1 * 3 + 2) * 4 + 1])
    assert (g[0] == out[1, :, 2, 1]).all()
    o = np.array([1.0, -1.0, 1e-9])
    assert bench.rel_err(o, o) == 0.0
    assert bench.rel_err(o + np.array([0.0, 0.0, 1e-3]), o) == pytest.approx(1e-3 / np.sqrt(2 / 3))


def test_checkpointing_scan_counts_its_checkpoints():
    """--op fwd_ckpt also writes each direction's checkpoints: the state
    entering every 4-step chunk, 16 fp32 per channel."""
    a, b = bench.workload_info(1), bench.workload_info(1, "fwd_ckpt")
    assert b["elems"] == a["elems"]
    assert b["bytes"] - a["bytes"] == 2 * 64 * ((197 + 3) // 4) * 768 * 16 * 4


def test_launch_count_follows_the_plan():
    """The launches a call makes, as bench.py counts them from the library's
    plan (host-only query): one pass for Vim-Tiny and the hi-res bf16 scan
    (four threads per channel) and Vim-Small, summary + carry + main for the
    long bf16 rows, and the whole-channel plan for the checkpointing
    variant; SSD one launch."""
    import types
    import selective_state_space_24_b200 as ssm
    lib = ssm.capi()
    expect = {(0, "scan"): 1, (1, "scan"): 1, (2, "scan"): 1, (3, "scan"): 3, (1, "fwd_ckpt"): 1,
              (1, "ordered"): 1, (3, "zoh"): 1, (4, "scan"): 1}
    for (cfg, op), n in expect.items():
        w = bench.workload_info(cfg, op)
        dims = None
        if w["kind"] == "s6":
            dims = ssm.ssm_dims(w["batch"], w["seqlen"], w["dim"], w["dstate"],
                                ssm.SSM_F32 if w["dtype"] == "f32" else ssm.SSM_BF16)
        ns = types.SimpleNamespace(info=w, op=op, lib=lib, dims=dims)
        assert bench.DeviceWorkload._launches(ns) == n, (cfg, op)
    # the query leaves the layout choice to the cost model again
    assert ssm.scan_plan(1, 196, 384, 16) == (1, -4)
