#!/usr/bin/env python
"""Benchmark of the selective-scan hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config I] [--impl ours|reference]

One step = one call of the hot path over one batch of the workload:
config 1 (default) is the Vim-Small bidirectional scan, fp32, batch 64,
L 197, d_inner 768, N 16 (bidir_scan_fwd); configs 0, 2, 3 are the other S6
workloads and 4 the Mamba2 SSD workload.  Inputs are seeded synthetic
tensors (ssm_gen) with the shapes and value distributions of those
workloads.

Timing: W untimed warm-up steps, then K timed steps.  Before every timed
step a 512 MB buffer is written to flush the 126 MB L2; each step is
bracketed by CUDA events on the launching stream, and the step times are
summed (the flush is outside the events).  The timed region is bracketed by
a barrier and torch.cuda.synchronize(); with N > 1 every rank runs its own
batch (weak scaling, no collective on the data path) and the time is the
max over ranks.  nvidia-smi samples SM clocks and throttle reasons during
the timed region.

Rank 0 prints one JSON line.  `--impl reference` times the float64 CPU
oracle instead (bounded sample per step, all host cores).
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import ssm_gen  # noqa: E402

METRIC = "scan elements/s (B·L·D·N) and HBM GB/s as % of B200 peak, per config"
HBM_FALLBACK_GBS = 6650.0
L2_FLUSH_BYTES = 512 << 20
SMS = 148
# DRAM bytes (read + write) per launch of the dominant kernel, from one ncu
# capture of the current kernels (summaries under profiles/); absent where no
# capture matches them.
NCU_TRAFFIC = {1: 193.52e6, 4: 397.22e6}
NCU_TRAFFIC_STEP = 62.01e6
NCU_TRAFFIC_BWD = {1: 408.07e6}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=1000)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--config", type=int, default=1)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-per-config", action="store_true",
                   help="skip timing the other workloads after the headline one")
    p.add_argument("--op", default="scan", choices=["scan", "ordered", "conv", "fwd_ckpt", "zoh", "step", "bwd",
                                                    "bidir_bwd", "bwd_ckpt", "bidir_bwd_ckpt"],
                   help="scan: the workload's scan (default); ordered: the same bidirectional "
                        "workload along a random order of the positions with 30%% of the tokens "
                        "masked; conv: the same with a width-4 conv1d + SiLU per direction computed "
                        "inside the scan; zoh: the same with the exact zero-order-hold input coefficient "
                        "(bidir_scan_fwd_zoh); step: one decode step of a batch-512 x 1536-channel x "
                        "16-state fp32 state (ssm_step); bwd: the gradients (ssm_scan_bwd) of the "
                        "forward direction of the workload; bidir_bwd: the gradients of the whole "
                        "bidirectional scan (bidir_scan_bwd); fwd_ckpt: the bidirectional scan that also "
                        "stores the checkpoints its backward reads (bidir_scan_fwd_ckpt); bwd_ckpt / "
                        "bidir_bwd_ckpt: the gradients from those checkpoints (ssm_scan_bwd_ckpt / "
                        "bidir_scan_bwd_ckpt; the checkpointing forward runs once, untimed, before)")
    return p.parse_args()


# --------------------------------------------------------------- workload

def workload_info(cfg: int, op: str = "scan"):
    """Sizes of workload cfg: elements per call and algorithmic bytes (each
    input and output moved once; with op fwd_ckpt also the checkpoint arrays
    the checkpointing scan writes -- the state entering every 4-step chunk,
    16 fp32 per channel and direction)."""
    w = dict(ssm_gen.WORKLOADS[cfg])
    if w["kind"] == "s6":
        ndir = 2 if w["bidir"] else 1
        es = 4 if w["dtype"] == "f32" else 2
        B, L, D, N = w["batch"], w["seqlen"], w["dim"], w["dstate"]
        elems = B * L * D * N * ndir
        io = B * L * D * es * (2 + ndir + 1)          # x, delta, z per direction, out
        io += B * L * N * es * 2 * ndir               # B, C per direction
        io += ndir * (D * N + 2 * D) * 4              # A, D, delta_bias
        if w.get("last_state"):
            io += ndir * B * D * N * 4
        if op == "fwd_ckpt":
            ns = 4 if N <= 4 else 8 if N <= 8 else 16
            io += ndir * B * ((L + 3) // 4) * D * ns * 4
        w.update(ndir=ndir, elems=elems, bytes=io)
    else:
        B, L, H, P, N = w["batch"], w["seqlen"], w["nheads"], w["headdim"], w["dstate"]
        es = 2
        elems = B * L * H * P * N
        io = B * L * H * P * es * 3 + B * L * N * es * 2 + B * L * H * es + H * 12
        w.update(ndir=1, elems=elems, bytes=io)
    return w


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return {"hbm_gbs": HBM_FALLBACK_GBS, "bf16_tflops": 1590.0, "sm_max_mhz": 1965.0}, "fallback"


def alu_peak_elems(sm_mhz: float) -> float:
    """Element rate the SM pipes allow for the S6 inner step (one exp and four
    FMA-pipe operations per element): exps split between the MUFU unit
    (16/clk/SM) and an 8-operation FMA-pipe polynomial so that both pipes
    (MUFU 16/clk/SM, FMA 128/clk/SM) finish together -> 64/3 elements per
    clock per SM."""
    return SMS * sm_mhz * 1e6 * (64.0 / 3.0)


def mufu_peak_elems(sm_mhz: float) -> float:
    """Element rate of the S6 step if every exp ran on the MUFU unit (measured
    15.9 ex2 per clock per SM on B200; 16 taken) and nothing else limited it:
    one exp per element -> 16 elements per clock per SM."""
    return SMS * sm_mhz * 1e6 * 16.0


# tcgen05.mma instructions per (chunk, head) in the SSD kernel -- G 8, Yo 8,
# dS 4, Yd 8 -- and the tensor-pipe cycles one instruction of these shapes
# occupies (measured on B200 by a one-off probe: ~67 cycles for every
# M in {64, 128}, N <= 128, K = 16)
SSD_MMA_PER_CHUNK_HEAD = 28
SSD_CYCLES_PER_MMA = 67.0


def ssd_tensor_pipe_est(info, kern_s: float, sm_mhz: float) -> dict:
    """Issue-based estimate of the SSD kernel's tensor-pipe utilisation: MMA
    count x cycles per MMA over (kernel cycles x SMs).  ncu's measured
    figure is in profiles/; this one is recomputed from every run's time."""
    chunks = -(-info["seqlen"] // info["chunk"])
    busy = info["batch"] * info["nheads"] * chunks * SSD_MMA_PER_CHUNK_HEAD * SSD_CYCLES_PER_MMA
    cyc = kern_s * sm_mhz * 1e6
    ctas = info["batch"] * info["nheads"]
    return {"all_sms": busy / (cyc * SMS), "sms_used": min(ctas, SMS),
            "over_sms_used": busy / (cyc * min(ctas, SMS)),
            "mma_per_chunk_head": SSD_MMA_PER_CHUNK_HEAD, "cycles_per_mma": SSD_CYCLES_PER_MMA}


def step_stats(ms):
    """Median, p10 and p90 of the per-step CUDA-event times (ms)."""
    if len(ms) < 2:
        return {"median": ms[0], "p10": ms[0], "p90": ms[0]}
    q = statistics.quantiles(ms, n=10, method="inclusive")
    return {"median": statistics.median(ms), "p10": q[0], "p90": q[-1]}


def bwd_alu_peak_elems(sm_mhz: float) -> float:
    """Element rate the SM pipes allow for the backward (per element: three
    exps -- checkpoint pass, recompute, adjoint -- and 19 FMA-pipe operations:
    3 + 3 for the two forward recurrences, 11 in the adjoint step and about 2
    adds of the dB / dC warp reduction).  Exps split between the MUFU unit
    and an 8-operation FMA-pipe polynomial so that both pipes finish
    together: x / 16 = (19 + 8 (3 - x)) / 128 gives x = 43 / 16, i.e.
    256 / 43 elements per clock per SM."""
    return SMS * sm_mhz * 1e6 * (256.0 / 43.0)


# ------------------------------------------------------- multi-rank helpers

def rank_seed(rank: int) -> int:
    """Each rank scans its own batch (weak scaling): rank r draws seed r."""
    return rank


def max_over_ranks(ms: float, world: int, device=None) -> float:
    """The job's time: the max of a per-rank device time over all ranks."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step: float, world: int, steps: int, job_ms: float) -> float:
    """Units all ranks processed per second of job time."""
    return units_per_rank_step * world * steps / (job_ms * 1e-3)


def run_timed(step, flush, steps, world, device, new_event, sync):
    """The timed region every rank runs: a barrier and a synchronize on both
    sides, `steps` calls each bracketed by a pair of events (the flush before
    each call outside them), then the sum of the step times max-reduced over
    ranks.  new_event() returns an object with record() and
    elapsed_time(other) in ms (CUDA events on the launching stream on a GPU).
    Returns (per-step ms of this rank, job ms)."""
    import torch.distributed as dist
    evs = [(new_event(), new_event()) for _ in range(steps)]
    if world > 1:
        dist.barrier()
    sync()
    for i in range(steps):
        flush(i)
        evs[i][0].record()
        step()
        evs[i][1].record()
    sync()
    if world > 1:
        dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    return step_ms, max_over_ranks(float(sum(step_ms)), world, device)


class StreamEvent:
    """A timing CUDA event recorded on one stream."""

    def __init__(self, stream):
        import torch
        self.stream = stream
        self.ev = torch.cuda.Event(enable_timing=True)

    def record(self):
        self.ev.record(self.stream)

    def elapsed_time(self, other):
        return self.ev.elapsed_time(other.ev)


# ----------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows),
                "power_w_max": max((float(r[3]) for r in rows if r[3].replace(".", "").isdigit()),
                                   default=None)}


# ----------------------------------------------------------- device side

class DeviceWorkload:
    """Inputs resident in HBM plus the raw C-ABI call of one step."""

    def __init__(self, cfg, seed, device, op="scan"):
        import torch
        import selective_state_space_24_b200 as ssm
        self.torch, self.ssm, self.dev = torch, ssm, device
        self.cfg = cfg
        self.op = op
        self.info = workload_info(cfg)
        self.inp = ssm_gen.make_workload(cfg, seed=seed)
        self.lib = ssm.load()
        self.host = {}      # pinned host copies (for e2e)
        self.d = {}         # device tensors
        tdt = torch.float32 if self.inp.dtype == "f32" else torch.bfloat16
        for k, v in vars(self.inp).items():
            if isinstance(v, np.ndarray):
                io = k in self.inp.io_tensors()
                t = torch.from_numpy(np.ascontiguousarray(v, np.float32))
                t = (t.to(tdt) if io else t).pin_memory()
                self.host[k] = t
                self.d[k] = t.to(device)
        self.out = torch.empty_like(self.d["x"])
        self.out_host = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        self.last = {}
        if self.info["kind"] == "s6":
            self.dims = ssm.ssm_dims(self.inp.batch, self.inp.seqlen, self.inp.dim, self.inp.dstate,
                                     ssm.SSM_F32 if self.inp.dtype == "f32" else ssm.SSM_BF16)
            if self.info.get("last_state"):
                for s in ("f", "b"):
                    self.last[s] = torch.empty((self.inp.batch, self.inp.dim, self.inp.dstate),
                                               dtype=torch.float32, device=device)
            if self.info["ndir"] == 2:
                need = self.lib.bidir_scan_workspace_size(ctypes.byref(self.dims))
            else:
                need = self.lib.ssm_scan_workspace_size(ctypes.byref(self.dims))
        else:
            i = self.inp
            self.dims = ssm.ssd_dims(i.batch, i.seqlen, i.nheads, i.headdim, i.dstate, i.chunk,
                                     ssm.SSM_BF16)
            need = self.lib.ssd_chunk_workspace_size(ctypes.byref(self.dims))
        self.ws = torch.empty(max(int(need), 16), dtype=torch.uint8, device=device)
        self.ws_bytes = int(need)
        if op != "scan":
            assert self.info["kind"] == "s6" and self.info["ndir"] == 2, \
                "ordered / conv / fwd_ckpt / zoh: bidirectional S6"
            i = self.inp
            rng = np.random.default_rng(seed + 1)
            if op == "fwd_ckpt":
                nck = int(self.lib.ssm_scan_ckpt_size(ctypes.byref(self.dims))) // 4
                self.ckpt = (torch.empty(nck, dtype=torch.float32, device=device),
                             torch.empty(nck, dtype=torch.float32, device=device))
            elif op == "zoh":
                pass
            elif op == "ordered":
                self.order = torch.from_numpy(ssm_gen.order_random(i.seqlen, seed=seed)).to(device)
                self.mask = torch.from_numpy(ssm_gen.token_mask(i.batch, i.seqlen, 0.7, seed=seed)).to(device)
            else:
                mk = lambda: torch.from_numpy((rng.standard_normal((i.dim, 4)) / 2).astype(np.float32)).to(device)
                self.convw = (mk(), mk())
                self.convb = torch.zeros(i.dim, device=device)
                self.conv_f = ssm.ssm_conv_params(self.convw[0].data_ptr(), self.convb.data_ptr(), 4, 1)
                self.conv_b = ssm.ssm_conv_params(self.convw[1].data_ptr(), self.convb.data_ptr(), 4, 1)
        self.launches_per_step = self._launches()
        self._bind()

    def _launches(self):
        """Kernel launches of one call: the S6 plan's segment count decides
        (summary, carry and main passes, or the main pass alone).  The plain
        and checkpointing scans take the reported plan; the ordered / conv
        variants always give each thread whole channels, so their plan is
        read under that layout."""
        if self.info["kind"] != "s6" or self.op == "zoh":
            return 1   # (the zero-order-hold scans always run as one split-state pass)
        seg, cpl = ctypes.c_int(0), ctypes.c_int(0)
        query = lambda: self.lib.ssm_scan_plan(ctypes.byref(self.dims), int(self.info["ndir"] == 2),
                                               ctypes.byref(seg), ctypes.byref(cpl))
        if self.op in ("scan", "fwd_ckpt"):
            st = query()
        else:
            self.lib.ssm_debug_s6_mapping(1)
            try:
                st = query()
            finally:
                self.lib.ssm_debug_s6_mapping(0)
        assert st == 0, st
        return 3 if seg.value > 1 else 1

    def _bind(self):
        d = self.d
        p = lambda t: None if t is None else t.data_ptr()
        if self.info["kind"] == "s6" and self.info["ndir"] == 2:
            self.fwd = self.ssm.ssm_dir_params(p(d["dt_bias_f"]), p(d["A_f"]), p(d["B_f"]),
                                               p(d["C_f"]), p(d["D_f"]), p(d.get("z_f")),
                                               p(self.last.get("f")))
            self.bwd = self.ssm.ssm_dir_params(p(d["dt_bias_b"]), p(d["A_b"]), p(d["B_b"]),
                                               p(d["C_b"]), p(d["D_b"]), p(d.get("z_b")),
                                               p(self.last.get("b")))

    def step(self, stream_handle):
        """One call of the hot path through the C ABI (inputs resident)."""
        d, lib = self.d, self.lib
        p = lambda t: None if t is None else t.data_ptr()
        if self.op == "ordered":
            st = lib.bidir_scan_fwd_ordered(ctypes.byref(self.dims), p(d["x"]), p(d["delta"]), 1,
                                            ctypes.byref(self.fwd), ctypes.byref(self.bwd), p(self.order),
                                            p(self.mask), p(self.out), p(self.ws), self.ws_bytes,
                                            stream_handle)
        elif self.op == "fwd_ckpt":
            st = lib.bidir_scan_fwd_ckpt(ctypes.byref(self.dims), p(d["x"]), p(d["delta"]), 1,
                                         ctypes.byref(self.fwd), ctypes.byref(self.bwd), p(self.out),
                                         p(self.ckpt[0]), p(self.ckpt[1]), p(self.ws), self.ws_bytes,
                                         stream_handle)
        elif self.op == "zoh":
            st = lib.bidir_scan_fwd_zoh(ctypes.byref(self.dims), p(d["x"]), p(d["delta"]), 1,
                                        ctypes.byref(self.fwd), ctypes.byref(self.bwd), p(self.out),
                                        p(self.ws), self.ws_bytes, stream_handle)
        elif self.op == "conv":
            st = lib.bidir_scan_fwd_conv(ctypes.byref(self.dims), p(d["x"]), p(d["delta"]), 1,
                                         ctypes.byref(self.fwd), ctypes.byref(self.bwd),
                                         ctypes.byref(self.conv_f), ctypes.byref(self.conv_b), p(self.out),
                                         p(self.ws), self.ws_bytes, stream_handle)
        elif self.info["kind"] == "s6" and self.info["ndir"] == 2:
            st = lib.bidir_scan_fwd(ctypes.byref(self.dims), p(d["x"]), p(d["delta"]), 1,
                                    ctypes.byref(self.fwd), ctypes.byref(self.bwd), p(self.out),
                                    p(self.ws), self.ws_bytes, stream_handle)
        elif self.info["kind"] == "s6":
            st = lib.ssm_scan_fwd(ctypes.byref(self.dims), p(d["x"]), p(d["delta"]),
                                  p(d["dt_bias_f"]), 1, p(d["A_f"]), p(d["B_f"]), p(d["C_f"]),
                                  p(d["D_f"]), p(d.get("z_f")), 0, p(self.out), None, p(self.ws),
                                  self.ws_bytes, stream_handle)
        else:
            st = lib.ssd_chunk_fwd(ctypes.byref(self.dims), p(d["x"]), p(d["delta"]),
                                   p(d["dt_bias"]), 1, p(d["A"]), p(d["B"]), p(d["C"]), p(d["D"]),
                                   p(d.get("z")), p(self.out), None, p(self.ws), self.ws_bytes,
                                   stream_handle)
        if st != 0:
            raise RuntimeError(f"hot path returned {self.ssm.STATUS.get(st, st)}")

    def e2e_setup(self):
        """A second device copy of the inputs and output, one stream per copy
        direction and the events that order them, for the pipelined
        end-to-end loop (step i's result can go out while step i + 1's
        inputs come in: PCIe carries both directions at once)."""
        torch = self.torch
        self.sets = [(self.d, self.out),
                     ({k: torch.empty_like(v) for k, v in self.d.items()}, torch.empty_like(self.out))]
        self.s_h2d = torch.cuda.Stream(self.dev)
        self.s_d2h = torch.cuda.Stream(self.dev)
        self.ev = {n: [torch.cuda.Event(), torch.cuda.Event()] for n in ("h2d", "comp", "d2h")}
        self.used = [False, False]

    def e2e_step(self, i, comp):
        """Step i end to end: H2D of every input from pinned memory into buffer
        set i % 2 (after step i - 2's call is done with it), the call on
        stream `comp`, D2H of its output (the call waits until step i - 2's
        output has left the set).  Returns (h2d bytes, d2h bytes)."""
        torch = self.torch
        s = i % 2
        d, out = self.sets[s]
        if self.used[s]:
            self.s_h2d.wait_event(self.ev["comp"][s])
        hb = 0
        with torch.cuda.stream(self.s_h2d):
            for k, t in self.host.items():
                d[k].copy_(t, non_blocking=True)
                hb += t.numel() * t.element_size()
            self.ev["h2d"][s].record(self.s_h2d)
        comp.wait_event(self.ev["h2d"][s])
        if self.used[s]:
            comp.wait_event(self.ev["d2h"][s])
        self.d, self.out = d, out
        self._bind()
        self.step(comp.cuda_stream)
        self.ev["comp"][s].record(comp)
        self.s_d2h.wait_event(self.ev["comp"][s])
        with torch.cuda.stream(self.s_d2h):
            self.out_host.copy_(out, non_blocking=True)
            self.ev["d2h"][s].record(self.s_d2h)
        self.used[s] = True
        return hb, out.numel() * out.element_size()

    def e2e_done(self, comp):
        """Join the copy streams into `comp` and go back to buffer set 0."""
        comp.wait_stream(self.s_h2d)
        comp.wait_stream(self.s_d2h)
        self.d, self.out = self.sets[0]
        self._bind()


def config_dict(info, cfg, op, world):
    """The workload a line measures; the same dict in both arms."""
    return {"workload": info["name"] + ("" if op == "scan" else "_" + op),
            "config_index": cfg, "op": op,
            **{k: info[k] for k in ("batch", "seqlen", "dim", "dstate", "nheads", "headdim", "chunk")
               if k in info},
            "directions": info["ndir"], "parallelism": f"dp{world} (independent batches)",
            "l2": "flushed before every timed step (512 MB write)",
            "algorithmic_bytes_per_step": info["bytes"],
            "elements_per_step": info["elems"]}


def roofline(info, kern_s, traffic):
    """Roofline of one call: the HBM fraction of the algorithmic bytes (the
    graded bound for every workload), and beside it, for S6, the two derived
    on-chip bounds (MUFU-only exp, and exps split between MUFU and the FMA
    pipe); for SSD the issue-based tensor-pipe estimate."""
    peaks, peak_src = load_peaks()
    mhz = peaks.get("sm_max_mhz", 1965.0)
    hbm_ach = info["bytes"] / kern_s / 1e9
    r = {"bound": "hbm", "achieved": hbm_ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
         "frac": hbm_ach / peaks["hbm_gbs"], "traffic": traffic, "peak_source": peak_src,
         "algorithmic_bytes": info["bytes"], "kernel_ms_median": kern_s * 1e3}
    if info["kind"] == "s6":
        ach = info["elems"] / kern_s
        mp, ap = mufu_peak_elems(mhz), alu_peak_elems(mhz)
        r.update({"elements_per_s": ach, "mufu_peak_gelems": mp / 1e9, "mufu_frac": ach / mp,
                  "alu_peak_gelems": ap / 1e9, "alu_frac": ach / ap,
                  "derived_bounds": "derived, not measured peaks: mufu = one exp per element on the "
                                    "MUFU unit (16/clk/SM); alu = exps split between MUFU and an "
                                    "8-operation FMA-pipe polynomial, 4 FMA-pipe operations per "
                                    "element (64/3 elements/clk/SM); both at sm_max_mhz"})
    else:
        r["tensor_pipe_est"] = ssd_tensor_pipe_est(info, kern_s, mhz)
    return r


def time_steps(wl, stream, flush, warmup, steps):
    """Per-step CUDA-event times (ms) of `steps` calls after `warmup` untimed
    ones, the L2 flushed (outside the events) before every call."""
    import torch
    sh = stream.cuda_stream
    for _ in range(max(warmup, 3)):
        flush.fill_(1.0)
        wl.step(sh)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for i in range(steps):
        flush.fill_(float(i))
        evs[i][0].record(stream)
        wl.step(sh)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


ERR_SAMPLE_COLS = 256


def output_columns(out, info, cols):
    """Whole-sequence output columns `cols` of one call's output, as (n, L):
    column b * D + d of an S6 output (B, L, D), (b * H + h) * P + p of an SSD
    output (B, L, H, P)."""
    cols = np.asarray(cols)
    if info["kind"] == "s6":
        b, d = np.divmod(cols, info["dim"])
        return out[b, :, d]
    H, P = info["nheads"], info["headdim"]
    b, r = np.divmod(cols, H * P)
    h, p = np.divmod(r, P)
    return out[b, :, h, p]


def sample_columns(wl, cfg):
    """A seeded sample of whole-sequence output columns of the last call,
    copied to the host (for the CPU leg's check against the oracle)."""
    import torch
    info = wl.info
    ncols = info["batch"] * (info["dim"] if info["kind"] == "s6" else info["nheads"] * info["headdim"])
    rng = np.random.default_rng(1000 + cfg)
    cols = np.sort(rng.choice(ncols, min(ncols, ERR_SAMPLE_COLS), replace=False))
    g = output_columns(wl.out.float().cpu().numpy(), info, cols)
    return cols, ncols, np.asarray(g, dtype=np.float64)


PER_CONFIG_WARMUP, PER_CONFIG_STEPS = 20, 100


def measure_configs(device, stream, flush):
    """Every workload (0-4) timed the same way -- 20 warm-up and 100 timed
    calls, L2 flushed before each -- with its roofline; returns the entries
    and, per workload, a sample of output columns for the oracle check."""
    import torch
    entries, samples = [], {}
    for cfg in sorted(ssm_gen.WORKLOADS):
        wl = DeviceWorkload(cfg, seed=0, device=device)
        ms = time_steps(wl, stream, flush, PER_CONFIG_WARMUP, PER_CONFIG_STEPS)
        info = wl.info
        st = step_stats(ms)
        kern_s = st["median"] * 1e-3
        roof = roofline(info, kern_s, NCU_TRAFFIC.get(cfg))
        e = {"config_index": cfg, "workload": info["name"], "ms": st,
             "elements_per_s": info["elems"] / kern_s, "hbm_gbs": roof["achieved"],
             "hbm_frac": roof["frac"], "launches_per_call": wl.launches_per_step}
        if info["kind"] == "s6":
            e.update(mufu_frac=roof["mufu_frac"], alu_frac=roof["alu_frac"])
        else:
            e["tensor_pipe_est"] = roof["tensor_pipe_est"]
        entries.append(e)
        samples[cfg] = (wl.inp, info, *sample_columns(wl, cfg))
        del wl
        torch.cuda.empty_cache()
    return entries, samples


def rel_err(g, o) -> float:
    """max_i |g_i - o_i| / max(|o_i|, rms(o)): the error measure of the parity
    tests (a plain ratio is meaningless at gated near-zero outputs)."""
    rms = float(np.sqrt(np.mean(o * o))) if o.size else 0.0
    den = np.maximum(np.abs(o), max(rms, 1e-30))
    return float(np.max(np.abs(g - o) / den)) if o.size else 0.0


def oracle_errors(samples, threads):
    """CPU leg: the float64 oracle on each sampled column set, and the max
    relative error of the GPU columns against it."""
    import oracle
    res = {}
    for cfg, (inp, info, cols, ncols, g) in samples.items():
        t0 = time.perf_counter()
        if info["kind"] == "s6":
            ref = (oracle.bidir(inp, cols=cols, nthreads=threads)[0] if info["ndir"] == 2
                   else oracle.s6(inp, cols=cols, nthreads=threads)[0])
        else:
            ref = oracle.ssd_seq(inp, cols=cols, nthreads=threads)[0]
        o = output_columns(ref, info, cols)
        err = rel_err(g, o)
        tol = 1e-4 if info["dtype"] == "f32" else 2e-2
        res[cfg] = {"max_rel_err": err, "tol": tol, "pass": bool(err <= tol),
                    "sample": f"{len(cols)} of {ncols} columns, whole sequence each",
                    "oracle_s": time.perf_counter() - t0}
    return res


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from selective_state_space_24_b200 import build as ssm_build
    ssm_build.build()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    info = workload_info(args.config, args.op)
    wl = DeviceWorkload(args.config, seed=rank_seed(rank), device=device, op=args.op)
    stream = torch.cuda.current_stream(device)
    sh = stream.cuda_stream
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)

    for _ in range(max(args.warmup, 3)):
        flush.fill_(1.0)
        wl.step(sh)
    torch.cuda.synchronize()
    assert torch.isfinite(wl.out.float()).all().item(), "non-finite output"

    sampler = ClockSampler(local_rank)
    sampler.start()
    t_wall = time.perf_counter()
    step_ms, total_ms = run_timed(lambda: wl.step(sh), lambda i: flush.fill_(float(i)), args.steps, world,
                                  device, lambda: StreamEvent(stream), torch.cuda.synchronize)
    wall = time.perf_counter() - t_wall
    clocks = sampler.stop()
    per_step_ms = total_ms / args.steps
    value = job_throughput(info["elems"], world, args.steps, total_ms)

    # roofline of the call (one launch when the plan has a single segment;
    # else summary + carry + main, all inside the measured time)
    kern_s = statistics.median(step_ms) * 1e-3
    roof = roofline(info, kern_s, NCU_TRAFFIC.get(args.config) if args.op == "scan" else None)

    e2e = None
    if not args.no_e2e:
        ke = max(3, min(args.steps, 20))
        wl.e2e_setup()
        for i in range(2):
            wl.e2e_step(i, stream)
        wl.e2e_done(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        wl.s_h2d.wait_event(e0)       # every copy of the timed steps starts after e0
        hb = db = 0
        for i in range(ke):
            hb, db = wl.e2e_step(i, stream)
        wl.e2e_done(stream)           # e1 follows the last D2H
        e1.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), world, device)
        e2e = {"value": job_throughput(info["elems"], world, ke, ems), "unit": "elements/s",
               "h2d_bytes_per_step": hb, "d2h_bytes_per_step": db, "steps": ke,
               "ms_per_step": ems / ke}
    launches = wl.launches_per_step * args.steps
    del wl
    torch.cuda.empty_cache()

    # every workload, one GPU only (the per-rank batch sharding of the
    # headline needs no second pass at N > 1)
    per_config, samples, pc_clocks = None, None, None
    if world == 1 and args.op == "scan" and not args.no_per_config:
        pcs = ClockSampler(local_rank)
        pcs.start()
        per_config, samples = measure_configs(device, stream, flush)
        pc_clocks = pcs.stop()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.op == "scan":
        cpu = cpu_baseline(args.config, budget_s=10.0)
        if samples:
            errs = oracle_errors(samples, cpu["cores"])
            for e in per_config:
                e["oracle_check"] = errs[e["config_index"]]

    res = {
        "metric": METRIC, "value": value, "unit": "elements/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step_ms,
        "step_ms": step_stats(step_ms),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32" if info["dtype"] == "f32" else "bf16 storage, f32 compute",
        "data": "synthetic (seeded ssm_gen inputs with the workload's shapes and distributions)",
        "config": config_dict(info, args.config, args.op, world),
        "hbm_gbs": info["bytes"] / (per_step_ms * 1e-3) / 1e9,
        "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks, "wall_s_timed_region": wall,
    }
    if per_config is not None:
        res["per_config"] = per_config
        res["per_config_protocol"] = (f"{PER_CONFIG_WARMUP} warm-up and {PER_CONFIG_STEPS} timed calls "
                                      "per workload, L2 flushed before each, CUDA events; oracle_check "
                                      "from the CPU leg (float64 oracle on sampled columns)")
        res["per_config_clocks"] = pc_clocks
    return res


# ------------------------------------------------------- decode step

STEP_WORKLOAD = {"batch": 512, "dim": 1536, "dstate": 16}


def run_step(args):
    """One decode step (ssm_step) of a (512, 1536, 16) fp32 state with fp32
    activations, timed like the scan: inputs resident, L2 flushed before
    every step, CUDA events on the launching stream.  HBM-bound: the state
    is read and written once."""
    import ctypes
    import torch
    from selective_state_space_24_b200 import build as ssm_build
    import selective_state_space_24_b200 as ssm
    ssm_build.build()
    lib = ssm.load()
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    Bz, Dm, N = STEP_WORKLOAD["batch"], STEP_WORKLOAD["dim"], STEP_WORKLOAD["dstate"]
    inp = ssm_gen.make_s6_inputs(Bz, 1, Dm, N, dtype="f32", seed=0)
    f = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)
    x, delta, z = f(inp.x[:, 0]), f(inp.delta[:, 0]), f(inp.z_f[:, 0])
    Bm, Cm = f(inp.B_f[:, 0]), f(inp.C_f[:, 0])
    A, bias, Dv = f(inp.A_f), f(inp.dt_bias_f), f(inp.D_f)
    state = torch.zeros((Bz, Dm, N), device=device)
    out = torch.empty_like(x)
    dims = ssm.ssm_dims(Bz, 1, Dm, N, ssm.SSM_F32)
    p = lambda t: t.data_ptr()
    stream = torch.cuda.current_stream(device)
    sh = stream.cuda_stream

    def step():
        st = lib.ssm_step(ctypes.byref(dims), p(x), p(delta), p(bias), 1, p(A), p(Bm), p(Cm), p(Dv),
                          p(z), p(state), p(out), sh)
        if st != 0:
            raise RuntimeError(f"ssm_step returned {ssm.STATUS.get(st, st)}")

    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    for _ in range(max(args.warmup, 3)):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    sampler = ClockSampler(0)
    sampler.start()
    for i in range(args.steps):
        flush.fill_(float(i))
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = [a.elapsed_time(b) for a, b in evs]
    med = statistics.median(ms)
    elems = Bz * Dm * N
    nbytes = 2 * elems * 4 + 4 * Bz * Dm * 4 + 2 * Bz * N * 4 + Dm * N * 4 + 2 * Dm * 4
    peaks, peak_src = load_peaks()
    hbm = nbytes / (med * 1e-3) / 1e9
    return {
        "metric": "decode step: state elements/s (B·D·N) and HBM GB/s", "value": elems / (med * 1e-3),
        "unit": "elements/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sum(ms) / len(ms), "step_ms": step_stats(ms), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded ssm_gen inputs)",
        "config": {"workload": "decode_step_b512_d1536_n16_fp32", **STEP_WORKLOAD,
                   "l2": "flushed before every timed step (512 MB write)",
                   "algorithmic_bytes_per_step": nbytes},
        "roofline": {"bound": "hbm", "achieved": hbm, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": hbm / peaks["hbm_gbs"], "traffic": NCU_TRAFFIC_STEP, "peak_source": peak_src,
                     "kernel_ms_median": med},
        "gpu_launches": args.steps, "clocks": clocks,
    }


# ---------------------------------------------------------- backward

def run_bwd(args):
    """Gradients of an S6 workload: of its forward direction (ssm_scan_bwd,
    --op bwd) or of the whole bidirectional scan (bidir_scan_bwd, --op
    bidir_bwd); inputs and the incoming gradient resident, L2 flushed before
    every step, CUDA events on the launching stream."""
    import ctypes
    import torch
    from selective_state_space_24_b200 import build as ssm_build
    import selective_state_space_24_b200 as ssm
    ssm_build.build()
    lib = ssm.load()
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    info = workload_info(args.config)
    assert info["kind"] == "s6", "bwd: an S6 workload"
    inp = ssm_gen.make_workload(args.config, seed=0)
    tdt = torch.float32 if inp.dtype == "f32" else torch.bfloat16
    io = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(tdt).to(device)
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)
    x, delta, z, Bm, Cm = io(inp.x), io(inp.delta), io(inp.z_f), io(inp.B_f), io(inp.C_f)
    dout = io(np.random.default_rng(1).standard_normal(inp.x.shape))
    A, bias, Dv = f32(inp.A_f), f32(inp.dt_bias_f), f32(inp.D_f)
    e = lambda shape: torch.empty(shape, dtype=torch.float32, device=device)
    g = [e(x.shape), e(x.shape), e(A.shape), e(Bm.shape), e(Cm.shape), e(Dv.shape), e(x.shape),
         e(bias.shape)]
    dims = ssm.ssm_dims(inp.batch, inp.seqlen, inp.dim, inp.dstate,
                        ssm.SSM_F32 if inp.dtype == "f32" else ssm.SSM_BF16)
    need = int(lib.ssm_scan_bwd_workspace_size(ctypes.byref(dims)))
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=device)
    p = lambda t: t.data_ptr()
    stream = torch.cuda.current_stream(device)
    sh = stream.cuda_stream
    bidir = args.op in ("bidir_bwd", "bidir_bwd_ckpt")
    from_ckpt = args.op.endswith("_ckpt")
    if bidir:
        assert info["ndir"] == 2, "bidir_bwd: a bidirectional workload"
        zb, Bb, Cb = io(inp.z_b), io(inp.B_b), io(inp.C_b)
        Ab, biasb, Db = f32(inp.A_b), f32(inp.dt_bias_b), f32(inp.D_b)
        pf = ssm.ssm_dir_params(p(bias), p(A), p(Bm), p(Cm), p(Dv), p(z), None)
        pb = ssm.ssm_dir_params(p(biasb), p(Ab), p(Bb), p(Cb), p(Db), p(zb), None)
        gb = [e(A.shape), e(Bb.shape), e(Cb.shape), e(Dv.shape), e(x.shape), e(bias.shape)]
        gf_c = ssm.ssm_dir_grads(*[p(t) for t in (g[2], g[3], g[4], g[5], g[6], g[7])])
        gb_c = ssm.ssm_dir_grads(*[p(t) for t in gb])

    if from_ckpt:
        # the checkpoints of the checkpointing forward, written once (untimed)
        nck = int(lib.ssm_scan_ckpt_size(ctypes.byref(dims))) // 4
        ck = [torch.empty(nck, dtype=torch.float32, device=device) for _ in range(2)]
        out = torch.empty_like(x)
        wsz = lib.bidir_scan_workspace_size if bidir else lib.ssm_scan_workspace_size
        fws = torch.empty(max(int(wsz(ctypes.byref(dims))), 16), dtype=torch.uint8, device=device)
        if bidir:
            st = lib.bidir_scan_fwd_ckpt(ctypes.byref(dims), p(x), p(delta), 1, ctypes.byref(pf), ctypes.byref(pb),
                                         p(out), p(ck[0]), p(ck[1]), p(fws), fws.numel(), sh)
        else:
            st = lib.ssm_scan_fwd_ckpt(ctypes.byref(dims), p(x), p(delta), p(bias), 1, p(A), p(Bm), p(Cm), p(Dv),
                                       p(z), 0, p(out), None, p(ck[0]), p(fws), fws.numel(), sh)
        if st != 0:
            raise RuntimeError(f"checkpointing forward returned {ssm.STATUS.get(st, st)}")

    def step():
        if bidir and from_ckpt:
            st = lib.bidir_scan_bwd_ckpt(ctypes.byref(dims), p(x), p(delta), 1, ctypes.byref(pf), ctypes.byref(pb),
                                         p(dout), p(g[0]), p(g[1]), ctypes.byref(gf_c), ctypes.byref(gb_c),
                                         p(ck[0]), p(ck[1]), sh)
        elif bidir:
            st = lib.bidir_scan_bwd(ctypes.byref(dims), p(x), p(delta), 1, ctypes.byref(pf), ctypes.byref(pb),
                                    p(dout), p(g[0]), p(g[1]), ctypes.byref(gf_c), ctypes.byref(gb_c), p(ws),
                                    need, sh)
        elif from_ckpt:
            st = lib.ssm_scan_bwd_ckpt(ctypes.byref(dims), p(x), p(delta), p(bias), 1, p(A), p(Bm), p(Cm), p(Dv),
                                       p(z), 0, p(dout), *[p(t) for t in g], p(ck[0]), sh)
        else:
            st = lib.ssm_scan_bwd(ctypes.byref(dims), p(x), p(delta), p(bias), 1, p(A), p(Bm), p(Cm), p(Dv),
                                  p(z), 0, p(dout), *[p(t) for t in g], p(ws), need, sh)
        if st != 0:
            raise RuntimeError(f"backward returned {ssm.STATUS.get(st, st)}")

    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    for _ in range(max(args.warmup, 3)):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    sampler = ClockSampler(0)
    sampler.start()
    for i in range(args.steps):
        flush.fill_(float(i))
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = [a.elapsed_time(b) for a, b in evs]
    med = statistics.median(ms)
    nd = 2 if bidir else 1
    elems = nd * inp.batch * inp.seqlen * inp.dim * inp.dstate
    es = 4 if inp.dtype == "f32" else 2
    BL, BLD = inp.batch * inp.seqlen, inp.batch * inp.seqlen * inp.dim
    # inputs x, delta, dout (dtype) and per direction z, B, C; outputs dx, ddelta (fp32) and per
    # direction dz, dB, dC (fp32)
    nbytes = (3 + nd) * BLD * es + 2 * nd * BL * inp.dstate * es + (2 + nd) * BLD * 4 \
        + 2 * nd * BL * inp.dstate * 4
    peaks, peak_src = load_peaks()
    alu_peak = bwd_alu_peak_elems(peaks.get("sm_max_mhz", 1965.0))
    return {
        "metric": "backward: scan elements/s (B·L·D·N)", "value": elems / (med * 1e-3),
        "unit": "elements/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sum(ms) / len(ms), "step_ms": step_stats(ms), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": info["dtype"], "data": "synthetic (seeded ssm_gen inputs)",
        "config": {"workload": info["name"] + ("_bidir_bwd" if bidir else "_fwd_direction_bwd")
                   + ("_from_checkpoints" if from_ckpt else ""),
                   "config_index": args.config,
                   "l2": "flushed before every timed step (512 MB write)",
                   "algorithmic_bytes_per_step": nbytes, "elements_per_step": elems},
        "hbm_gbs": nbytes / (med * 1e-3) / 1e9,
        "roofline": {"bound": "alu", "achieved": elems / (med * 1e-3) / 1e9, "peak": alu_peak / 1e9,
                     "unit": "Gelem/s", "frac": elems / (med * 1e-3) / alu_peak,
                     "traffic": None if (bidir or from_ckpt) else NCU_TRAFFIC_BWD.get(args.config),
                     "peak_source": peak_src,
                     "kernel_ms_median": med,
                     "note": ("achieved over the whole call (backward kernel per direction, the checkpoints "
                              "read from the checkpointing forward); " if from_ckpt else
                              "achieved over the whole call (checkpoint pass + backward kernel per direction); ")
                             + "traffic of the backward kernel, the dominant launch"},
        "gpu_launches": (1 if from_ckpt else 2) * nd * args.steps, "clocks": clocks,
    }


# ------------------------------------------------------------ CPU oracle

def _oracle_sample(cfg, frac_cols):
    """Inputs and column sample for a bounded oracle run of workload cfg."""
    inp = ssm_gen.make_workload(cfg, seed=0)
    info = workload_info(cfg)
    if info["kind"] == "s6":
        ncols_all = inp.batch * inp.dim
    else:
        ncols_all = inp.batch * inp.nheads * inp.headdim
    n = max(1, min(ncols_all, int(ncols_all * frac_cols)))
    cols = np.random.default_rng(0).choice(ncols_all, n, replace=False)
    return inp, info, cols, ncols_all


def _oracle_call(inp, info, cols, threads):
    import oracle
    if info["kind"] == "s6":
        if info["ndir"] == 2:
            oracle.bidir(inp, cols=cols, nthreads=threads)
        else:
            oracle.s6(inp, cols=cols, nthreads=threads)
    else:
        oracle.ssd_seq(inp, cols=cols, nthreads=threads)


def cpu_baseline(cfg, budget_s=10.0):
    """The float64 oracle as it stands, on this host's cores, over a sample of
    the workload's columns sized to about `budget_s` seconds (the whole
    workload, repeated, when one pass is shorter)."""
    threads = len(os.sched_getaffinity(0))
    inp, info, cols, ncols_all = _oracle_sample(cfg, 1.0)
    per_col = info["elems"] / ncols_all
    _oracle_call(inp, info, cols[: threads * 4], threads)        # warm the thread pool
    probe = cols[: max(threads * 16, ncols_all // 16)]
    t0 = time.perf_counter()
    _oracle_call(inp, info, probe, threads)
    per_col_s = max(time.perf_counter() - t0, 1e-6) / len(probe)
    if per_col_s * ncols_all <= budget_s:
        reps = max(1, int(budget_s / (per_col_s * ncols_all)))
        sample, what = cols, f"the whole workload ({ncols_all} columns) x {reps}"
    else:
        reps = 1
        sample = cols[: max(len(probe), int(budget_s / per_col_s))]
        what = f"{len(sample)} of {ncols_all} (batch, channel) columns, whole sequence each"
    t0 = time.perf_counter()
    for _ in range(reps):
        _oracle_call(inp, info, sample, threads)
    el = time.perf_counter() - t0
    # the same oracle on one core, over a sample sized to about budget_s / 2
    col1_s = per_col_s * threads                      # estimate of one column on one core
    one = cols[: max(1, min(len(cols), int(budget_s / 2 / col1_s)))]
    reps1 = max(1, int(budget_s / 2 / (col1_s * len(one))))
    t0 = time.perf_counter()
    for _ in range(reps1):
        _oracle_call(inp, info, one, 1)
    el1 = time.perf_counter() - t0
    return {"value": len(sample) * reps * per_col / el, "unit": "elements/s", "cores": threads,
            "kind": "oracle", "sample": f"{what}, {el:.1f} s, float64 C oracle, OpenMP",
            "seconds": el,
            "one_core": {"value": len(one) * reps1 * per_col / el1, "unit": "elements/s", "cores": 1,
                         "sample": f"{len(one)} of {ncols_all} columns x {reps1}, {el1:.1f} s"}}


def run_reference(args):
    threads = len(os.sched_getaffinity(0))
    info = workload_info(args.config)
    inp, _, cols, ncols_all = _oracle_sample(args.config, 1.0)
    per_col = info["elems"] / ncols_all
    probe = cols[: max(threads * 2, 8)]
    t0 = time.perf_counter()
    _oracle_call(inp, info, probe, threads)
    dt = max(time.perf_counter() - t0, 1e-6)
    # size each step so that warm-up + steps take about one minute in all
    per_step_budget = 60.0 / max(1, args.steps + args.warmup)
    n = int(min(len(cols), max(len(probe), len(probe) * per_step_budget / dt)))
    sample = cols[:n]
    for _ in range(args.warmup):
        _oracle_call(inp, info, sample, threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_call(inp, info, sample, threads)
    el = time.perf_counter() - t0
    value = n * per_col * args.steps / el
    samp = f"{n} of {ncols_all} (batch, channel) columns per step, whole sequence each"
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "elements/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(info, args.config, "scan", args.gpus),
        "cpu_baseline": {"value": value, "unit": "elements/s", "cores": threads,
                         "kind": "oracle", "sample": samp},
        "e2e": {"value": value, "unit": "elements/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if args.op in ("step", "bwd", "bidir_bwd", "bwd_ckpt", "bidir_bwd_ckpt"):
        if rank == 0:
            print(json.dumps(run_step(args) if args.op == "step" else run_bwd(args)), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        res = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
