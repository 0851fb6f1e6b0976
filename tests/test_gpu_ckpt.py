"""The checkpointing training pair (ssm_scan_fwd_ckpt / ssm_scan_bwd_ckpt and
the bidirectional forms) through the C ABI: the forward's outputs equal the
plain forward's, its checkpoint array equals the one the backward's own
recompute pass writes, and the gradients from it match the float64 autograd
oracle."""
import ctypes

import numpy as np
import pytest
import torch

import ssm_gen
import selective_state_space_24_b200 as ssm
from oracle import grads as ograds
from gpu_util import TOL, dev, dir_params, f32dev, rel_err


def host_f(t):
    return t.float().cpu().numpy()

pytestmark = pytest.mark.gpu

NAMES = {"dx": "x", "ddelta": "delta", "dA": "A", "dB": "B", "dC": "C", "dD": "D", "dz": "z",
         "ddelta_bias": "delta_bias"}


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    ssm.load()


def _inputs(inp, dtype):
    return dict(x=dev(inp.x, dtype), delta=dev(inp.delta, dtype), A=f32dev(inp.A_f), B=dev(inp.B_f, dtype),
                C=dev(inp.C_f, dtype), delta_bias=f32dev(inp.dt_bias_f), D=f32dev(inp.D_f),
                z=dev(inp.z_f, dtype))


def _ckpt_segments(B, L, D, dtype):
    """Segments of the checkpointing forward's plan (the plain call's plan:
    one for the split-state layouts)."""
    return ssm.scan_plan(B, L, D, 16, ssm.SSM_F32 if dtype == "f32" else ssm.SSM_BF16)[0]


def _recomputed_ckpt(t, reverse, dout):
    """The checkpoint array the backward's own recompute pass writes (the
    raw C call, with a workspace the test owns)."""
    lib = ssm.capi()
    dims = ssm.s6_dims(t["x"], t["A"].shape[1])
    need = lib.ssm_scan_bwd_workspace_size(ctypes.byref(dims))
    ws = torch.zeros(need // 4, dtype=torch.float32, device="cuda")
    f32 = lambda shape: torch.empty(shape, dtype=torch.float32, device="cuda")
    x = t["x"]
    g = [f32(x.shape), f32(x.shape), f32(t["A"].shape), f32(t["B"].shape), f32(t["C"].shape), f32(t["D"].shape),
         f32(x.shape), f32(t["delta_bias"].shape)]
    p = lambda u: u.data_ptr()
    st = lib.ssm_scan_bwd(ctypes.byref(dims), p(x), p(t["delta"]), p(t["delta_bias"]), 1, p(t["A"]), p(t["B"]),
                          p(t["C"]), p(t["D"]), p(t["z"]), int(reverse), p(dout), *[p(u) for u in g], p(ws), need,
                          torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    return ws


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("L", [101, 3000])
def test_fwd_ckpt_outputs_and_checkpoints(dtype, reverse, L):
    """The checkpointing forward writes the plain forward's outputs and last
    state bit for bit (both take the plan's layout), and to rounding those
    of the one-channel layout when the plan splits the states over threads.
    It also writes the state entering every 4-step chunk: equal bit for bit
    to the backward's recompute when the plan has one segment, and within
    rounding of it when the sequence is cut into segments (entering states
    then come from the carry pass)."""
    inp = ssm_gen.make_s6_inputs(2, L, 96, 16, dtype=dtype, seed=L + reverse, random_A=True, random_D=True)
    t = _inputs(inp, dtype)
    ls0 = torch.zeros((2, 96, 16), device="cuda")
    ls1 = torch.zeros((2, 96, 16), device="cuda")
    ls2 = torch.zeros((2, 96, 16), device="cuda")
    kw = dict(delta_bias=t["delta_bias"], D=t["D"], z=t["z"], reverse=reverse)
    out0 = ssm.ssm_scan_fwd(t["x"], t["delta"], t["A"], t["B"], t["C"], last_state=ls0, **kw)
    with ssm.s6_mapping(ssm.MAPPING_WHOLE_CHANNELS):
        out2 = ssm.ssm_scan_fwd(t["x"], t["delta"], t["A"], t["B"], t["C"], last_state=ls2, **kw)
    out1, ck = ssm.ssm_scan_fwd_ckpt(t["x"], t["delta"], t["A"], t["B"], t["C"], last_state=ls1, **kw)
    torch.cuda.synchronize()
    assert torch.equal(out0, out1) and torch.equal(ls0, ls1)
    assert rel_err(host_f(out2), host_f(out1)) <= TOL[dtype] and rel_err(host_f(ls2), host_f(ls1)) <= TOL["f32"]
    dout = dev(np.ones(inp.x.shape, np.float32), dtype)
    ref = _recomputed_ckpt(t, reverse, dout)
    assert ck.shape == ref.shape
    nck = (L + 3) // 4
    c4 = ck.view(2, nck, 96, 16)
    assert torch.count_nonzero(c4[:, 0]).item() == 0          # chunk 0 enters from zero
    seg = _ckpt_segments(2, L, 96, dtype)
    if seg == 1:
        assert torch.equal(ck, ref)
    else:
        # entering states composed by the carry pass (the chunked scan of the
        # Mamba2 page, sec. 3.2) instead of one long sequential product: fp32
        # rounding apart, checked at the library's fp32 tolerance
        assert rel_err(ck.cpu().numpy(), ref.cpu().numpy()) <= TOL["f32"]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("B,L,D", [(2, 101, 96), (128, 40, 768)])
def test_bwd_ckpt_matches_autograd(dtype, reverse, B, L, D):
    """Every gradient from the checkpoints against the float64 autograd
    oracle.  When the forward's plan has one segment the checkpoints are the
    recompute's bit for bit, so the per-element gradients (dx, ddelta, dz)
    equal the recomputing backward's bit for bit; with segments only dx is
    independent of the states (the adjoint does not read them)."""
    inp = ssm_gen.make_s6_inputs(B, L, D, 16, dtype=dtype, seed=7 + reverse, random_A=True, random_D=True)
    dout = np.random.default_rng(11).standard_normal(inp.x.shape).astype(np.float32)
    if dtype == "bf16":
        dout = ssm_gen.round_to_bf16(dout)
    t = _inputs(inp, dtype)
    dd = dev(dout, dtype)
    kw = dict(delta_bias=t["delta_bias"], D=t["D"], z=t["z"], reverse=reverse)
    _, ck = ssm.ssm_scan_fwd_ckpt(t["x"], t["delta"], t["A"], t["B"], t["C"], **kw)
    g = ssm.ssm_scan_bwd_ckpt(t["x"], t["delta"], t["A"], t["B"], t["C"], dd, ck, **kw)
    g0 = ssm.ssm_scan_bwd(t["x"], t["delta"], t["A"], t["B"], t["C"], dd, **kw)
    torch.cuda.synchronize()
    ref = ograds.s6_grads(inp.x, inp.delta, inp.A_f, inp.B_f, inp.C_f, dout, delta_bias=inp.dt_bias_f,
                          D=inp.D_f, z=inp.z_f, reverse=reverse)
    assert set(g) == set(g0)
    for k, v in g.items():
        e = rel_err(v.cpu().numpy(), ref[NAMES[k]])
        assert e <= TOL[dtype], f"{k}: rel err {e:.3e}"
    seg = _ckpt_segments(B, L, D, dtype)
    for k in (("dx", "ddelta", "dz") if seg == 1 else ("dx",)):
        assert torch.equal(g[k], g0[k]), k


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("L", [77, 2500])
def test_bidir_ckpt_pair_matches_autograd(dtype, L):
    """The bidirectional pair: the forward's output equals bidir_scan_fwd's,
    and the gradients from its two checkpoint arrays match the oracle (one
    segment, and a sequence cut into segments)."""
    inp = ssm_gen.make_s6_inputs(2, L, 96, 16, dtype=dtype, bidir=True, seed=31 + L, random_A=True,
                                 random_D=True)
    dout = np.random.default_rng(5).standard_normal(inp.x.shape).astype(np.float32)
    if dtype == "bf16":
        dout = ssm_gen.round_to_bf16(dout)
    f, b = dir_params(inp, "f"), dir_params(inp, "b")
    x, delta, dd = dev(inp.x, dtype), dev(inp.delta, dtype), dev(dout, dtype)
    out0 = ssm.bidir_scan_fwd(x, delta, f, b)
    out1, ckf, ckb = ssm.bidir_scan_fwd_ckpt(x, delta, f, b)
    dx, ddelta, gf, gb = ssm.bidir_scan_bwd_ckpt(x, delta, f, b, dd, ckf, ckb)
    torch.cuda.synchronize()
    assert torch.equal(out0, out1)
    fw = dict(delta_bias=inp.dt_bias_f, A=inp.A_f, B=inp.B_f, C=inp.C_f, D=inp.D_f, z=inp.z_f)
    bw = dict(delta_bias=inp.dt_bias_b, A=inp.A_b, B=inp.B_b, C=inp.C_b, D=inp.D_b, z=inp.z_b)
    ref = ograds.bidir_grads(inp.x, inp.delta, fw, bw, dout)
    tol = TOL[dtype]
    assert rel_err(dx.cpu().numpy(), ref["x"]) <= tol
    assert rel_err(ddelta.cpu().numpy(), ref["delta"]) <= tol
    for g, side in ((gf, "fwd"), (gb, "bwd")):
        for k, v in g.items():
            e = rel_err(v.cpu().numpy(), ref[side][NAMES[k]])
            assert e <= tol, f"{side} {k}: rel err {e:.3e}"


def test_bidir_ckpt_full_size_workload():
    """Vim-Small (B 64, L 197, D 768, N 16, fp32), the bench's workload: dx,
    ddelta and dz from the checkpoints equal the recomputing backward's bit
    for bit; the parameter gradients (atomic sums) agree to 1e-5."""
    inp = ssm_gen.make_workload(1)
    dout = np.random.default_rng(1).standard_normal(inp.x.shape).astype(np.float32)
    f, b = dir_params(inp, "f"), dir_params(inp, "b")
    x, delta, dd = dev(inp.x, "f32"), dev(inp.delta, "f32"), dev(dout, "f32")
    _, ckf, ckb = ssm.bidir_scan_fwd_ckpt(x, delta, f, b)
    dx1, dd1, gf1, gb1 = ssm.bidir_scan_bwd_ckpt(x, delta, f, b, dd, ckf, ckb)
    dx0, dd0, gf0, gb0 = ssm.bidir_scan_bwd(x, delta, f, b, dd)
    torch.cuda.synchronize()
    assert torch.equal(dx1, dx0) and torch.equal(dd1, dd0)
    for g1, g0 in ((gf1, gf0), (gb1, gb0)):
        assert torch.equal(g1["dz"], g0["dz"])
        for k in ("dA", "dB", "dC", "dD", "ddelta_bias"):
            assert rel_err(g1[k].cpu().numpy(), g0[k].cpu().numpy()) <= 1e-5, k
