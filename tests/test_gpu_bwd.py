"""GPU parity of the S6 backward pass (ssm_scan_bwd) against the float64
autograd oracle (oracle/grads.py), through the C ABI."""
import numpy as np
import pytest
import torch

import ssm_gen
import selective_state_space_24_b200 as ssm
from oracle import grads as ograds
from gpu_util import TOL, dev, f32dev, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    ssm.load()


def _run(inp, dtype, dout, reverse, gate=True, D=True, bias=True, softplus=True):
    g = ssm.ssm_scan_bwd(dev(inp.x, dtype), dev(inp.delta, dtype), f32dev(inp.A_f), dev(inp.B_f, dtype),
                         dev(inp.C_f, dtype), dev(dout, dtype),
                         delta_bias=f32dev(inp.dt_bias_f) if bias else None, delta_softplus=softplus,
                         D=f32dev(inp.D_f) if D else None, z=dev(inp.z_f, dtype) if gate else None,
                         reverse=reverse)
    torch.cuda.synchronize()
    ref = ograds.s6_grads(inp.x, inp.delta, inp.A_f, inp.B_f, inp.C_f, dout,
                          delta_bias=inp.dt_bias_f if bias else None, softplus=softplus,
                          D=inp.D_f if D else None, z=inp.z_f if gate else None, reverse=reverse)
    return g, ref


def _check(g, ref, tol):
    names = {"dx": "x", "ddelta": "delta", "dA": "A", "dB": "B", "dC": "C", "dD": "D", "dz": "z",
             "ddelta_bias": "delta_bias"}
    for k, t in g.items():
        e = rel_err(t.cpu().numpy(), ref[names[k]])
        assert e <= tol, f"{k}: rel err {e:.3e}"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("N", [16, 5, 8, 3])
def test_bwd_matches_autograd(dtype, reverse, N):
    """Every gradient; L = 101 leaves a ragged last 4-step chunk and 16-step
    input stage, D = 96 leaves a CTA of 64 channels half full; N covers the
    three padded state counts (4, 8, 16)."""
    inp = ssm_gen.make_s6_inputs(2, 101, 96, N, dtype=dtype, seed=N + reverse, random_A=True,
                                 random_D=True)
    dout = np.random.default_rng(N).standard_normal(inp.x.shape).astype(np.float32)
    if dtype == "bf16":
        dout = ssm_gen.round_to_bf16(dout)
    g, ref = _run(inp, dtype, dout, reverse)
    _check(g, ref, TOL[dtype])


@pytest.mark.parametrize("gate,D,bias,softplus", [(False, True, True, True), (True, False, False, True),
                                                  (True, True, False, False)])
def test_bwd_optional_inputs(gate, D, bias, softplus):
    inp = ssm_gen.make_s6_inputs(1, 64, 32, 16, dtype="f32", seed=3, random_A=True, random_D=True)
    if not softplus:   # keep dt positive without the softplus
        inp.delta = np.abs(inp.delta) * 0.1
    dout = np.random.default_rng(4).standard_normal(inp.x.shape).astype(np.float32)
    g, ref = _run(inp, "f32", dout, False, gate=gate, D=D, bias=bias, softplus=softplus)
    assert ("dz" in g) == gate and ("dD" in g) == D and ("ddelta_bias" in g) == bias
    _check(g, ref, TOL["f32"])


@pytest.mark.parametrize("L", [1, 4, 15, 16, 17, 33])
def test_bwd_short_sequences(L):
    """Sequences of one step, one chunk, one input stage and just past
    stage boundaries."""
    inp = ssm_gen.make_s6_inputs(2, L, 64, 16, dtype="f32", seed=40 + L, random_A=True, random_D=True)
    dout = np.random.default_rng(L).standard_normal(inp.x.shape).astype(np.float32)
    g, ref = _run(inp, "f32", dout, L % 2 == 1)
    _check(g, ref, TOL["f32"])


def test_bwd_long_sequence():
    """A longer sequence (many checkpointed chunks), sampled against the
    oracle on one batch row."""
    inp = ssm_gen.make_s6_inputs(1, 1000, 64, 16, dtype="f32", seed=8, random_A=True, random_D=True)
    dout = np.random.default_rng(9).standard_normal(inp.x.shape).astype(np.float32)
    g, ref = _run(inp, "f32", dout, False)
    _check(g, ref, TOL["f32"])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_bidir_bwd_matches_autograd(dtype):
    """Gradients of the bidirectional scan: dx and ddelta sum both
    directions, each direction's parameter gradients separately."""
    from gpu_util import dir_params
    inp = ssm_gen.make_s6_inputs(2, 77, 96, 16, dtype=dtype, bidir=True, seed=31, random_A=True,
                                 random_D=True)
    dout = np.random.default_rng(5).standard_normal(inp.x.shape).astype(np.float32)
    if dtype == "bf16":
        dout = ssm_gen.round_to_bf16(dout)
    f, b = dir_params(inp, "f"), dir_params(inp, "b")
    dx, ddelta, gf, gb = ssm.bidir_scan_bwd(dev(inp.x, dtype), dev(inp.delta, dtype), f, b, dev(dout, dtype))
    torch.cuda.synchronize()
    fw = dict(delta_bias=inp.dt_bias_f, A=inp.A_f, B=inp.B_f, C=inp.C_f, D=inp.D_f, z=inp.z_f)
    bw = dict(delta_bias=inp.dt_bias_b, A=inp.A_b, B=inp.B_b, C=inp.C_b, D=inp.D_b, z=inp.z_b)
    ref = ograds.bidir_grads(inp.x, inp.delta, fw, bw, dout)
    tol = TOL[dtype]
    assert rel_err(dx.cpu().numpy(), ref["x"]) <= tol
    assert rel_err(ddelta.cpu().numpy(), ref["delta"]) <= tol
    names = {"dA": "A", "dB": "B", "dC": "C", "dD": "D", "dz": "z", "ddelta_bias": "delta_bias"}
    for g, side in ((gf, "fwd"), (gb, "bwd")):
        for k, t in g.items():
            e = rel_err(t.cpu().numpy(), ref[side][names[k]])
            assert e <= tol, f"{side} {k}: rel err {e:.3e}"


@pytest.mark.parametrize("layout", [ssm.MAPPING_WHOLE_CHANNELS, ssm.MAPPING_SPLIT_STATES, ssm.MAPPING_SPLIT_STATES_2],
                         ids=["whole", "q4", "q2"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("reverse", [False, True])
def test_bwd_checkpoint_pass_in_every_layout(layout, dtype, reverse):
    """The plain backward's recompute pass runs on the forward layout the
    plan gives the sizes (here forced): the split-state kernel without
    outputs with two or four threads per channel, or the one-thread-per-
    channel checkpoint kernel (which mode also selects the one-thread
    backward sweep).  L = 70 leaves a short last chunk; D = 40 leaves warps
    partly past D in every layout."""
    inp = ssm_gen.make_s6_inputs(3, 70, 40, 16, dtype=dtype, seed=60 + reverse, random_A=True, random_D=True)
    dout = np.random.default_rng(61).standard_normal(inp.x.shape).astype(np.float32)
    if dtype == "bf16":
        dout = ssm_gen.round_to_bf16(dout)
    with ssm.s6_mapping(layout):
        g, ref = _run(inp, dtype, dout, reverse)
    _check(g, ref, TOL[dtype])
