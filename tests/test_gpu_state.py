"""GPU parity of the scan from a given initial state (ssm_scan_fwd_state)
and of the one-step decode kernel (ssm_step) against the float64 oracle,
through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import ssm_gen
import selective_state_space_24_b200 as ssm
from gpu_util import TOL, dev, f32dev, host, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    ssm.load()


def _params(inp, dtype):
    return dict(A=f32dev(inp.A_f), B=dev(inp.B_f, dtype), C=dev(inp.C_f, dtype),
                delta_bias=f32dev(inp.dt_bias_f), D=f32dev(inp.D_f), z=dev(inp.z_f, dtype))


def _oracle_scan(inp, h0, reverse, cols=None, sl=slice(None)):
    return oracle.s6_arrays(inp.x[:, sl], inp.delta[:, sl], inp.A_f, inp.B_f[:, sl], inp.C_f[:, sl],
                            delta_bias=inp.dt_bias_f, D=inp.D_f, z=inp.z_f[:, sl], reverse=reverse,
                            initial_state=h0, cols=cols, nthreads=8)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("batch,L,D", [(2, 150, 64), (1, 3000, 32)])   # one segment; many segments
def test_scan_from_initial_state(dtype, reverse, batch, L, D):
    inp = ssm_gen.make_s6_inputs(batch, L, D, 16, dtype=dtype, seed=L + reverse, random_A=True,
                                 random_D=True)
    h0 = np.random.default_rng(L).standard_normal((batch, D, 16)).astype(np.float32)
    p = _params(inp, dtype)
    last = torch.empty((batch, D, 16), device="cuda")
    out = ssm.ssm_scan_fwd_state(dev(inp.x, dtype), dev(inp.delta, dtype), p["A"], p["B"], p["C"],
                                 initial_state=f32dev(h0), delta_bias=p["delta_bias"], D=p["D"],
                                 z=p["z"], reverse=reverse, last_state=last)
    torch.cuda.synchronize()
    ref, rst = _oracle_scan(inp, h0, reverse)
    assert rel_err(host(out), ref) <= TOL[dtype]
    assert rel_err(last.cpu().numpy(), rst) <= TOL[dtype]


@pytest.mark.parametrize("reverse", [False, True])
def test_pieces_chain_in_place(reverse):
    """A sequence run in pieces on the GPU, the state carried in one tensor
    updated in place (initial_state is last_state), equals the oracle's
    single run."""
    batch, L, D = 2, 700, 64
    inp = ssm_gen.make_s6_inputs(batch, L, D, 16, dtype="f32", seed=41 + reverse, random_A=True)
    p = _params(inp, "f32")
    x, delta = dev(inp.x, "f32"), dev(inp.delta, "f32")
    state = torch.zeros((batch, D, 16), device="cuda")
    out = torch.empty_like(x)
    cuts = [0, 1, 17, 300, 301, L]
    pieces = list(zip(cuts[:-1], cuts[1:]))
    if reverse:
        pieces = pieces[::-1]
    for a, e in pieces:
        sl = slice(a, e)
        o = ssm.ssm_scan_fwd_state(x[:, sl].contiguous(), delta[:, sl].contiguous(), p["A"],
                                   p["B"][:, sl].contiguous(), p["C"][:, sl].contiguous(),
                                   initial_state=state, delta_bias=p["delta_bias"], D=p["D"],
                                   z=p["z"][:, sl].contiguous(), reverse=reverse, last_state=state)
        out[:, sl] = o
    torch.cuda.synchronize()
    ref, rst = _oracle_scan(inp, None, reverse)
    assert rel_err(host(out), ref) <= TOL["f32"]
    assert rel_err(state.cpu().numpy(), rst) <= TOL["f32"]


def test_empty_sequence_keeps_initial_state():
    inp = ssm_gen.make_s6_inputs(2, 4, 32, 16, dtype="f32", seed=3)
    p = _params(inp, "f32")
    h0 = torch.randn((2, 32, 16), device="cuda")
    last = torch.zeros_like(h0)
    x = torch.empty((2, 0, 32), device="cuda")
    ssm.ssm_scan_fwd_state(x, x.clone(), p["A"], p["B"][:, :0].contiguous(), p["C"][:, :0].contiguous(),
                           initial_state=h0, last_state=last)
    torch.cuda.synchronize()
    assert torch.equal(last, h0)


@pytest.mark.parametrize("dtype,N,batch,D", [("f32", 4, 3, 96), ("f32", 7, 3, 96), ("f32", 16, 3, 96),
                                              ("bf16", 4, 3, 96), ("bf16", 7, 3, 96), ("bf16", 16, 3, 96),
                                              ("bf16", 8, 5, 200), ("f32", 16, 512, 1536),
                                              ("bf16", 16, 512, 1536), ("f32", 16, 700, 136),
                                              ("bf16", 16, 3, 8)])
def test_step_matches_oracle(dtype, N, batch, D):
    """One decode step against the oracle; (512, 1536) is the bench's decode
    workload (several 128-row tiles per CTA of the N = 16 kernel), every row
    compared; (700, 136) gives some CTAs a second tile and a 96-row last
    tile; (3, 8) bf16 a single 24-row tile."""
    inp = ssm_gen.make_s6_inputs(batch, 1, D, N, dtype=dtype, seed=N, random_A=True, random_D=True)
    state0 = np.random.default_rng(N).standard_normal((batch, D, N)).astype(np.float32)
    p = _params(inp, dtype)
    state = f32dev(state0)
    y = ssm.ssm_step(dev(inp.x[:, 0], dtype), dev(inp.delta[:, 0], dtype), p["A"],
                     p["B"][:, 0].contiguous(), p["C"][:, 0].contiguous(), state,
                     delta_bias=p["delta_bias"], D=p["D"], z=p["z"][:, 0].contiguous())
    torch.cuda.synchronize()
    ry, rst = oracle.step_arrays(inp.x[:, 0], inp.delta[:, 0], inp.A_f, inp.B_f[:, 0], inp.C_f[:, 0],
                                 state0, delta_bias=inp.dt_bias_f, D=inp.D_f, z=inp.z_f[:, 0])
    assert rel_err(host(y), ry) <= TOL[dtype]
    assert rel_err(state.cpu().numpy(), rst) <= TOL[dtype]


def test_decode_loop_equals_scan():
    """L decode steps from a zero state reproduce the L-step scan (outputs
    and final state), checked against the oracle."""
    batch, L, D = 2, 40, 64
    inp = ssm_gen.make_s6_inputs(batch, L, D, 16, dtype="f32", seed=77, random_A=True)
    p = _params(inp, "f32")
    x, delta = dev(inp.x, "f32"), dev(inp.delta, "f32")
    state = torch.zeros((batch, D, 16), device="cuda")
    ys = []
    for t in range(L):
        ys.append(ssm.ssm_step(x[:, t].contiguous(), delta[:, t].contiguous(), p["A"],
                               p["B"][:, t].contiguous(), p["C"][:, t].contiguous(), state,
                               delta_bias=p["delta_bias"], D=p["D"], z=p["z"][:, t].contiguous()))
    torch.cuda.synchronize()
    ref, rst = _oracle_scan(inp, None, False)
    assert rel_err(torch.stack(ys, 1).cpu().numpy(), ref) <= TOL["f32"]
    assert rel_err(state.cpu().numpy(), rst) <= TOL["f32"]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_step_optional_inputs_absent(dtype):
    """N = 16 decode step with no gate, skip or bias and softplus off."""
    batch, D = 40, 64
    inp = ssm_gen.make_s6_inputs(batch, 1, D, 16, dtype=dtype, seed=5, random_A=True)
    delta = np.abs(inp.delta[:, 0])
    state0 = np.random.default_rng(6).standard_normal((batch, D, 16)).astype(np.float32)
    state = f32dev(state0)
    y = ssm.ssm_step(dev(inp.x[:, 0], dtype), dev(delta, dtype), f32dev(inp.A_f),
                     dev(inp.B_f[:, 0], dtype), dev(inp.C_f[:, 0], dtype), state, delta_softplus=False)
    torch.cuda.synchronize()
    ry, rst = oracle.step_arrays(inp.x[:, 0], delta, inp.A_f, inp.B_f[:, 0], inp.C_f[:, 0], state0,
                                 softplus=False)
    assert rel_err(host(y), ry) <= TOL[dtype]
    assert rel_err(state.cpu().numpy(), rst) <= TOL[dtype]
    ssm.check_device()   # no device-side error word set
