"""GPU parity of the exact zero-order-hold scans (ssm_scan_fwd_zoh,
bidir_scan_fwd_zoh; the Mamba2 page, sec. 2.2: Bbar = (dt A)^-1
(exp(dt A) - I) dt B instead of dt B) against the float64 oracle's zoh form.
Both split-state layouts are forced through the library's test hook, and
the one-channel layout's setting is checked to fall back to four threads
per channel.  A holds entries on both sides of the kernel's series /
direct switch (|dt a| = 1/16), exact zeros and small positive values."""
import numpy as np
import pytest
import torch

import oracle
import ssm_gen
import selective_state_space_24_b200 as ssm
from gpu_util import NTHREADS, TOL, dev, f32dev, host, rel_err

pytestmark = pytest.mark.gpu

LAYOUTS = [ssm.MAPPING_AUTO, ssm.MAPPING_SPLIT_STATES, ssm.MAPPING_SPLIT_STATES_2, ssm.MAPPING_WHOLE_CHANNELS]
LAYOUT_IDS = ["auto", "q4", "q2", "whole-falls-back"]


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    ssm.load()


def _inputs(batch, L, D, dtype, seed, bidir=False):
    inp = ssm_gen.make_s6_inputs(batch, L, D, 16, dtype=dtype, bidir=bidir, seed=seed, random_A=True,
                                 random_D=True)
    rng = np.random.default_rng(seed)
    for name in ("A_f", "A_b") if bidir else ("A_f",):
        A = getattr(inp, name).copy()
        A[rng.random(A.shape) < 0.05] = 0.0                       # the a = 0 limit
        A[rng.random(A.shape) < 0.03] = 0.05                      # growing states
        A[:, 0] = -1e-3                                           # deep in the series branch
        setattr(inp, name, A)
    return inp


def _single(inp, reverse, h0, zoh=True):
    x, delta = dev(inp.x, inp.dtype), dev(inp.delta, inp.dtype)
    last = torch.empty((inp.batch, inp.dim, 16), device="cuda")
    fn = ssm.ssm_scan_fwd_zoh if zoh else ssm.ssm_scan_fwd_state
    out = fn(x, delta, f32dev(inp.A_f), dev(inp.B_f, inp.dtype), dev(inp.C_f, inp.dtype),
             delta_bias=f32dev(inp.dt_bias_f), D=f32dev(inp.D_f), z=dev(inp.z_f, inp.dtype), reverse=reverse,
             initial_state=None if h0 is None else f32dev(h0), last_state=last)
    torch.cuda.synchronize()
    return out, last


def _ref_single(inp, reverse, h0):
    return oracle.s6_arrays(inp.x, inp.delta, inp.A_f, inp.B_f, inp.C_f, delta_bias=inp.dt_bias_f, D=inp.D_f,
                            z=inp.z_f, reverse=reverse, initial_state=h0, zoh=True, nthreads=NTHREADS)


@pytest.mark.parametrize("layout", LAYOUTS, ids=LAYOUT_IDS)
@pytest.mark.parametrize("L", [1, 5, 64, 197])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("reverse", [False, True])
def test_single_direction(layout, L, dtype, reverse):
    inp = _inputs(2, L, 40, dtype, seed=300 + L)
    h0 = np.random.default_rng(L).standard_normal((2, 40, 16)).astype(np.float32)
    with ssm.s6_mapping(layout):
        out, last = _single(inp, reverse, h0)
    ref, rst = _ref_single(inp, reverse, h0)
    assert rel_err(host(out), ref) <= TOL[dtype]
    assert rel_err(last.cpu().numpy(), rst) <= TOL[dtype]


def _bidir(inp):
    x, delta = dev(inp.x, inp.dtype), dev(inp.delta, inp.dtype)
    mk = {}
    for s in ("f", "b"):
        mk[s] = ssm.DirParams(A=f32dev(getattr(inp, "A_" + s)), B=dev(getattr(inp, "B_" + s), inp.dtype),
                              C=dev(getattr(inp, "C_" + s), inp.dtype),
                              delta_bias=f32dev(getattr(inp, "dt_bias_" + s)), D=f32dev(getattr(inp, "D_" + s)),
                              z=dev(getattr(inp, "z_" + s), inp.dtype),
                              last_state=torch.empty((inp.batch, inp.dim, 16), device="cuda"))
    out = ssm.bidir_scan_fwd_zoh(x, delta, mk["f"], mk["b"])
    torch.cuda.synchronize()
    return out, mk["f"].last_state, mk["b"].last_state


def _ref_bidir(inp, cols=None):
    f = dict(delta_bias=inp.dt_bias_f, A=inp.A_f, B=inp.B_f, C=inp.C_f, D=inp.D_f, z=inp.z_f)
    b = dict(delta_bias=inp.dt_bias_b, A=inp.A_b, B=inp.B_b, C=inp.C_b, D=inp.D_b, z=inp.z_b)
    return oracle.bidir_arrays(inp.x, inp.delta, f, b, zoh=True, cols=cols, nthreads=NTHREADS)


@pytest.mark.parametrize("layout", LAYOUTS, ids=LAYOUT_IDS)
@pytest.mark.parametrize("L", [1, 6, 9, 197])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_bidirectional(layout, L, dtype):
    inp = _inputs(2, L, 48, dtype, seed=400 + L, bidir=True)
    with ssm.s6_mapping(layout):
        out, lf, lb = _bidir(inp)
    ref, rlf, rlb = _ref_bidir(inp)
    assert rel_err(host(out), ref) <= TOL[dtype]
    assert rel_err(lf.cpu().numpy(), rlf) <= TOL[dtype]
    assert rel_err(lb.cpu().numpy(), rlb) <= TOL[dtype]


def test_vim_small_bidirectional_full_size():
    """Vim-Small bidirectional, fp32, B 64 L 197 D 768 with the exact
    zero-order hold: every output and both last states."""
    inp = ssm_gen.make_workload(1)
    out, lf, lb = _bidir(inp)
    ref, rlf, rlb = _ref_bidir(inp)
    assert rel_err(host(out), ref) <= TOL["f32"]
    assert rel_err(lf.cpu().numpy(), rlf) <= TOL["f32"]
    assert rel_err(lb.cpu().numpy(), rlb) <= TOL["f32"]


def test_differs_from_the_dt_B_scan():
    """The option changes the result by about dt a / 2 relative per term:
    far above the fp32 tolerance for these A and dt, so a call that ignored
    the flag would fail here as well as against the oracle."""
    inp = _inputs(2, 64, 40, "f32", seed=7)
    y_z, _ = _single(inp, False, None)
    y_e, _ = _single(inp, False, None, zoh=False)
    assert rel_err(host(y_e), host(y_z)) > 100 * TOL["f32"]


def test_state_sizes_other_than_16_are_refused():
    inp = ssm_gen.make_s6_inputs(1, 8, 16, 8, dtype="f32", seed=1)
    x, delta = dev(inp.x, "f32"), dev(inp.delta, "f32")
    with pytest.raises(ssm.SSMError, match="UNSUPPORTED_SHAPE"):
        ssm.ssm_scan_fwd_zoh(x, delta, f32dev(inp.A_f), dev(inp.B_f, "f32"), dev(inp.C_f, "f32"))


def test_hires_bidirectional_bf16_full_size():
    """B 8 L 1024 D 768 bf16 with the exact zero-order hold: every output
    and both last states."""
    inp = ssm_gen.make_workload(2)
    out, lf, lb = _bidir(inp)
    ref, rlf, rlb = _ref_bidir(inp)
    assert rel_err(host(out), ref) <= TOL["bf16"]
    assert rel_err(lf.cpu().numpy(), rlf) <= TOL["bf16"]
    assert rel_err(lb.cpu().numpy(), rlb) <= TOL["bf16"]


@pytest.mark.parametrize("layout", [ssm.MAPPING_SPLIT_STATES, ssm.MAPPING_SPLIT_STATES_2], ids=["q4", "q2"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_optional_inputs_absent(layout, dtype):
    """No gate, no skip, no bias, softplus off, in both entry points."""
    inp = _inputs(2, 37, 24, dtype, seed=13, bidir=True)
    delta = np.abs(inp.delta)
    if dtype == "bf16":
        delta = ssm_gen.round_to_bf16(delta)
    x, dl = dev(inp.x, dtype), dev(delta, dtype)
    mk = lambda s: ssm.DirParams(A=f32dev(getattr(inp, "A_" + s)), B=dev(getattr(inp, "B_" + s), dtype),
                                 C=dev(getattr(inp, "C_" + s), dtype))
    with ssm.s6_mapping(layout):
        out = ssm.bidir_scan_fwd_zoh(x, dl, mk("f"), mk("b"), delta_softplus=False)
        one = ssm.ssm_scan_fwd_zoh(x, dl, f32dev(inp.A_f), dev(inp.B_f, dtype), dev(inp.C_f, dtype),
                                   delta_softplus=False, reverse=True)
    torch.cuda.synchronize()
    ref, _, _ = oracle.bidir_arrays(inp.x, delta, dict(A=inp.A_f, B=inp.B_f, C=inp.C_f),
                                    dict(A=inp.A_b, B=inp.B_b, C=inp.C_b), softplus=False, zoh=True)
    ref1, _ = oracle.s6_arrays(inp.x, delta, inp.A_f, inp.B_f, inp.C_f, softplus=False, reverse=True, zoh=True)
    assert rel_err(host(out), ref) <= TOL[dtype]
    assert rel_err(host(one), ref1) <= TOL[dtype]
