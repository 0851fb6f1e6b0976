"""GPU parity of the split-state layouts of the plain S6 scans (s6_split.cu:
four or two threads per channel) against the float64 oracle.  The layout is forced with the
library's test hook, so shapes the cost model would give to the other
layout are covered too: sequence lengths whose last 4-step group is short,
the bidirectional exchange point falling inside a group or on its edge, a
warp only partly inside D, absent optional inputs, initial and last states,
and agreement with the one-or-two-channels-per-thread layout at full
sizes."""
import numpy as np
import pytest
import torch

import oracle
import ssm_gen
import selective_state_space_24_b200 as ssm
from gpu_util import NTHREADS, TOL, dev, f32dev, host, rel_err, run_bidir, run_s6

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    ssm.load()


# every test runs with four and with two threads per channel
@pytest.fixture(autouse=True, params=[ssm.MAPPING_SPLIT_STATES, ssm.MAPPING_SPLIT_STATES_2], ids=["q4", "q2"])
def _split_layout(request):
    with ssm.s6_mapping(request.param):
        yield request.param


@pytest.fixture
def threads(_split_layout):
    return 4 if _split_layout == ssm.MAPPING_SPLIT_STATES else 2


def _plan_is_split(inp, bidir, threads):
    code = ssm.SSM_F32 if inp.dtype == "f32" else ssm.SSM_BF16
    return ssm.scan_plan(inp.batch, inp.seqlen, inp.dim, 16, code, bidirectional=bidir) == (1, -threads)


# L % 4 covers every length of the last group; for the pair, ceil(L / 2) and
# floor(L / 2) put the exchange point at every offset inside a group
@pytest.mark.parametrize("L", [1, 2, 3, 4, 5, 6, 7, 8, 9, 13, 64, 197])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_bidir_every_exchange_offset(L, dtype, threads):
    inp = ssm_gen.make_s6_inputs(2, L, 24, 16, dtype=dtype, bidir=True, seed=100 + L, random_A=True,
                                 random_D=True)
    assert _plan_is_split(inp, True, threads)
    out, lf, lb = run_bidir(inp, last_state=True)
    ref, rlf, rlb = oracle.bidir(inp, nthreads=NTHREADS)
    tol = TOL[dtype]
    assert rel_err(host(out), ref) <= tol
    assert rel_err(lf.cpu().numpy(), rlf) <= tol
    assert rel_err(lb.cpu().numpy(), rlb) <= tol


@pytest.mark.parametrize("L", [1, 3, 4, 5, 31, 197])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("reverse", [False, True])
def test_single_direction_ragged(L, dtype, reverse, threads):
    inp = ssm_gen.make_s6_inputs(3, L, 40, 16, dtype=dtype, seed=200 + L, random_A=True, random_D=True)
    assert _plan_is_split(inp, False, threads)
    out, st = run_s6(inp, reverse=reverse)
    ref, rst = oracle.s6(inp, reverse=reverse, nthreads=NTHREADS)
    tol = TOL[dtype]
    assert rel_err(host(out), ref) <= tol
    assert rel_err(st.cpu().numpy(), rst) <= tol


@pytest.mark.parametrize("bidir", [False, True])
def test_warp_partly_inside_d(bidir):
    """fp32 with D = 12: the last block of channels (8 a warp with four
    threads per channel, 16 with two) reaches past D, so part of its copies
    of x / delta / z are zero-filled and part of its threads idle."""
    inp = ssm_gen.make_s6_inputs(2, 37, 12, 16, dtype="f32", bidir=bidir, seed=7, random_A=True,
                                 random_D=True)
    tol = TOL["f32"]
    if bidir:
        out, lf, lb = run_bidir(inp, last_state=True)
        ref, rlf, rlb = oracle.bidir(inp, nthreads=NTHREADS)
        assert rel_err(lf.cpu().numpy(), rlf) <= tol and rel_err(lb.cpu().numpy(), rlb) <= tol
    else:
        out, st = run_s6(inp, reverse=True)
        ref, rst = oracle.s6(inp, reverse=True, nthreads=NTHREADS)
        assert rel_err(st.cpu().numpy(), rst) <= tol
    assert rel_err(host(out), ref) <= tol


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_optional_inputs_absent(dtype):
    """No gate, no skip, no bias, softplus off (both directions)."""
    inp = ssm_gen.make_s6_inputs(2, 50, 16, 16, dtype=dtype, bidir=True, seed=9, gate=False)
    delta = np.abs(inp.delta)
    x, dl = dev(inp.x, dtype), dev(delta, dtype)
    mk = lambda s: ssm.DirParams(A=f32dev(getattr(inp, "A" + s)), B=dev(getattr(inp, "B" + s), dtype),
                                 C=dev(getattr(inp, "C" + s), dtype))
    out = ssm.bidir_scan_fwd(x, dl, mk("_f"), mk("_b"), delta_softplus=False)
    one = ssm.ssm_scan_fwd(x, dl, f32dev(inp.A_f), dev(inp.B_f, dtype), dev(inp.C_f, dtype),
                           delta_softplus=False)
    torch.cuda.synchronize()
    xr = host(x).astype(np.float64) if dtype == "bf16" else inp.x
    dr = host(dl).astype(np.float64) if dtype == "bf16" else delta
    ref, _, _ = oracle.bidir_arrays(xr, dr, dict(A=inp.A_f, B=inp.B_f, C=inp.C_f),
                                    dict(A=inp.A_b, B=inp.B_b, C=inp.C_b), softplus=False)
    ref1, _ = oracle.s6_arrays(xr, dr, inp.A_f, inp.B_f, inp.C_f, softplus=False)
    assert rel_err(host(out), ref) <= TOL[dtype]
    assert rel_err(host(one), ref1) <= TOL[dtype]


@pytest.mark.parametrize("reverse", [False, True])
def test_initial_state_and_chained_pieces(reverse):
    """A scan from a given state, and a sequence scanned as three pieces with
    the state handed on in place, both against one oracle scan."""
    Bsz, L, D = 2, 90, 32
    inp = ssm_gen.make_s6_inputs(Bsz, L, D, 16, dtype="f32", seed=11 + reverse, random_A=True, random_D=True)
    h0 = np.random.default_rng(3).standard_normal((Bsz, D, 16)).astype(np.float32)
    A, B, C = f32dev(inp.A_f), dev(inp.B_f, "f32"), dev(inp.C_f, "f32")
    kw = dict(delta_bias=f32dev(inp.dt_bias_f), D=f32dev(inp.D_f), reverse=reverse)
    x, delta, z = dev(inp.x, "f32"), dev(inp.delta, "f32"), dev(inp.z_f, "f32")
    last = torch.empty((Bsz, D, 16), device="cuda")
    out = ssm.ssm_scan_fwd_state(x, delta, A, B, C, z=z, initial_state=f32dev(h0), last_state=last, **kw)
    torch.cuda.synchronize()
    ref, rst = oracle.s6_arrays(inp.x, inp.delta, inp.A_f, inp.B_f, inp.C_f, delta_bias=inp.dt_bias_f,
                                D=inp.D_f, z=inp.z_f, reverse=reverse, initial_state=h0)
    assert rel_err(host(out), ref) <= TOL["f32"] and rel_err(last.cpu().numpy(), rst) <= TOL["f32"]
    # three pieces in scan order, the state carried in place
    state = f32dev(h0)
    pieces = [slice(0, 37), slice(37, 38), slice(38, L)]
    out2 = torch.empty_like(out)
    for sl in (reversed(pieces) if reverse else pieces):
        o = ssm.ssm_scan_fwd_state(x[:, sl].contiguous(), delta[:, sl].contiguous(), A, B[:, sl].contiguous(),
                                   C[:, sl].contiguous(), z=z[:, sl].contiguous(), initial_state=state,
                                   last_state=state, **kw)
        out2[:, sl] = o
    torch.cuda.synchronize()
    assert rel_err(host(out2), ref) <= TOL["f32"] and rel_err(state.cpu().numpy(), rst) <= TOL["f32"]


@pytest.mark.parametrize("dtype,bidir,batch,L,D", [("f32", True, 64, 197, 768), ("bf16", True, 8, 1024, 768),
                                                   ("f32", False, 16, 197, 768), ("bf16", False, 4, 300, 1536)])
def test_layouts_agree_at_full_size(dtype, bidir, batch, L, D):
    """Every output of the two layouts on the same inputs (the cost model
    picks either for such sizes), and sampled columns against the oracle."""
    inp = ssm_gen.make_s6_inputs(batch, L, D, 16, dtype=dtype, bidir=bidir, seed=batch + L)
    run = (lambda: run_bidir(inp, last_state=True)) if bidir else (lambda: run_s6(inp))
    split = run()
    with ssm.s6_mapping(ssm.MAPPING_WHOLE_CHANNELS):
        whole = run()
    tol = TOL[dtype]
    for a, b in zip(split, whole):
        assert rel_err(host(a), host(b)) <= tol
    cols = np.random.default_rng(0).choice(batch * D, 24, replace=False)
    bb, dd = np.divmod(cols, D)
    ref = (oracle.bidir(inp, cols=cols, nthreads=NTHREADS) if bidir
           else oracle.s6(inp, cols=cols, nthreads=NTHREADS))[0]
    assert rel_err(host(split[0])[bb, :, dd], ref[bb, :, dd]) <= tol


@pytest.mark.parametrize("batch,L,D", [(4, 120, 256), (100, 40, 768)])   # the second mixes rows
def test_noalloc_takes_the_same_layout(batch, L, D):
    """ssm_scan_fwd_noalloc takes the layout ssm_scan_fwd takes: bit for bit."""
    inp = ssm_gen.make_s6_inputs(batch, L, D, 16, dtype="f32", seed=5, random_A=True, random_D=True)
    x, delta = dev(inp.x, "f32"), dev(inp.delta, "f32")
    A, B, C = f32dev(inp.A_f), dev(inp.B_f, "f32"), dev(inp.C_f, "f32")
    kw = dict(delta_bias=f32dev(inp.dt_bias_f), D=f32dev(inp.D_f), z=dev(inp.z_f, "f32"))
    ref = ssm.ssm_scan_fwd(x, delta, A, B, C, **kw)
    out = ssm.ssm_scan_fwd_noalloc(x, delta, A, B, C, **kw)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


@pytest.mark.parametrize("dtype,bidir,batch,L,D", [("f32", True, 64, 60, 768), ("bf16", True, 62, 33, 768),
                                                   ("f32", False, 13, 57, 768), ("bf16", False, 26, 41, 384)])
def test_mixed_rows_in_one_launch(dtype, bidir, batch, L, D, threads):
    """With two threads per channel, sizes whose warps overfill the last
    round of the SM sub-partitions run their trailing batch rows with four
    threads per channel in the same launch; every output and last state
    against the oracle (under the four-thread setting these sizes run
    unmixed)."""
    inp = ssm_gen.make_s6_inputs(batch, L, D, 16, dtype=dtype, bidir=bidir, seed=batch + L, random_A=True,
                                 random_D=True)
    tol = TOL[dtype]
    if bidir:
        out, lf, lb = run_bidir(inp, last_state=True)
        ref, rlf, rlb = oracle.bidir(inp, nthreads=NTHREADS)
        assert rel_err(lf.cpu().numpy(), rlf) <= tol and rel_err(lb.cpu().numpy(), rlb) <= tol
    else:
        out, st = run_s6(inp, reverse=True)
        ref, rst = oracle.s6(inp, reverse=True, nthreads=NTHREADS)
        assert rel_err(st.cpu().numpy(), rst) <= tol
    assert rel_err(host(out), ref) <= tol
