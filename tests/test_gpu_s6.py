"""GPU parity of the S6 and bidirectional scans against the float64 oracle,
through the C ABI (libssm.so), on seeded inputs from ssm_gen."""
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


def _check_s6(inp, reverse):
    out, st = run_s6(inp, reverse=reverse)
    ref, rst = oracle.s6(inp, reverse=reverse, nthreads=NTHREADS)
    e = rel_err(host(out), ref)
    es = rel_err(st.cpu().numpy(), rst)
    tol = TOL[inp.dtype]
    assert e <= tol, f"out rel err {e:.3e}"
    assert es <= tol, f"last_state rel err {es:.3e}"
    return e


def _check_bidir(inp, last_state=False, cols=None):
    out, lf, lb = run_bidir(inp, last_state=last_state)
    ref, rlf, rlb = oracle.bidir(inp, cols=cols, nthreads=NTHREADS)
    g = host(out)
    tol = TOL[inp.dtype]
    if cols is None:
        e = rel_err(g, ref)
    else:
        b, d = np.divmod(np.asarray(cols), inp.dim)
        e = rel_err(g[b, :, d], ref[b, :, d])
    assert e <= tol, f"out rel err {e:.3e}"
    if last_state:
        if cols is None:
            es = max(rel_err(lf.cpu().numpy(), rlf), rel_err(lb.cpu().numpy(), rlb))
        else:
            es = max(rel_err(lf.cpu().numpy()[b, d], rlf[b, d]),
                     rel_err(lb.cpu().numpy()[b, d], rlb[b, d]))
        assert es <= tol, f"last_state rel err {es:.3e}"
    return e


# ------------------------------------------------------- the workloads' shapes

@pytest.mark.parametrize("reverse", [False, True])
def test_vim_tiny_single_direction_full(reverse):
    """Vim-Tiny S6, fp32: batch 1, L 196, d_inner 384, N 16 -- every output."""
    inp = ssm_gen.make_workload(0)
    _check_s6(inp, reverse)


def test_vim_small_bidir_reduced_batch_full_compare():
    inp = ssm_gen.make_s6_inputs(2, 197, 768, 16, dtype="f32", bidir=True, seed=0)
    _check_bidir(inp, last_state=True)


def test_vim_small_bidir_full_size():
    """Vim-Small bidirectional, fp32, B 64 L 197 D 768 -- the bench's launch;
    every output and both last states against the oracle."""
    inp = ssm_gen.make_workload(1)
    _check_bidir(inp, last_state=True)


def test_hires_bidir_bf16_reduced_full_compare():
    inp = ssm_gen.make_s6_inputs(1, 1024, 768, 16, dtype="bf16", bidir=True, seed=0)
    _check_bidir(inp, last_state=True)


def test_hires_bidir_bf16_full_size():
    """B 8 L 1024 D 768 bf16 with last_state per direction; every output."""
    inp = ssm_gen.make_workload(2)
    _check_bidir(inp, last_state=True)


def test_long_row_bidir_bf16_full_size():
    """Mamba-YOLO stage-1 rows: B 4 L 16384 D 192 bf16; every output."""
    inp = ssm_gen.make_workload(3)
    _check_bidir(inp, last_state=True)


# ------------------------------------------------- both lane mappings

@pytest.mark.parametrize("batch,L,D,bidir,dtype,cpl", [
    (32, 300, 768, True, "f32", 2),    # two channels per lane, two segments
    (64, 100, 768, False, "f32", 2),   # single direction, two per lane, two segments
    (2, 300, 96, True, "bf16", 1),     # one per lane, 16-step segments, 3 warps of channels
    (3, 500, 40, False, "f32", 1),     # one per lane, a warp only partly inside D
])
def test_lane_mappings(batch, L, D, bidir, dtype, cpl):
    """Both thread layouts (one or two channels per lane), with and without
    segments, against the oracle on sampled columns (reversed for the
    single-direction cases)."""
    code = ssm.SSM_F32 if dtype == "f32" else ssm.SSM_BF16
    with ssm.s6_mapping(ssm.MAPPING_WHOLE_CHANNELS):
        _lane_mapping_case(batch, L, D, bidir, dtype, cpl, code)


def _lane_mapping_case(batch, L, D, bidir, dtype, cpl, code):
    seg, got = ssm.scan_plan(batch, L, D, 16, code, bidirectional=bidir)
    assert got == cpl and seg > 1
    inp = ssm_gen.make_s6_inputs(batch, L, D, 16, dtype=dtype, bidir=bidir, seed=L + D,
                                 random_A=True, random_D=True)
    rng = np.random.default_rng(L)
    cols = rng.choice(batch * D, min(48, batch * D), replace=False)
    b, d = np.divmod(cols, D)
    tol = TOL[dtype]
    if bidir:
        out, lf, lb = run_bidir(inp, last_state=True)
        ref, rlf, rlb = oracle.bidir(inp, cols=cols, nthreads=NTHREADS)
        assert rel_err(host(out)[b, :, d], ref[b, :, d]) <= tol
        assert rel_err(lf.cpu().numpy()[b, d], rlf[b, d]) <= tol
        assert rel_err(lb.cpu().numpy()[b, d], rlb[b, d]) <= tol
    else:
        out, st = run_s6(inp, reverse=True)
        ref, rst = oracle.s6(inp, reverse=True, cols=cols, nthreads=NTHREADS)
        assert rel_err(host(out)[b, :, d], ref[b, :, d]) <= tol
        assert rel_err(st.cpu().numpy()[b, d], rst[b, d]) <= tol


# ------------------------------------------------------------ ragged / edges

@pytest.mark.parametrize("L", [1, 2, 3, 17, 255, 256, 257, 1000, 4099])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_bidir_ragged_lengths(L, dtype):
    inp = ssm_gen.make_s6_inputs(2, L, 72, 16, dtype=dtype, bidir=True, seed=L,
                                 random_A=True, random_D=True)
    _check_bidir(inp, last_state=True)


@pytest.mark.parametrize("N", [1, 2, 4, 7, 8, 13, 16])
def test_state_sizes(N):
    inp = ssm_gen.make_s6_inputs(3, 50, 40, N, dtype="f32", bidir=True, seed=N, random_A=True)
    _check_bidir(inp, last_state=True)
    _check_s6(inp, reverse=False)
    _check_s6(inp, reverse=True)


@pytest.mark.parametrize("L", [1, 33, 600, 3000])
@pytest.mark.parametrize("reverse", [False, True])
def test_single_direction_ragged(L, reverse):
    inp = ssm_gen.make_s6_inputs(2, L, 24, 16, dtype="bf16", seed=100 + L, random_A=True,
                                 random_D=True)
    _check_s6(inp, reverse)


def test_parameter_swap_guard():
    """Directions with visibly different A and D: swapping them fails."""
    inp = ssm_gen.make_s6_inputs(2, 64, 64, 16, dtype="f32", bidir=True, seed=9,
                                 random_A=True, random_D=True)
    out, _, _ = run_bidir(inp)
    ref, _, _ = oracle.bidir(inp)
    assert rel_err(host(out), ref) <= TOL["f32"]
    swapped = ssm_gen.make_s6_inputs(2, 64, 64, 16, dtype="f32", bidir=True, seed=9,
                                     random_A=True, random_D=True)
    swapped.A_f, swapped.A_b = swapped.A_b, swapped.A_f
    sref, _, _ = oracle.bidir(swapped)
    assert rel_err(sref, ref) > 100 * TOL["f32"]


def test_optional_inputs_absent():
    """No gate, no skip, no bias, softplus off."""
    inp = ssm_gen.make_s6_inputs(2, 40, 32, 16, dtype="f32", bidir=True, seed=10, gate=False)
    x, delta = dev(inp.x, "f32"), dev(np.abs(inp.delta), "f32")
    mk = lambda s: ssm.DirParams(A=f32dev(getattr(inp, "A" + s)), B=dev(getattr(inp, "B" + s), "f32"),
                                 C=dev(getattr(inp, "C" + s), "f32"))
    out = ssm.bidir_scan_fwd(x, delta, mk("_f"), mk("_b"), delta_softplus=False)
    ref, _, _ = oracle.bidir_arrays(inp.x, np.abs(inp.delta),
                                    dict(A=inp.A_f, B=inp.B_f, C=inp.C_f),
                                    dict(A=inp.A_b, B=inp.B_b, C=inp.C_b), softplus=False)
    assert rel_err(host(out), ref) <= TOL["f32"]


def test_deterministic_bitwise():
    inp = ssm_gen.make_s6_inputs(4, 300, 128, 16, dtype="bf16", bidir=True, seed=11)
    a, _, _ = run_bidir(inp)
    b, _, _ = run_bidir(inp)
    assert torch.equal(a, b)
    inp3 = ssm_gen.make_workload(3, batch=1)
    a, _, _ = run_bidir(inp3)
    b, _, _ = run_bidir(inp3)
    assert torch.equal(a, b)


def test_empty_sequence_zeroes_last_state():
    inp = ssm_gen.make_s6_inputs(2, 1, 16, 16, dtype="f32", bidir=True, seed=12)
    x = torch.empty((2, 0, 16), device="cuda")
    f = ssm.DirParams(A=f32dev(inp.A_f), B=torch.empty((2, 0, 16), device="cuda"),
                      C=torch.empty((2, 0, 16), device="cuda"),
                      last_state=torch.full((2, 16, 16), 7.0, device="cuda"))
    out = ssm.bidir_scan_fwd(x, x, f, f)
    torch.cuda.synchronize()
    assert out.shape == (2, 0, 16)
    assert torch.count_nonzero(f.last_state).item() == 0


def test_no_device_timeout_flagged():
    inp = ssm_gen.make_s6_inputs(1, 20, 16, 16, bidir=True, seed=13)
    run_bidir(inp)
    ssm.check_device()
