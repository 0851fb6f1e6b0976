"""GPU parity of the Mamba2 SSD chunked scan (tcgen05 path) against the
float64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import ssm_gen
import selective_state_space_24_b200 as ssm
from gpu_util import NTHREADS, TOL, dev, f32dev, host, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    ssm.load()


def run_ssd(inp, last_state=True, gate=True, D=True, bias=True):
    x = dev(inp.x, "bf16")
    delta = dev(inp.delta, "bf16")
    ls = None
    if last_state:
        ls = torch.full((inp.batch, inp.nheads, inp.headdim, inp.dstate), 7.0, device="cuda")
    out = ssm.ssd_chunk_fwd(x, delta, f32dev(inp.A), dev(inp.B, "bf16"), dev(inp.C, "bf16"),
                            chunk=inp.chunk, delta_bias=f32dev(inp.dt_bias) if bias else None,
                            D=f32dev(inp.D) if D else None,
                            z=dev(inp.z, "bf16") if gate else None, last_state=ls)
    torch.cuda.synchronize()
    ssm.check_device()
    return out, ls


def _ref(inp, cols=None, gate=True, D=True, bias=True):
    return oracle.ssd_seq_arrays(inp.x, inp.delta, inp.A, inp.B, inp.C,
                                 delta_bias=inp.dt_bias if bias else None, softplus=True,
                                 D=inp.D if D else None, z=inp.z if gate else None, cols=cols,
                                 nthreads=NTHREADS)


@pytest.mark.parametrize("L", [1, 63, 64, 65, 200, 333])
def test_ssd_small_full_compare(L):
    inp = ssm_gen.make_ssd_inputs(2, L, 3, 64, 128, 64, dtype="bf16", seed=L, random_D=True)
    out, ls = run_ssd(inp)
    ref, rls = _ref(inp)
    e = rel_err(host(out), ref)
    es = rel_err(ls.cpu().numpy(), rls)
    assert e <= TOL["bf16"], f"out rel err {e:.3e}"
    assert es <= TOL["bf16"], f"last_state rel err {es:.3e}"


def test_ssd_matches_chunked_oracle_form():
    inp = ssm_gen.make_ssd_inputs(1, 256, 2, 64, 128, 64, dtype="bf16", seed=5)
    out, _ = run_ssd(inp, last_state=False)
    refc, _ = oracle.ssd_chunked(inp, chunk=64, nthreads=NTHREADS)
    assert rel_err(host(out), refc) <= TOL["bf16"]


@pytest.mark.parametrize("gate,D,bias", [(False, True, True), (True, False, True), (True, True, False)])
def test_ssd_optional_inputs(gate, D, bias):
    inp = ssm_gen.make_ssd_inputs(1, 150, 2, 64, 128, 64, dtype="bf16", seed=9, random_D=True)
    out, ls = run_ssd(inp, gate=gate, D=D, bias=bias)
    ref, rls = _ref(inp, gate=gate, D=D, bias=bias)
    assert rel_err(host(out), ref) <= TOL["bf16"]
    assert rel_err(ls.cpu().numpy(), rls) <= TOL["bf16"]


def test_ssd_full_size():
    """Mamba2 SSD workload: B 4, L 8192, 32 heads x 64, N 128, chunk 64;
    every output and the whole last state against the sequential oracle."""
    inp = ssm_gen.make_workload(4)
    out, ls = run_ssd(inp)
    ref, rls = _ref(inp)
    assert rel_err(host(out), ref) <= TOL["bf16"]
    assert rel_err(ls.cpu().numpy(), rls) <= TOL["bf16"]


def test_ssd_deterministic():
    inp = ssm_gen.make_ssd_inputs(2, 512, 4, 64, 128, 64, dtype="bf16", seed=11)
    a, _ = run_ssd(inp)
    b, _ = run_ssd(inp)
    assert torch.equal(a, b)


def test_ssd_unsupported_shape_rejected():
    inp = ssm_gen.make_ssd_inputs(1, 64, 2, 32, 128, 64, dtype="bf16", seed=1)
    with pytest.raises(ssm.SSMError):
        ssm.ssd_chunk_fwd(dev(inp.x, "bf16"), dev(inp.delta, "bf16"), f32dev(inp.A),
                          dev(inp.B, "bf16"), dev(inp.C, "bf16"))


def test_ssd_device_timeout_is_reported_and_the_next_call_is_clean():
    """A bounded device wait that runs out: the producer warp withholds its
    dt signal for chunk 2 (a signal nothing else gives), with every wait
    limited to 4096 polls.  The call still completes -- it waits for the
    copies and MMAs it issued and frees its tensor memory -- and
    ssm_check_device reports SSM_ERR_DEVICE_TIMEOUT.  The error word is then
    clear, and a normal call on the same context is correct."""
    lib = ssm.capi()
    inp = ssm_gen.make_ssd_inputs(2, 320, 3, 64, 128, 64, dtype="bf16", seed=31)
    lib.ssm_debug_ssd_stall(2, 1 << 12)
    try:
        x = dev(inp.x, "bf16")
        ssm.ssd_chunk_fwd(x, dev(inp.delta, "bf16"), f32dev(inp.A), dev(inp.B, "bf16"), dev(inp.C, "bf16"),
                          delta_bias=f32dev(inp.dt_bias), D=f32dev(inp.D), z=dev(inp.z, "bf16"))
        status = lib.ssm_check_device(torch.cuda.current_stream().cuda_stream)
    finally:
        lib.ssm_debug_ssd_stall(-1, 0)
    assert status == 7, ssm.STATUS.get(status, status)
    assert lib.ssm_check_device(torch.cuda.current_stream().cuda_stream) == 0   # cleared
    out, ls = run_ssd(inp)            # raises if the clean call flags anything
    ref, rls = _ref(inp)
    assert rel_err(host(out), ref) <= TOL["bf16"]
    assert rel_err(ls.cpu().numpy(), rls) <= TOL["bf16"]
