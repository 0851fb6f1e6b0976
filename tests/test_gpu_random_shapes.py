"""Randomised parity of the plain S6 entry points against the float64 oracle.

A hundred seeded cases draw the batch, length, width, state count, element
type, direction(s) and which optional inputs are present, so that the
library's plan (segments or not, one or two channels per thread, two or
four threads per channel) is exercised at sizes no hand-written case
picks; every output and last state is compared in full.  Twenty-five more
draw backward problems and compare every gradient with the autograd
oracle, and fifteen draw Mamba2 SSD problems (batch, length, heads,
optional inputs) against the sequential oracle."""
import numpy as np
import pytest
import torch

import oracle
import ssm_gen
import selective_state_space_24_b200 as ssm
from oracle import grads as ograds
from gpu_util import NTHREADS, TOL, dev, f32dev, host, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    ssm.load()


def _draw(seed, max_elems=3_000_000):
    rng = np.random.default_rng(seed)
    dtype = "f32" if rng.random() < 0.5 else "bf16"
    vec = 4 if dtype == "f32" else 8
    while True:
        Bz = int(rng.integers(1, 7))
        L = int(rng.choice([int(rng.integers(1, 40)), int(rng.integers(40, 700)), int(rng.integers(700, 3000))]))
        D = vec * int(rng.integers(1, 96))
        N = int(rng.choice([16, 16, 16, int(rng.integers(1, 17))]))
        if Bz * L * D * N <= max_elems:
            break
    flags = dict(bidir=bool(rng.random() < 0.5), gate=bool(rng.random() < 0.7), skip=bool(rng.random() < 0.7),
                 bias=bool(rng.random() < 0.7), softplus=bool(rng.random() < 0.8), reverse=bool(rng.random() < 0.5))
    if not flags["softplus"]:   # dt = |delta| > 0 then, with no (negative) bias added
        flags["bias"] = False
    return dtype, Bz, L, D, N, flags


@pytest.mark.parametrize("seed", range(100))
def test_forward(seed):
    dtype, Bz, L, D, N, f = _draw(1000 + seed)
    inp = ssm_gen.make_s6_inputs(Bz, L, D, N, dtype=dtype, bidir=f["bidir"], seed=seed, gate=f["gate"],
                                 random_A=True, random_D=True)
    delta = inp.delta if f["softplus"] else ssm_gen.round_to_bf16(np.abs(inp.delta)) if dtype == "bf16" \
        else np.abs(inp.delta)
    x, dl = dev(inp.x, dtype), dev(delta, dtype)

    def params(s):
        return dict(A=getattr(inp, "A_" + s), B=getattr(inp, "B_" + s), C=getattr(inp, "C_" + s),
                    D=getattr(inp, "D_" + s) if f["skip"] else None,
                    z=getattr(inp, "z_" + s) if f["gate"] else None,
                    delta_bias=getattr(inp, "dt_bias_" + s) if f["bias"] else None)

    def dirp(s):
        p = params(s)
        return ssm.DirParams(A=f32dev(p["A"]), B=dev(p["B"], dtype), C=dev(p["C"], dtype), D=f32dev(p["D"]),
                             z=dev(p["z"], dtype), delta_bias=f32dev(p["delta_bias"]),
                             last_state=torch.empty((Bz, D, N), device="cuda"))

    tol = TOL[dtype]
    if f["bidir"]:
        pf, pb = dirp("f"), dirp("b")
        out = ssm.bidir_scan_fwd(x, dl, pf, pb, delta_softplus=f["softplus"])
        torch.cuda.synchronize()
        ref, rlf, rlb = oracle.bidir_arrays(inp.x, delta, params("f"), params("b"), softplus=f["softplus"],
                                            nthreads=NTHREADS)
        assert rel_err(pf.last_state.cpu().numpy(), rlf) <= tol
        assert rel_err(pb.last_state.cpu().numpy(), rlb) <= tol
    else:
        p = dirp("f")
        out = ssm.ssm_scan_fwd(x, dl, p.A, p.B, p.C, delta_bias=p.delta_bias, delta_softplus=f["softplus"],
                               D=p.D, z=p.z, reverse=f["reverse"], last_state=p.last_state)
        torch.cuda.synchronize()
        q = params("f")
        ref, rst = oracle.s6_arrays(inp.x, delta, q["A"], q["B"], q["C"], delta_bias=q["delta_bias"],
                                    softplus=f["softplus"], D=q["D"], z=q["z"], reverse=f["reverse"],
                                    nthreads=NTHREADS)
        assert rel_err(p.last_state.cpu().numpy(), rst) <= tol
    assert rel_err(host(out), ref) <= tol, (dtype, Bz, L, D, N, f)


@pytest.mark.parametrize("seed", range(25))
def test_backward(seed):
    dtype, Bz, L, D, N, f = _draw(2000 + seed, max_elems=1_200_000)
    inp = ssm_gen.make_s6_inputs(Bz, L, D, N, dtype=dtype, seed=seed, gate=f["gate"], random_A=True,
                                 random_D=True)
    dout = np.random.default_rng(seed).standard_normal(inp.x.shape).astype(np.float32)
    if dtype == "bf16":
        dout = ssm_gen.round_to_bf16(dout)
    g = ssm.ssm_scan_bwd(dev(inp.x, dtype), dev(inp.delta, dtype), f32dev(inp.A_f), dev(inp.B_f, dtype),
                         dev(inp.C_f, dtype), dev(dout, dtype),
                         delta_bias=f32dev(inp.dt_bias_f) if f["bias"] else None,
                         D=f32dev(inp.D_f) if f["skip"] else None, z=dev(inp.z_f, dtype) if f["gate"] else None,
                         reverse=f["reverse"])
    torch.cuda.synchronize()
    ref = ograds.s6_grads(inp.x, inp.delta, inp.A_f, inp.B_f, inp.C_f, dout,
                          delta_bias=inp.dt_bias_f if f["bias"] else None, D=inp.D_f if f["skip"] else None,
                          z=inp.z_f if f["gate"] else None, reverse=f["reverse"])
    names = {"dx": "x", "ddelta": "delta", "dA": "A", "dB": "B", "dC": "C", "dD": "D", "dz": "z",
             "ddelta_bias": "delta_bias"}
    for k, t in g.items():
        e = rel_err(t.cpu().numpy(), ref[names[k]])
        assert e <= TOL[dtype], (k, e, dtype, Bz, L, D, N, f)


@pytest.mark.parametrize("seed", range(15))
def test_ssd(seed):
    rng = np.random.default_rng(3000 + seed)
    Bz, L, H = int(rng.integers(1, 4)), int(rng.integers(1, 700)), int(rng.integers(1, 7))
    N = 128   # the one state size the SSD kernel supports (headdim 64, chunk 64)
    gate, skip, bias = (bool(rng.random() < 0.7) for _ in range(3))
    inp = ssm_gen.make_ssd_inputs(Bz, L, H, 64, N, 64, dtype="bf16", seed=seed, gate=gate, random_D=True)
    ls = torch.empty((Bz, H, 64, N), device="cuda")
    out = ssm.ssd_chunk_fwd(dev(inp.x, "bf16"), dev(inp.delta, "bf16"), f32dev(inp.A), dev(inp.B, "bf16"),
                            dev(inp.C, "bf16"), chunk=64, delta_bias=f32dev(inp.dt_bias) if bias else None,
                            D=f32dev(inp.D) if skip else None, z=dev(inp.z, "bf16") if gate else None,
                            last_state=ls)
    torch.cuda.synchronize()
    ssm.check_device()
    ref, rls = oracle.ssd_seq_arrays(inp.x, inp.delta, inp.A, inp.B, inp.C,
                                     delta_bias=inp.dt_bias if bias else None, softplus=True,
                                     D=inp.D if skip else None, z=inp.z if gate else None, nthreads=NTHREADS)
    assert rel_err(host(out), ref) <= TOL["bf16"], (Bz, L, H, N, gate, skip, bias)
    assert rel_err(ls.cpu().numpy(), rls) <= TOL["bf16"]
