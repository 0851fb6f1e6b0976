"""Helpers shared by the GPU tests: moving generator inputs to the device and
the error metric.

Error metric (max relative error with a floor): near-zero outputs (gated
values, two directions cancelling) make a plain elementwise ratio
meaningless, so each element's error is divided by max(|o_i|, rms(o)):
    err = max_i |g_i - o_i| / max(|o_i|, rms(o))
Tolerances: 1e-4 for float32 inputs, 2e-2 for bf16 inputs with float32
state (the bf16 output rounding alone is 2^-9 relative).
"""
import os

import numpy as np
import torch

import selective_state_space_24_b200 as ssm

TOL = {"f32": 1e-4, "bf16": 2e-2}

# the oracle runs on every host core the process may use
NTHREADS = max(1, len(os.sched_getaffinity(0)))


def dev(a, dtype, device="cuda"):
    """numpy float32 array (bf16-exact if dtype is bf16) -> device tensor."""
    if a is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t.to(device)


def f32dev(a, device="cuda"):
    if a is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def rel_err(g, o) -> float:
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    if o.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(o * o)))
    den = np.maximum(np.abs(o), max(rms, 1e-30))
    return float(np.max(np.abs(g - o) / den))


def host(t):
    return t.float().cpu().numpy().astype(np.float64)


def dir_params(inp, which, last_state=False, device="cuda"):
    s = "_f" if which == "f" else "_b"
    dt = inp.dtype
    ls = None
    if last_state:
        ls = torch.zeros((inp.batch, inp.dim, inp.dstate), dtype=torch.float32, device=device)
    return ssm.DirParams(A=f32dev(getattr(inp, "A" + s), device), B=dev(getattr(inp, "B" + s), dt, device),
                         C=dev(getattr(inp, "C" + s), dt, device),
                         delta_bias=f32dev(getattr(inp, "dt_bias" + s), device),
                         D=f32dev(getattr(inp, "D" + s), device), z=dev(getattr(inp, "z" + s), dt, device),
                         last_state=ls)


def run_bidir(inp, last_state=False, device="cuda"):
    x = dev(inp.x, inp.dtype, device)
    delta = dev(inp.delta, inp.dtype, device)
    f = dir_params(inp, "f", last_state, device)
    b = dir_params(inp, "b", last_state, device)
    out = ssm.bidir_scan_fwd(x, delta, f, b)
    torch.cuda.synchronize()
    return out, f.last_state, b.last_state


def run_s6(inp, reverse=False, last_state=True, device="cuda"):
    x = dev(inp.x, inp.dtype, device)
    delta = dev(inp.delta, inp.dtype, device)
    p = dir_params(inp, "f", last_state, device)
    out = ssm.ssm_scan_fwd(x, delta, p.A, p.B, p.C, delta_bias=p.delta_bias, D=p.D, z=p.z,
                           reverse=reverse, last_state=p.last_state)
    torch.cuda.synchronize()
    return out, p.last_state
