"""ssm_scan_fwd_noalloc: the single-direction scan for callers that cannot
allocate device memory when they run it (a plugin that only gets tensors and
a stream at enqueue time, a serving loop that allows no allocation after
start-up).  It draws its scratch from an array the library owns; its results
must equal ssm_scan_fwd's with a caller workspace.  Collected last."""
import ctypes

import numpy as np
import pytest
import torch

import ssm_gen
import selective_state_space_24_b200 as ssm
from gpu_util import dev, f32dev

pytestmark = pytest.mark.gpu


def _call_both(inp, reverse):
    x, delta = dev(inp.x, inp.dtype), dev(inp.delta, inp.dtype)
    A, B, C = f32dev(inp.A_f), dev(inp.B_f, inp.dtype), dev(inp.C_f, inp.dtype)
    bias, D, z = f32dev(inp.dt_bias_f), f32dev(inp.D_f), dev(inp.z_f, inp.dtype)
    ls_ref = torch.zeros((inp.batch, inp.dim, inp.dstate), device="cuda")
    ref = ssm.ssm_scan_fwd(x, delta, A, B, C, delta_bias=bias, D=D, z=z, reverse=reverse,
                           last_state=ls_ref)
    outs = []
    for _ in range(2):   # two calls in a row share the scratch array
        ls = torch.full((inp.batch, inp.dim, inp.dstate), 3.0, device="cuda")
        o = ssm.ssm_scan_fwd_noalloc(x, delta, A, B, C, delta_bias=bias, D=D, z=z,
                                     reverse=reverse, last_state=ls)
        outs.append((o, ls))
    torch.cuda.synchronize()
    return ref, ls_ref, outs


@pytest.mark.parametrize("dtype,reverse", [("f32", False), ("bf16", True)])
def test_noalloc_matches_workspace_path(cuda_device, dtype, reverse):
    # long enough that the scan is cut into segments and needs scratch
    inp = ssm_gen.make_s6_inputs(2, 3000, 96, 16, dtype=dtype, seed=21, random_A=True)
    dims = ssm.ssm_dims(inp.batch, inp.seqlen, inp.dim, inp.dstate,
                        ssm.SSM_F32 if dtype == "f32" else ssm.SSM_BF16)
    assert ssm.capi().ssm_scan_workspace_size(ctypes.byref(dims)) > 0
    ref, ls_ref, outs = _call_both(inp, reverse)
    # the same kernels on the same plan: the results must be bit-identical
    # (a stale carry left in the shared array by the first call would show
    # up in the second)
    for o, ls in outs:
        assert torch.equal(o, ref)
        assert torch.equal(ls, ls_ref)
