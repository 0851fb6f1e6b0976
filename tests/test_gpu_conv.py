"""GPU parity of the scans with the depthwise causal conv1d computed inside
(ssm_scan_fwd_conv, bidir_scan_fwd_conv) against the float64 oracle,
through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import ssm_gen
import selective_state_space_24_b200 as ssm
from gpu_util import TOL, dev, f32dev, host, rel_err, dir_params

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    ssm.load()


def _conv(rng, D, width, bias, silu):
    w = (rng.standard_normal((D, width)) / np.sqrt(width)).astype(np.float32)
    b = (0.1 * rng.standard_normal(D)).astype(np.float32) if bias else None
    return dict(weight=w, bias=b, silu=silu)


def _dev_conv(c):
    return ssm.Conv(weight=f32dev(c["weight"]), bias=f32dev(c["bias"]), silu=c["silu"])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("width", [1, 2, 3, 4])
@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("L", [150, 2500])   # one segment; many segments (window preloaded)
def test_single_direction_conv(dtype, width, reverse, L):
    rng = np.random.default_rng(width + 10 * reverse + L)
    batch, D = 2, 64
    inp = ssm_gen.make_s6_inputs(batch, L, D, 16, dtype=dtype, seed=L + width, random_A=True,
                                 random_D=True)
    c = _conv(rng, D, width, bias=width % 2 == 1, silu=width != 2)
    p = dir_params(inp, "f", last_state=True)
    out = ssm.ssm_scan_fwd_conv(dev(inp.x, dtype), _dev_conv(c), dev(inp.delta, dtype), p.A, p.B, p.C,
                                delta_bias=p.delta_bias, D=p.D, z=p.z, reverse=reverse,
                                last_state=p.last_state)
    torch.cuda.synchronize()
    ref, rst = oracle.s6_conv_arrays(inp.x, c["weight"], inp.delta, inp.A_f, inp.B_f, inp.C_f,
                                     conv_bias=c["bias"], conv_silu=c["silu"], reverse=reverse,
                                     delta_bias=inp.dt_bias_f, D=inp.D_f, z=inp.z_f, nthreads=8)
    assert rel_err(host(out), ref) <= TOL[dtype]
    assert rel_err(p.last_state.cpu().numpy(), rst) <= TOL[dtype]


@pytest.mark.parametrize("dtype,batch,L,D", [("f32", 2, 197, 768), ("bf16", 2, 3000, 96)])
def test_bidir_conv(dtype, batch, L, D):
    """Each direction convolves x_in with its own kernel along its own scan
    direction (Vim's per-direction conv), then the two scans are summed."""
    rng = np.random.default_rng(L)
    inp = ssm_gen.make_s6_inputs(batch, L, D, 16, dtype=dtype, bidir=True, seed=L, random_A=True,
                                 random_D=True)
    cf, cb = _conv(rng, D, 4, True, True), _conv(rng, D, 3, False, True)
    f = dir_params(inp, "f", last_state=True)
    b = dir_params(inp, "b", last_state=True)
    out = ssm.bidir_scan_fwd_conv(dev(inp.x, dtype), dev(inp.delta, dtype), f, b, _dev_conv(cf),
                                  _dev_conv(cb))
    torch.cuda.synchronize()
    fw = dict(delta_bias=inp.dt_bias_f, A=inp.A_f, B=inp.B_f, C=inp.C_f, D=inp.D_f, z=inp.z_f)
    bw = dict(delta_bias=inp.dt_bias_b, A=inp.A_b, B=inp.B_b, C=inp.C_b, D=inp.D_b, z=inp.z_b)
    cols = np.random.default_rng(2).choice(batch * D, 48, replace=False)
    ref, rlf, rlb = oracle.bidir_conv_arrays(inp.x, inp.delta, fw, bw, cf, cb, cols=cols, nthreads=8)
    bb, dd = np.divmod(cols, D)
    g = host(out)
    assert rel_err(g[bb, :, dd], ref[bb, :, dd]) <= TOL[dtype]
    assert rel_err(f.last_state.cpu().numpy()[bb, dd], rlf[bb, dd]) <= TOL[dtype]
    assert rel_err(b.last_state.cpu().numpy()[bb, dd], rlb[bb, dd]) <= TOL[dtype]
