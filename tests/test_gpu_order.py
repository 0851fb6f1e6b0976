"""GPU parity of the scans along a given order of the positions (row,
column, centre-out spiral, random permutations) with and without a token
mask, against the float64 oracle, through the C ABI."""
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


def _order(kind, L, side):
    if kind == "cols":
        return ssm_gen.order_cols(side, L // side)
    if kind == "spiral":
        return ssm_gen.order_spiral(side, L // side)
    return ssm_gen.order_random(L, seed=L)


def _i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def _u8(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("kind,L,side", [("cols", 196, 14), ("spiral", 196, 14), ("random", 1500, 1)])
@pytest.mark.parametrize("masked", [False, True])
@pytest.mark.parametrize("reverse", [False, True])
def test_single_direction_ordered(dtype, kind, L, side, masked, reverse):
    batch, D = 2, 64
    inp = ssm_gen.make_s6_inputs(batch, L, D, 16, dtype=dtype, seed=L + 3 * masked + reverse,
                                 random_A=True, random_D=True)
    order = _order(kind, L, side)
    mask = ssm_gen.token_mask(batch, L, 0.7, seed=5) if masked else None
    p = dir_params(inp, "f", last_state=True)
    out = ssm.ssm_scan_fwd_ordered(dev(inp.x, dtype), dev(inp.delta, dtype), p.A, p.B, p.C,
                                   order=_i32(order), mask=None if mask is None else _u8(mask),
                                   delta_bias=p.delta_bias, D=p.D, z=p.z, reverse=reverse,
                                   last_state=p.last_state)
    torch.cuda.synchronize()
    ssm.check_device()
    ref, rst = oracle.s6_ordered_arrays(inp.x, inp.delta, inp.A_f, inp.B_f, inp.C_f, order=order,
                                        mask=mask, delta_bias=inp.dt_bias_f, D=inp.D_f, z=inp.z_f,
                                        reverse=reverse, nthreads=8)
    assert rel_err(host(out), ref) <= TOL[dtype]
    assert rel_err(p.last_state.cpu().numpy(), rst) <= TOL[dtype]
    if masked:
        assert torch.all(out.float().cpu()[torch.from_numpy(mask == 0)] == 0)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("kind,L,side,batch,D", [("spiral", 196, 14, 2, 64), ("random", 2048, 1, 2, 96),
                                                   ("cols", 1024, 32, 16, 768)])
@pytest.mark.parametrize("masked", [False, True])
def test_bidir_ordered(dtype, kind, L, side, batch, D, masked):
    inp = ssm_gen.make_s6_inputs(batch, L, D, 16, dtype=dtype, bidir=True, seed=L + masked,
                                 random_A=True, random_D=True)
    order = _order(kind, L, side)
    mask = ssm_gen.token_mask(batch, L, 0.6, seed=9) if masked else None
    f = dir_params(inp, "f", last_state=True)
    b = dir_params(inp, "b", last_state=True)
    out = ssm.bidir_scan_fwd_ordered(dev(inp.x, dtype), dev(inp.delta, dtype), f, b, order=_i32(order),
                                     mask=None if mask is None else _u8(mask))
    torch.cuda.synchronize()
    ssm.check_device()
    cols = None
    if batch * D > 256:
        cols = np.random.default_rng(1).choice(batch * D, 48, replace=False)
    fw = dict(delta_bias=inp.dt_bias_f, A=inp.A_f, B=inp.B_f, C=inp.C_f, D=inp.D_f, z=inp.z_f)
    bw = dict(delta_bias=inp.dt_bias_b, A=inp.A_b, B=inp.B_b, C=inp.C_b, D=inp.D_b, z=inp.z_b)
    ref, rlf, rlb = oracle.bidir_ordered_arrays(inp.x, inp.delta, fw, bw, order=order, mask=mask,
                                                cols=cols, nthreads=8)
    g = host(out)
    if cols is None:
        assert rel_err(g, ref) <= TOL[dtype]
        assert rel_err(f.last_state.cpu().numpy(), rlf) <= TOL[dtype]
        assert rel_err(b.last_state.cpu().numpy(), rlb) <= TOL[dtype]
    else:
        bb, dd = np.divmod(cols, D)
        assert rel_err(g[bb, :, dd], ref[bb, :, dd]) <= TOL[dtype]
        assert rel_err(f.last_state.cpu().numpy()[bb, dd], rlf[bb, dd]) <= TOL[dtype]
        assert rel_err(b.last_state.cpu().numpy()[bb, dd], rlb[bb, dd]) <= TOL[dtype]


def test_identity_order_is_bitwise_plain():
    inp = ssm_gen.make_s6_inputs(2, 300, 64, 16, dtype="f32", bidir=True, seed=12)
    f, b = dir_params(inp, "f"), dir_params(inp, "b")
    x, delta = dev(inp.x, "f32"), dev(inp.delta, "f32")
    with ssm.s6_mapping(ssm.MAPPING_WHOLE_CHANNELS):   # the layout the ordered scan takes
        plain = ssm.bidir_scan_fwd(x, delta, f, b)
    ordered = ssm.bidir_scan_fwd_ordered(x, delta, f, b, order=_i32(np.arange(300)),
                                         mask=_u8(np.ones((2, 300))))
    torch.cuda.synchronize()
    assert torch.equal(plain, ordered)


def test_out_of_range_order_is_reported():
    """An order entry outside [0, L) is caught by the kernel's bounds check
    (no access outside the tensors) and reported by ssm_check_device."""
    inp = ssm_gen.make_s6_inputs(1, 64, 32, 16, dtype="f32", seed=2)
    p = dir_params(inp, "f")
    order = np.arange(64)
    order[10] = 64
    ssm.check_device()   # start clean
    ssm.ssm_scan_fwd_ordered(dev(inp.x, "f32"), dev(inp.delta, "f32"), p.A, p.B, p.C, order=_i32(order),
                             delta_bias=p.delta_bias, D=p.D, z=p.z)
    with pytest.raises(ssm.SSMError) as e:
        ssm.check_device()
    assert e.value.status == 1
    ssm.check_device()   # the error word was cleared
