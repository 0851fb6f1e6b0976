"""The seeded input generator: determinism, substream independence, bf16
rounding and the value recipe of the workloads."""
import numpy as np
import torch

import ssm_gen


def test_deterministic_and_seeded():
    a = ssm_gen.make_s6_inputs(2, 10, 8, 16, bidir=True, seed=1)
    b = ssm_gen.make_s6_inputs(2, 10, 8, 16, bidir=True, seed=1)
    c = ssm_gen.make_s6_inputs(2, 10, 8, 16, bidir=True, seed=2)
    for k, v in a.io_tensors().items():
        np.testing.assert_array_equal(v, b.io_tensors()[k])
        assert not np.array_equal(v, c.io_tensors()[k])


def test_substreams_do_not_depend_on_other_tensors():
    a = ssm_gen.make_s6_inputs(2, 10, 8, 16, bidir=False, seed=1, gate=False)
    b = ssm_gen.make_s6_inputs(2, 10, 8, 16, bidir=True, seed=1)
    np.testing.assert_array_equal(a.x, b.x)
    np.testing.assert_array_equal(a.B_f, b.B_f)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    v = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))).astype(np.float32)
    mine = ssm_gen.round_to_bf16(v)
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(mine, ref)
    bits = ssm_gen.bf16_bits(mine)
    back = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(back, mine)


def test_recipe_of_the_workloads():
    inp = ssm_gen.make_s6_inputs(4, 256, 512, 16, bidir=True, seed=0)
    np.testing.assert_array_equal(inp.A_f[3], -(np.arange(16) + 1.0))
    np.testing.assert_array_equal(inp.A_b, inp.A_f)
    assert inp.A_b is not inp.A_f
    assert np.all(inp.D_f == 1.0)
    # dt = softplus(bias) lies in [1e-3, 1e-1]
    dt = np.log1p(np.exp(inp.dt_bias_f.astype(np.float64)))
    assert dt.min() >= 1e-3 * (1 - 1e-5) and dt.max() <= 1e-1 * (1 + 1e-5)
    assert abs(inp.x.std() - 1.0) < 0.01 and abs(inp.delta.std() - 0.5) < 0.01
    assert not np.array_equal(inp.B_f, inp.B_b)
    ssd = ssm_gen.make_ssd_inputs(2, 128, 8, 16, 64, 64, dtype="bf16", seed=0)
    assert np.all((ssd.A <= -1.0) & (ssd.A >= -16.0))
    assert abs(ssd.B.std() * 8.0 - 1.0) < 0.05
    assert np.array_equal(ssm_gen.round_to_bf16(ssd.x), ssd.x)


def test_workload_table():
    w = ssm_gen.WORKLOADS
    assert (w[1]["batch"], w[1]["seqlen"], w[1]["dim"], w[1]["dstate"]) == (64, 197, 768, 16)
    assert (w[3]["batch"], w[3]["seqlen"], w[3]["dim"]) == (4, 16384, 192)
    assert (w[4]["nheads"], w[4]["headdim"], w[4]["dstate"], w[4]["chunk"]) == (32, 64, 128, 64)
