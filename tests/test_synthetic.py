"""The seeded input generator: published splitmix64 outputs, bf16 rounding
against torch, counter addressing and the workload recipes.  No GPU."""
import numpy as np
import torch

from mixture_experts_layer_56_b200 import synthetic as S


def test_splitmix64_published_sequence():
    # the first three outputs of splitmix64 seeded with 0 (state advances by
    # the golden gamma before each output)
    g = 0x9E3779B97F4A7C15
    got = S.splitmix64(np.array([0, g, (2 * g) % 2**64], dtype=np.uint64))
    assert [int(v) for v in got] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 7,
                        np.array([0.0, -0.0, 1e-40, 3.0e38, np.inf, -np.inf], np.float32)])
    ours = S.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    np.testing.assert_array_equal(S.bf16_bits_to_f32(ours),
                                  torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_counter_addressing_and_moments():
    a = S.standard_normal(0, 5, 1 << 23)
    b = S.standard_normal(0, 5, 1000, start=4321)
    np.testing.assert_array_equal(a[4321:5321], b)
    assert abs(a.mean()) < 2e-3 and abs(a.std() - 1.0) < 2e-3


def test_workload_recipe_shapes():
    wl = S.custom_workload("t", T=10, d=64, n_routed=5, n_shared=2, inter=64, top_k=2,
                           bias_var=0.5, zipf_s=1.1)
    x = S.make_inputs(wl)
    assert x.u.shape == (10, 64) and x.u.dtype == np.uint16
    assert x.W1.shape == (5, 64, 64) and x.W2.shape == (5, 64, 64)
    assert x.W1_s.shape == (2, 64, 64) and x.bias.dtype == np.float32
    c = S.zipf_row_scale(128, 1.1)
    np.testing.assert_allclose(c.mean(), 1.0)
    assert np.all(np.diff(c) < 0)
    t = S.make_inputs(S.WORKLOADS["tiny"])
    assert t.u.dtype == np.float32 and t.bias is None
