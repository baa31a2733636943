"""The seeded input generator: deterministic, same bytes on host (NumPy) and
torch devices, and the stated distributions."""
import numpy as np
import torch

from group_limited_routed_moe_b200 import synth as S


def test_weights_numpy_equals_torch_cpu():
    a = S.weight_bits_np(7, 3, S.W_DOWN, experts=[0, 5, 127])
    b = S.weight_bits_torch(7, 3, S.W_DOWN, "cpu")
    bb = b.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(a, bb[[0, 5, 127]])


def test_weights_deterministic_and_independent():
    a = S.weight_bits_np(0, 0, S.W_GATE, experts=[0, 1])
    b = S.weight_bits_np(0, 0, S.W_GATE, experts=[0, 1])
    c = S.weight_bits_np(0, 1, S.W_GATE, experts=[0, 1])
    assert np.array_equal(a, b)
    assert not np.array_equal(a[0], a[1]) and not np.array_equal(a, c)
    f = (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert abs(f.mean()) < 2e-4 and abs(f.std() - 0.02) < 2e-4
    # correlation between experts and layers is negligible
    g = (c.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert abs(np.corrcoef(f[0].ravel(), g[0].ravel())[0, 1]) < 1e-2


def test_tokens():
    t = S.make_tokens(2048, 2, hot=16)
    assert t.x_bits.shape == (2048, 1536) and t.x_bits.dtype == np.uint16
    assert t.logits.shape == (2048, 128) and t.logits.dtype == np.float32
    assert t.hot_experts.size == 16 and len(set(t.hot_experts.tolist())) == 16
    cold = np.setdiff1d(np.arange(128), t.hot_experts)
    assert abs(t.logits[:, t.hot_experts].mean() - 2.0) < 0.05
    assert abs(t.logits[:, cold].mean()) < 0.05
    assert abs(t.bias.std() - 0.1) < 0.03
    t2 = S.make_tokens(2048, 2, hot=16)
    assert np.array_equal(t.x_bits, t2.x_bits) and np.array_equal(t.logits, t2.logits)


def test_bf16_packing_round_nearest_even():
    v = np.array([1.0, 1.00390625, 1.01171875, -2.5, 0.0], np.float32)
    assert S.f32_to_bf16_bits(v).tolist() == [0x3F80, 0x3F80, 0x3F82, 0xC020, 0]
    r = np.random.default_rng(0).standard_normal(10000).astype(np.float32)
    ref = torch.from_numpy(r).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(S.f32_to_bf16_bits(r), ref)
