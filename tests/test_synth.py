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


def test_fp8_weights_are_block_quantised_bf16_weights():
    """The synthetic FP8 checkpoint: power-of-two scales with max|w| in
    (224 s, 448 s], no NaN code, and every code the E4M3 value nearest to w/s
    (the dequantised weight is within half an E4M3 spacing of w); the "amax"
    mode puts a code of magnitude 448 into every block."""
    w = S.weight_bits_np(0, 2, S.W_DOWN, experts=[5])
    wf = (w.astype(np.uint32) << 16).view(np.float32).astype(np.float64)[0]
    q, s = S.fp8_weights_np(0, 2, S.W_DOWN, experts=[5])
    assert q.shape == (1, 512, 1536) and q.dtype == np.uint8 and s.shape == (1, 4, 12)
    assert np.all((q & 0x7F) != 0x7F)
    m, _ = np.frexp(s)
    assert np.all(m == 0.5)                                   # powers of two
    amax = np.abs(wf).reshape(4, 128, 12, 128).max(axis=(1, 3))
    assert np.all(amax <= 448 * s[0]) and np.all(amax > 224 * s[0])
    v = torch.from_numpy(q[0]).view(torch.float8_e4m3fn).double().numpy()
    full_s = np.repeat(np.repeat(s[0].astype(np.float64), 128, 0), 128, 1)
    a = np.abs(wf / full_s)
    # spacing of E4M3 around |a|: 2**-9 below 2**-6, else 2**(floor(log2 a) - 3)
    spacing = np.where(a < 2.0 ** -6, 2.0 ** -9, np.exp2(np.floor(np.log2(np.maximum(a, 2.0 ** -6))) - 3))
    assert np.all(np.abs(v - wf / full_s) <= spacing / 2)
    q2, s2 = S.fp8_weights_np(0, 2, S.W_DOWN, experts=[5], mode="amax")
    assert np.allclose(s2[0], (amax / 448).astype(np.float32), rtol=0, atol=0)
    blocks = (q2[0] & 0x7F).reshape(4, 128, 12, 128).max(axis=(1, 3))
    assert np.all(blocks == 0x7E)
    j = S.fp8_scale_jitter((3, 12, 4), 1)
    assert set(np.log2(j).ravel().tolist()) <= {-2.0, -1.0, 0.0, 1.0, 2.0}


def test_nvfp4_weights_are_block_quantised_bf16_weights():
    """The synthetic NVFP4 checkpoint ([out, in] form): a power-of-two tensor
    scale g with max|w| <= 6 * 448 * g < 2 * max|w|, E4M3 block scales (no NaN)
    of 16 weights along the input dimension, every code the E2M1 value nearest
    to w / (s g) (within half an E2M1 spacing, saturated at 6), codes packed low
    nibble first; the encoder agrees with ml_dtypes' float4_e2m1fn rounding."""
    import ml_dtypes
    w = S.weight_bits_np(0, 1, S.W_UP, experts=[9])
    wf = (w.astype(np.uint32) << 16).view(np.float32).astype(np.float64)[0].T  # [512, 1536]
    q, s, g = S.nvfp4_weights_np(0, 1, S.W_UP, experts=[9])
    assert q.shape == (1, 512, 768) and s.shape == (1, 512, 96) and g.shape == (1,)
    assert np.all((s & 0x7F) != 0x7F)
    m, _ = np.frexp(g)
    assert np.all(m == 0.5)
    amax = np.abs(wf).max()
    assert amax <= 6 * 448 * float(g[0]) < 2 * amax
    codes = np.empty((512, 1536), np.uint8)
    codes[:, 0::2], codes[:, 1::2] = q[0] & 0xF, q[0] >> 4
    v = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    sv = torch.from_numpy(s[0]).view(torch.float8_e4m3fn).double().numpy()
    a = wf / (np.repeat(sv, 16, axis=1) * float(g[0]))
    spacing = np.where(np.abs(a) < 2, 0.5, np.where(np.abs(a) < 4, 1.0, 2.0))
    assert np.all(np.abs(v - np.clip(a, -6, 6)) <= spacing / 2 + 1e-12)
    enc = S._encode_e2m1(torch.from_numpy(np.clip(a, -6, 6).astype(np.float32))).numpy()
    lib = np.clip(a, -6, 6).astype(np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8)
    same = (enc == lib) | ((enc & 7) == 0) & ((lib & 7) == 0)  # +-0 either way
    assert np.all(same)
    _, _, g2 = S.nvfp4_weights_np(0, 1, S.W_UP, experts=[9], mode="amax")
    assert g2[0] == np.float32(np.float32(amax) / np.float32(6 * 448))
