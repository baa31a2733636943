"""Pins of the oracle's NVFP4 functions (e2m1_to_f64, unpack_fp4,
dequant_nvfp4, moe_layer_nvfp4) to things other than themselves:

* all 16 E2M1 codes against ml_dtypes' float4_e2m1fn (a library decoder
  written independently of the oracle), and the format's closed forms (the
  eight magnitudes 0 .. 6, sign symmetry, -0);
* the byte order: hand-built bytes whose nibbles differ, so that swapped
  nibbles or a wrong stride fail;
* the block structure: constant codes expose the block-scale map cell by cell
  on a grid with several rows and blocks (a transposed or mis-strided map
  fails), the tensor scale multiplies whole matrices, and random codes agree
  with an element-by-element loop over the two library decoders;
* the layer: with power-of-two tensor scales every dequantised weight is a
  bf16 value, so moe_layer_nvfp4 must equal the bf16 layer (itself pinned in
  test_oracle_layer.py) on those weights transposed to the x W form; gate and
  up swapped change it."""
import ml_dtypes
import numpy as np
import pytest
import torch

import oracle as O
from group_limited_routed_moe_b200 import synth


def _lib_e2m1(codes):
    return np.asarray(codes, np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)


def _lib_e4m3(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def test_e2m1_all_codes_match_library_decoder():
    codes = np.arange(16, dtype=np.uint8)
    got, lib = O.e2m1_to_f64(codes), _lib_e2m1(codes)
    assert np.array_equal(got, lib)
    assert np.array_equal(np.signbit(got), np.signbit(lib))


def test_e2m1_closed_forms():
    v = O.e2m1_to_f64(np.arange(16, dtype=np.uint8))
    assert v[:8].tolist() == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert np.array_equal(v[8:], -v[:8])
    assert v[8] == 0.0 and np.signbit(v[8]) and not np.signbit(v[0])
    assert v.max() == 6.0
    with pytest.raises(ValueError):
        O.e2m1_to_f64(np.array([16], np.uint8))


def test_unpack_low_nibble_first():
    packed = np.array([[0x21, 0x7F, 0x80]], np.uint8)
    assert O.unpack_fp4(packed).tolist() == [[1, 2, 0xF, 0x7, 0x0, 0x8]]
    w = O.dequant_nvfp4(np.array([[0x21] * 8], np.uint8), np.array([[0x38]], np.uint8),
                        np.float32(1.0))
    assert w[0, :4].tolist() == [0.5, 1.0, 0.5, 1.0]


def test_dequant_exposes_the_block_scale_map():
    rng = np.random.default_rng(5)
    R, C = 5, 64                                            # 5 rows x 4 blocks of 16
    sc = rng.integers(0x20, 0x50, size=(2, R, C // 16)).astype(np.uint8)
    g = np.array([1.0, 0.375], np.float32)
    packed = np.full((2, R, C // 2), 0x22, np.uint8)        # every code 1.0
    w = O.dequant_nvfp4(packed, sc, g)
    s = _lib_e4m3(sc)
    for m in range(2):
        for r in range(R):
            for c in (0, 15, 16, 31, 32, 47, 48, 63):
                assert w[m, r, c] == s[m, r, c // 16] * float(g[m])
    with pytest.raises(ValueError):
        O.dequant_nvfp4(packed, sc.transpose(0, 2, 1), g)
    with pytest.raises(ValueError):
        O.dequant_nvfp4(packed, sc, g[:1])


def test_dequant_random_codes_against_elementwise_loop():
    rng = np.random.default_rng(6)
    packed = rng.integers(0, 256, size=(3, 48)).astype(np.uint8)
    sc = rng.integers(0x08, 0x7E, size=(3, 6)).astype(np.uint8)
    g = np.float32(0.0123)
    w = O.dequant_nvfp4(packed, sc, g)
    s = _lib_e4m3(sc)
    for r in range(3):
        for c in range(96):
            byte = int(packed[r, c // 2])
            code = byte & 0xF if c % 2 == 0 else byte >> 4
            assert w[r, c] == _lib_e2m1([code])[0] * s[r, c // 16] * float(g)


def _nvfp4_layer_inputs(used, mode="pow2"):
    q, s, g = {}, {}, {}
    for name, which in (("g", synth.W_GATE), ("u", synth.W_UP), ("d", synth.W_DOWN)):
        qq, ss, gg = synth.nvfp4_weights_np(0, 0, which, used, mode=mode)
        full_q = np.zeros((128,) + qq.shape[1:], np.uint8)
        full_s = np.full((128,) + ss.shape[1:], 0x38, np.uint8)
        full_g = np.ones(128, np.float32)
        full_q[used], full_s[used], full_g[used] = qq, ss, gg
        q[name], s[name], g[name] = full_q, full_s, full_g
    return q, s, g


def test_layer_nvfp4_equals_bf16_layer_on_the_dequantised_weights():
    T = 3
    tok = synth.make_tokens(T, 23)
    rr = O.route(tok.logits, tok.bias)
    used = np.unique(rr.topk_idx)
    q, s, g = _nvfp4_layer_inputs(used)
    got = O.moe_layer_nvfp4(tok.x_bits, tok.logits, tok.bias, q["g"], s["g"], g["g"],
                            q["u"], s["u"], g["u"], q["d"], s["d"], g["d"], route_result=rr)
    bits = {}
    for name in "gud":
        w = O.dequant_nvfp4(q[name][used], s[name][used], g[name][used])
        b = O.f64_to_bf16_bits(w)
        assert np.array_equal(O.bf16_bits_to_f64(b), w)  # power-of-two tensor scales: exact
        xw = b.transpose(0, 2, 1)                          # [out, in] -> x W form
        full = np.zeros((128,) + xw.shape[1:], np.uint16)
        full[used] = xw
        bits[name] = full
    ref = O.moe_layer(tok.x_bits, tok.logits, tok.bias, bits["g"], bits["u"], bits["d"],
                      route_result=rr)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-15)
    swapped = O.moe_layer_nvfp4(tok.x_bits, tok.logits, tok.bias, q["u"], s["u"], g["u"],
                                q["g"], s["g"], g["g"], q["d"], s["d"], g["d"], route_result=rr)
    assert O.rel_l2(swapped, ref) > 0.1
