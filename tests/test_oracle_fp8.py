"""Pins of the oracle's block-FP8 functions (e4m3_to_f64, dequant_block_fp8,
moe_layer_fp8) to things other than themselves:

* every one of the 256 E4M3 codes against PyTorch's float8_e4m3fn (a library
  decoder written independently of the oracle), and the format's closed forms
  (largest finite 448, smallest subnormal 2**-9, 1.0, the two NaN codes, -0);
* the block structure: constant codes expose the scale map cell by cell on a
  non-square block grid (a transposed or mis-strided scale fails), and random
  codes against an element-by-element loop over the library decoder;
* the layer: with power-of-two scales every dequantised weight is a bf16
  value, so moe_layer_fp8 must equal the bf16 layer (itself pinned in
  test_oracle_layer.py) on those weights; gate and up swapped, or a
  transposed down block map, would not."""
import numpy as np
import pytest
import torch

import oracle as O
from group_limited_routed_moe_b200 import synth


def _lib_decode(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def test_e4m3_all_codes_match_library_decoder():
    codes = np.arange(256, dtype=np.uint8)
    got, lib = O.e4m3_to_f64(codes), _lib_decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(lib))
    ok = ~np.isnan(lib)
    assert np.array_equal(got[ok], lib[ok])
    assert np.array_equal(np.signbit(got[ok]), np.signbit(lib[ok]))


def test_e4m3_closed_forms():
    v = O.e4m3_to_f64(np.arange(256, dtype=np.uint8))
    assert v[0x00] == 0.0 and not np.signbit(v[0x00])
    assert v[0x80] == 0.0 and np.signbit(v[0x80])
    assert v[0x01] == 2.0 ** -9          # smallest subnormal
    assert v[0x07] == 7 * 2.0 ** -9      # largest subnormal
    assert v[0x08] == 2.0 ** -6          # smallest normal
    assert v[0x38] == 1.0
    assert v[0x3F] == 1.875
    assert v[0x40] == 2.0
    assert v[0x7E] == 448.0 and v[0xFE] == -448.0
    assert np.flatnonzero(np.isnan(v)).tolist() == [0x7F, 0xFF]
    assert np.array_equal(v[0x80:0xFF], -v[0x00:0x7F])


def test_e4m3_monotone_with_binade_spacing():
    v = O.e4m3_to_f64(np.arange(0x7F, dtype=np.uint8))
    d = np.diff(v)
    assert np.all(d > 0)
    # eight codes per binade, evenly spaced; subnormals continue the first binade's spacing
    assert np.all(d[:8] == 2.0 ** -9)
    for E in range(1, 16):
        lo = 8 * E
        seg = d[lo:min(lo + 8, len(d))]
        assert np.all(seg == 2.0 ** (E - 7 - 3))


def test_dequant_exposes_the_scale_map():
    rng = np.random.default_rng(3)
    s = rng.uniform(0.5, 2.0, size=(2, 3, 2)).astype(np.float32)   # 2 matrices, 3 x 2 blocks
    codes = np.full((2, 384, 256), 0x38, np.uint8)                  # every code 1.0
    w = O.dequant_block_fp8(codes, s)
    for m in range(2):
        for r in (0, 127, 128, 255, 256, 383):
            for c in (0, 127, 128, 255):
                assert w[m, r, c] == np.float64(s[m, r // 128, c // 128])
    with pytest.raises(ValueError):
        O.dequant_block_fp8(codes, s.transpose(0, 2, 1))


def test_dequant_random_codes_against_elementwise_loop():
    rng = np.random.default_rng(4)
    codes = rng.integers(0, 256, size=(256, 384)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x11
    s = rng.uniform(1e-4, 1e-2, size=(2, 3)).astype(np.float32)
    w = O.dequant_block_fp8(codes, s)
    lib = _lib_decode(codes)
    for r in range(0, 256, 7):
        for c in range(0, 384, 5):
            assert w[r, c] == lib[r, c] * float(s[r // 128, c // 128])


def test_layer_fp8_equals_bf16_layer_on_the_dequantised_weights():
    T = 3
    tok = synth.make_tokens(T, 21)
    rr = O.route(tok.logits, tok.bias)
    used = np.unique(rr.topk_idx)
    q, s = {}, {}
    for name, which in (("g", synth.W_GATE), ("u", synth.W_UP), ("d", synth.W_DOWN)):
        qq, ss = synth.fp8_weights_np(0, 0, which, used)
        ss = ss * synth.fp8_scale_jitter(ss.shape, 10 + which)
        full_q = np.zeros((128,) + qq.shape[1:], np.uint8)
        full_s = np.ones((128,) + ss.shape[1:], np.float32)
        full_q[used], full_s[used] = qq, ss
        q[name], s[name] = full_q, full_s
    got = O.moe_layer_fp8(tok.x_bits, tok.logits, tok.bias, q["g"], s["g"], q["u"], s["u"],
                          q["d"], s["d"], route_result=rr)
    bits = {}
    for name in "gud":
        w = O.dequant_block_fp8(q[name][used], s[name][used])
        b = O.f64_to_bf16_bits(w)
        assert np.array_equal(O.bf16_bits_to_f64(b), w)  # power-of-two scales: exact in bf16
        full = np.zeros(q[name].shape, np.uint16)
        full[used] = b
        bits[name] = full
    ref = O.moe_layer(tok.x_bits, tok.logits, tok.bias, bits["g"], bits["u"], bits["d"],
                      route_result=rr)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-15)
    # gate and up are not interchangeable: swapping them changes the layer
    swapped = O.moe_layer_fp8(tok.x_bits, tok.logits, tok.bias, q["u"], s["u"], q["g"], s["g"],
                              q["d"], s["d"], route_result=rr)
    assert O.rel_l2(swapped, ref) > 0.1
