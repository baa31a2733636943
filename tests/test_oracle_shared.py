"""Pins of the oracle's shared-expert layer (moe_layer_shared):

* closed form: one token x = e_k, one shared expert whose only non-zero
  weights are W_gate[k, j] = a, W_up[k, j] = b, W_down[j, n] = c gives
  out[n] = silu(a) * b * c with weight 1 and nothing elsewhere; swapping gate
  and up (a != b), transposing W_down or weighting the shared term by a
  routing weight would all change it;
* no shared experts, or all-zero shared weights, leave the routed layer
  exactly as it is;
* two shared experts add: the layer with both minus the layer with only one
  is the other's dense FFN on every token."""
import numpy as np

import oracle as O
from group_limited_routed_moe_b200 import synth

H, I = 1536, 512


def _bits(a):
    return synth.f32_to_bf16_bits(np.asarray(a, np.float32))


def test_shared_expert_closed_form():
    k, j, n = 700, 33, 1200
    a, b, c = 1.5, -0.75, 0.25
    sg = np.zeros((1, H, I), np.float32); sg[0, k, j] = a
    su = np.zeros((1, H, I), np.float32); su[0, k, j] = b
    sd = np.zeros((1, I, H), np.float32); sd[0, j, n] = c
    x = np.zeros((1, H), np.float32); x[0, k] = 1.0
    zg = np.zeros((128, H, I), np.uint16)
    zd = np.zeros((128, I, H), np.uint16)
    lg = np.zeros((1, 128), np.float32)
    out = O.moe_layer_shared(_bits(x), lg, None, zg, zg, zd, _bits(sg), _bits(su), _bits(sd))
    expect = np.zeros((1, H))
    expect[0, n] = a / (1.0 + np.exp(-a)) * b * c
    assert np.allclose(out, expect, rtol=1e-14, atol=0)
    assert np.count_nonzero(out) == 1


def test_no_or_zero_shared_experts_leave_the_routed_layer():
    T = 3
    tok = synth.make_tokens(T, 31)
    rr = O.route(tok.logits, tok.bias)
    wg, wu, wd = (np.zeros((128,) + shp, np.uint16) for shp in ((H, I), (H, I), (I, H)))
    used = np.unique(rr.topk_idx)
    g, u, d = synth.layer_weights_np(0, 0, used)
    wg[used], wu[used], wd[used] = g, u, d
    ref = O.moe_layer(tok.x_bits, tok.logits, tok.bias, wg, wu, wd, route_result=rr)
    none = O.moe_layer_shared(tok.x_bits, tok.logits, tok.bias, wg, wu, wd,
                              np.zeros((0, H, I), np.uint16), np.zeros((0, H, I), np.uint16),
                              np.zeros((0, I, H), np.uint16), route_result=rr)
    zero = O.moe_layer_shared(tok.x_bits, tok.logits, tok.bias, wg, wu, wd,
                              np.zeros((2, H, I), np.uint16), np.zeros((2, H, I), np.uint16),
                              np.zeros((2, I, H), np.uint16), route_result=rr)
    assert np.array_equal(none, ref) and np.array_equal(zero, ref)


def test_two_shared_experts_add():
    T = 2
    tok = synth.make_tokens(T, 32)
    rr = O.route(tok.logits, tok.bias)
    wg, wu, wd = (np.zeros((128,) + shp, np.uint16) for shp in ((H, I), (H, I), (I, H)))
    sg, su, sd = synth.shared_weights_np(0, 0, 2)
    both = O.moe_layer_shared(tok.x_bits, tok.logits, tok.bias, wg, wu, wd, sg, su, sd,
                              route_result=rr)
    first = O.moe_layer_shared(tok.x_bits, tok.logits, tok.bias, wg, wu, wd, sg[:1], su[:1],
                               sd[:1], route_result=rr)
    x = O.bf16_bits_to_f64(tok.x_bits)
    second = O.expert_ffn(x, O.bf16_bits_to_f64(sg[1]), O.bf16_bits_to_f64(su[1]),
                          O.bf16_bits_to_f64(sd[1]))
    assert np.allclose(both - first, second, rtol=1e-12, atol=1e-14)
    assert np.abs(second).max() > 1e-3  # a real contribution
