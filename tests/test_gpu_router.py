"""GPU parity of the router projection (moe_router, moe_route_from_x,
moe_layer_routed) against the float64 oracle.

Two projections are checked: the tensor-core GEMM (moe_router, and the routed
layer above 8 tokens) and the one-launch router + routing + sort of up to 8
tokens (moe_route_from_x and the routed layer at decode), whose logits are
CUDA-core dot products in another summation order.

Logits are fp32 sums of 1536 exact bf16 x bf16 products, so they may differ
from the float64 value by the accumulation rounding: at most K * 2**-23 *
sum_k |x_k w_k| (rounding of every partial sum, toward or away from zero).
Routing decided on those logits equals the oracle's routing on its float64
logits for every token whose score margins exceed what that error can move;
the few tokens closer to a tie are reported, and the layer output is compared
on the others."""
import numpy as np
import pytest
import torch

import oracle as O
from group_limited_routed_moe_b200 import synth
from gpu_helpers import DEV, REL_L2_TOL, W_TOL, layer0_weights, to_dev_bf16, to_host_bits, tokens_dev

pytestmark = pytest.mark.gpu
K = 1536


def _moe():
    from group_limited_routed_moe_b200 import moe
    return moe


def _router(seed=0, layer=0):
    moe = _moe()
    w_bits = synth.router_weight_bits_np(seed, layer)
    packed = moe.moe_pack_router(to_dev_bf16(w_bits))
    return w_bits, packed


def _bound(x_bits, w_bits):
    return K * 2.0 ** -23 * (np.abs(O.bf16_bits_to_f64(x_bits)) @ np.abs(O.bf16_bits_to_f64(w_bits)))


@pytest.mark.parametrize("T", [1, 16, 63, 64, 65, 333, 8189])
def test_router_logits_parity(T):
    moe = _moe()
    w_bits, packed = _router()
    tok = synth.make_tokens(T, 40 + T)
    x = to_dev_bf16(tok.x_bits)
    pad = 5
    logits = torch.full((T + pad, 128), float("nan"), dtype=torch.float32, device=DEV)
    moe.moe_router(x, packed, logits[:T])
    torch.cuda.synchronize()
    assert moe.get_device_status(0) == moe.MOE_OK, moe.last_error()
    got = logits[:T].double().cpu().numpy()
    ref = O.router_logits(tok.x_bits, w_bits)
    assert np.all(np.abs(got - ref) <= _bound(tok.x_bits, w_bits))
    assert O.rel_l2(got, ref) <= 1e-5
    assert torch.isnan(logits[T:]).all()  # rows past T untouched


def test_router_one_hot_rows_exact():
    """x = e_k: every logit is one exact product, so row k of W_router comes
    back bit for bit (a transposed or mis-tiled operand would not)."""
    moe = _moe()
    w_bits, packed = _router(seed=1)
    ks = [0, 1, 63, 64, 777, 1535] * 12  # 72 tokens: two tiles, the second ragged
    x = np.zeros((len(ks), K), np.float32)
    for i, k in enumerate(ks):
        x[i, k] = 1.0
    logits = moe.moe_router(to_dev_bf16(synth.f32_to_bf16_bits(x)), packed)
    torch.cuda.synchronize()
    assert np.array_equal(logits.double().cpu().numpy(), O.bf16_bits_to_f64(w_bits)[ks])


@pytest.mark.parametrize("T", [1, 4, 7, 8, 9, 16, 64, 65, 333])
def test_route_from_x_parity(T):
    """Logits within the accumulation bound of the float64 product, and the
    routing equal, bit for bit, to moe_route on those same logits."""
    moe = _moe()
    w_bits, packed = _router(seed=2)
    tok = synth.make_tokens(T, 70 + T)
    x, _, bias = tokens_dev(tok)
    lg, idx, w = moe.moe_route_from_x(x, packed, bias)
    idx2, w2 = moe.moe_route(lg, bias)
    torch.cuda.synchronize()
    assert moe.get_device_status(0) == moe.MOE_OK, moe.last_error()
    got = lg.double().cpu().numpy()
    ref = O.router_logits(tok.x_bits, w_bits)
    assert np.all(np.abs(got - ref) <= _bound(tok.x_bits, w_bits))
    assert O.rel_l2(got, ref) <= 1e-5
    assert torch.equal(idx, idx2)
    assert torch.equal(w.view(torch.int32), w2.view(torch.int32))


def test_route_from_x_one_hot_rows_exact():
    """The one-launch projection of x = e_k returns row k of W_router bit for
    bit (one exact product per logit), for every token slot of an 8-token batch."""
    moe = _moe()
    w_bits, packed = _router(seed=1)
    ks = [0, 1, 63, 64, 777, 1535, 8, 1000]
    x = np.zeros((len(ks), K), np.float32)
    for i, k in enumerate(ks):
        x[i, k] = 1.0
    lg, _, _ = moe.moe_route_from_x(to_dev_bf16(synth.f32_to_bf16_bits(x)), packed, None)
    torch.cuda.synchronize()
    assert np.array_equal(lg.double().cpu().numpy(), O.bf16_bits_to_f64(w_bits)[ks])


@pytest.mark.parametrize("T", [1, 8, 16, 64, 333, 2048])
def test_layer_routed_equals_router_then_layer(T):
    moe = _moe()
    W = layer0_weights()
    _, packed = _router()
    tok = synth.make_tokens(T, 50 + T)
    x, _, bias = tokens_dev(tok)
    idx1 = torch.empty((T, 8), dtype=torch.int32, device=DEV)
    w1 = torch.empty((T, 8), dtype=torch.float32, device=DEV)
    out1 = moe.moe_layer_routed(x, packed, bias, W.packed, topk_idx_out=idx1, topk_w_out=w1)
    lg, _, _ = moe.moe_route_from_x(x, packed, bias)  # the same projection as the layer's
    idx2 = torch.empty_like(idx1)
    w2 = torch.empty_like(w1)
    out2 = moe.moe_layer(x, lg, bias, W.packed, topk_idx_out=idx2, topk_w_out=w2)
    torch.cuda.synchronize()
    assert moe.get_device_status(0) == moe.MOE_OK, moe.last_error()
    assert torch.equal(idx1, idx2)
    assert torch.equal(w1.view(torch.int32), w2.view(torch.int32))
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


@pytest.mark.parametrize("T", [1, 8, 16, 2048])
def test_layer_routed_against_oracle(T):
    """End to end from x: routing on the fp32 router logits against the
    oracle's routing on float64 logits, and the layer output on every token
    whose decision no logit error of that size could change."""
    moe = _moe()
    W = layer0_weights()
    w_bits, packed = _router()
    tok = synth.make_tokens(T, 60 + T)
    x, _, bias = tokens_dev(tok)
    idx = torch.empty((T, 8), dtype=torch.int32, device=DEV)
    wts = torch.empty((T, 8), dtype=torch.float32, device=DEV)
    out = moe.moe_layer_routed(x, packed, bias, W.packed, topk_idx_out=idx, topk_w_out=wts)
    torch.cuda.synchronize()
    assert moe.get_device_status(0) == moe.MOE_OK, moe.last_error()
    lg_ref = O.router_logits(tok.x_bits, w_bits)
    rr = O.route(lg_ref, tok.bias)
    # the logit error actually incurred (its size is checked against the
    # accumulation bound in test_router_logits_parity), with a margin of 4x
    lg_gpu = moe.moe_route_from_x(x, packed, bias)[0].double().cpu().numpy()
    err = np.abs(lg_gpu - lg_ref)
    assert np.all(err <= _bound(tok.x_bits, w_bits))
    delta = 4 * err.max(axis=1) + 1e-12  # per token, on any logit
    # a logit error d moves a score s = sigmoid(z) by at most d/4, a group score by d/2
    # and a score difference by twice that
    close = (rr.group_margin <= 2 * delta) | (rr.expert_margin <= delta)
    assert close.mean() <= 0.01, f"{close.sum()} of {T} tokens within the logit error of a tie"
    keep = ~close
    gi, gw = idx.cpu().numpy()[keep], wts.cpu().numpy()[keep]
    oi, ow = rr.topk_idx[keep], rr.topk_w[keep]
    # the chosen set, and each chosen expert's weight (sigmoid of an fp32 vs a
    # float64 logit, renormalised), match on every kept token
    sg, so = np.argsort(gi, axis=1), np.argsort(oi, axis=1)
    assert np.array_equal(np.take_along_axis(gi, sg, 1), np.take_along_axis(oi, so, 1))
    assert np.abs(np.take_along_axis(gw, sg, 1) - np.take_along_axis(ow, so, 1)).max() \
        <= W_TOL + delta.max() / 2
    # the slot order (descending score) matches wherever adjacent chosen scores
    # are further apart than the error can close
    z = lg_ref[keep] + tok.bias[None, :]
    s_sel = np.take_along_axis(O.sigmoid(z), oi, 1)
    strict = ((s_sel[:, :-1] - s_sel[:, 1:]) > delta[keep, None] / 2).all(axis=1)
    assert np.array_equal(gi[strict], oi[strict])
    assert strict.mean() > 0.9
    rows = np.nonzero(keep)[0]
    wg, wu, wd = W.host(rr.topk_idx[rows])
    sub = O.RouteResult(rr.topk_idx[rows], rr.topk_w[rows], rr.kept_groups[rows],
                        rr.group_margin[rows], rr.expert_margin[rows])
    ref = O.moe_layer(tok.x_bits[rows], lg_ref[rows], tok.bias, wg, wu, wd, route_result=sub)
    got = O.bf16_bits_to_f64(to_host_bits(out))[rows]
    assert O.rel_l2(got, ref) <= REL_L2_TOL
