"""Pins of the oracle's router projection (logits = x W_router) against
results fixed by arithmetic alone, so that a transposed operand, a dropped
row or a wrong scale fails a test."""
import numpy as np

import oracle as O
from group_limited_routed_moe_b200 import synth


def _bf16(a):
    return synth.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def test_one_hot_rows_pick_router_rows():
    """x = e_k gives row k of W_router [1536, 128] exactly (not column k)."""
    w = synth.router_weight_bits_np(0, 0)
    ks = [0, 1, 511, 1535]
    x = np.zeros((len(ks), 1536), np.float32)
    for i, k in enumerate(ks):
        x[i, k] = 1.0
    got = O.router_logits(_bf16(x), w)
    assert got.shape == (len(ks), 128)
    assert np.array_equal(got, O.bf16_bits_to_f64(w)[ks])


def test_all_ones_row_gives_column_sums_of_small_integers():
    """Small-integer weights and x = 1: every product and sum is exact, so the
    logits are the weights' column sums (computed here with np.sum)."""
    rng = np.random.default_rng(3)
    wi = rng.integers(-8, 9, size=(1536, 128)).astype(np.float32)
    x = np.ones((2, 1536), np.float32)
    x[1] *= -2.0
    got = O.router_logits(_bf16(x), _bf16(wi))
    assert np.array_equal(got[0], wi.sum(axis=0).astype(np.float64))
    assert np.array_equal(got[1], -2.0 * wi.sum(axis=0).astype(np.float64))


def test_linear_in_x_exactly_for_exact_inputs():
    """Small-integer x and W: router(x1 + x2) == router(x1) + router(x2) and
    router(2 x) == 2 router(x), both exactly."""
    rng = np.random.default_rng(4)
    wi = rng.integers(-4, 5, size=(1536, 128)).astype(np.float32)
    x1 = rng.integers(-3, 4, size=(3, 1536)).astype(np.float32)
    x2 = rng.integers(-3, 4, size=(3, 1536)).astype(np.float32)
    w = _bf16(wi)
    r1, r2 = O.router_logits(_bf16(x1), w), O.router_logits(_bf16(x2), w)
    assert np.array_equal(O.router_logits(_bf16(x1 + x2), w), r1 + r2)
    assert np.array_equal(O.router_logits(_bf16(2 * x1), w), 2 * r1)


def test_router_weights_generator_shape_and_scale():
    w = O.bf16_bits_to_f64(synth.router_weight_bits_np(0, 0))
    assert w.shape == (1536, 128)
    assert abs(w.std() - 0.02) < 0.001 and abs(w.mean()) < 0.001
    assert not np.array_equal(synth.router_weight_bits_np(0, 0), synth.router_weight_bits_np(0, 1))
