"""moe_layer's fused launches for small batches against the separate step
kernels (moe_route, moe_permute, moe_expert_gate_up, moe_expert_down,
moe_combine) and the float64 oracle: route + permute in one block for T <= 64
(a warp per token, counting sort from shared memory), and gate/up and down in
one persistent launch for T <= 256.

The fused kernel must reproduce the step kernels exactly: same expert ids, the
same fp32 weights bit for bit, the same permutation, hence a bit-identical
layer output.  T = 65 and T = 257 are the first batches past each fused path."""
import numpy as np
import pytest
import torch

import oracle as O
from group_limited_routed_moe_b200 import synth
from gpu_helpers import (DEV, REL_L2_TOL, W_TOL, extreme_logits, layer0_weights, oracle_layer,
                         to_dev_bf16, tokens_dev)

pytestmark = pytest.mark.gpu


def _moe():
    from group_limited_routed_moe_b200 import moe
    return moe


def _layer(x, lg, bias, W):
    moe = _moe()
    T = x.shape[0]
    idx = torch.full((T, 8), -1, dtype=torch.int32, device=DEV)
    w = torch.full((T, 8), float("nan"), dtype=torch.float32, device=DEV)
    out = moe.moe_layer(x, lg, bias, W.packed, topk_idx_out=idx, topk_w_out=w)
    return idx, w, out


def _steps(x, lg, bias, W):
    moe = _moe()
    idx, w = moe.moe_route(lg, bias)
    counts, offsets, perm, inv = moe.moe_permute(idx)
    h = moe.moe_expert_gate_up(x, W.packed, offsets, perm)
    y = moe.moe_expert_down(h, W.packed, offsets)
    out = moe.moe_combine(y, w, inv)
    return idx, w, out


def _same_bits(a, b):
    return torch.equal(a.contiguous().view(torch.int16 if a.element_size() == 2 else torch.int32),
                       b.contiguous().view(torch.int16 if b.element_size() == 2 else torch.int32))


@pytest.mark.parametrize("T", [1, 2, 16, 31, 32, 33, 64, 65, 128, 256, 257])
def test_fused_small_layer_equals_steps_and_oracle(T):
    moe = _moe()
    W = layer0_weights()
    tok = synth.make_tokens(T, 100 + T)
    x, lg, bias = tokens_dev(tok)
    idx_l, w_l, out_l = _layer(x, lg, bias, W)
    idx_s, w_s, out_s = _steps(x, lg, bias, W)
    torch.cuda.synchronize()
    assert moe.get_device_status(0) == moe.MOE_OK, moe.last_error()
    assert torch.equal(idx_l, idx_s)
    assert _same_bits(w_l, w_s)
    assert _same_bits(out_l, out_s)
    ref, rr = oracle_layer(tok, W)
    assert not ((rr.group_margin < 1e-12) | (rr.expert_margin < 1e-12)).any()
    assert np.array_equal(idx_l.cpu().numpy(), rr.topk_idx)
    assert np.abs(w_l.cpu().numpy() - rr.topk_w).max() <= W_TOL
    got = out_l.float().cpu().numpy().astype(np.float64)
    assert O.rel_l2(got, ref) <= REL_L2_TOL


def test_fused_small_extreme_logits():
    """Saturated, underflowed and all-tied tokens: ids and weights as the
    oracle decides them (deliberate exact ties compare exactly), and the same
    bits as the step kernels."""
    moe = _moe()
    W = layer0_weights()
    lg_np, b_np = extreme_logits()
    T = lg_np.shape[0]
    x = to_dev_bf16(synth.make_tokens(T, 5).x_bits)
    lg = torch.from_numpy(lg_np).to(DEV)
    for bias_np in (None, b_np):
        bias = None if bias_np is None else torch.from_numpy(bias_np).to(DEV)
        idx_l, w_l, out_l = _layer(x, lg, bias, W)
        idx_s, w_s, out_s = _steps(x, lg, bias, W)
        torch.cuda.synchronize()
        assert moe.get_device_status(0) == moe.MOE_OK, moe.last_error()
        rr = O.route(lg_np, bias_np)
        assert np.array_equal(idx_l.cpu().numpy(), rr.topk_idx)
        gw = w_l.cpu().numpy()
        assert np.all(np.isfinite(gw))
        assert np.abs(gw - rr.topk_w).max() <= W_TOL
        assert torch.equal(idx_l, idx_s)
        assert _same_bits(w_l, w_s)
        assert _same_bits(out_l, out_s)
