"""GPU parity of the shared-expert layer (moe_pack_shared, moe_layer_shared)
against the float64 oracle, and its consistency with the routed-only layers.

The shared experts' rows go through the same grouped expert-FFN kernels as the
routed experts (one row per token and shared expert), so the tests cover the
skinny path (T <= 256) and the wide path (T > 256), one and two shared
experts, the residual, and block-FP8 routed experts beside bf16 shared ones."""
import functools

import numpy as np
import pytest
import torch

import oracle as O
from group_limited_routed_moe_b200 import synth
from gpu_helpers import DEV, REL_L2_TOL, W_TOL, layer0_weights, to_dev_bf16, tokens_dev

pytestmark = pytest.mark.gpu


def _moe():
    from group_limited_routed_moe_b200 import moe
    return moe


@functools.lru_cache(maxsize=2)
def shared_pack(n_shared: int):
    """Host bits (W_gate, W_up, W_down) of n_shared shared experts, and their pack."""
    moe = _moe()
    bits = synth.shared_weights_np(0, 0, n_shared)
    packed = moe.moe_pack_shared(*(to_dev_bf16(b) for b in bits))
    torch.cuda.synchronize()
    return bits, packed


def _oracle(tok, W, bits, rows=None):
    x, lg = tok.x_bits, tok.logits
    if rows is not None:
        x, lg = x[rows], lg[rows]
    rr = O.route(lg, tok.bias)
    wg, wu, wd = W.host(rr.topk_idx)
    return O.moe_layer_shared(x, lg, tok.bias, wg, wu, wd, *bits, route_result=rr), rr


def _status_ok():
    moe = _moe()
    assert moe.get_device_status(0) == moe.MOE_OK, moe.last_error()


@pytest.mark.parametrize("T,n_shared", [(1, 1), (16, 2), (77, 1), (256, 2), (300, 2), (1000, 1)])
def test_shared_layer_against_oracle(T, n_shared):
    moe = _moe()
    W = layer0_weights()
    bits, packed = shared_pack(n_shared)
    tok = synth.make_tokens(T, 700 + T)
    x, lg, bias = tokens_dev(tok)
    idx = torch.empty((T, 8), dtype=torch.int32, device=DEV)
    w = torch.empty((T, 8), dtype=torch.float32, device=DEV)
    out = moe.moe_layer_shared(x, lg, bias, packed, n_shared, packed_w=W.packed,
                               topk_idx_out=idx, topk_w_out=w)
    torch.cuda.synchronize()
    _status_ok()
    rows = None if T <= 300 else np.sort(np.random.default_rng(T).choice(T, 96, replace=False))
    ref, rr = _oracle(tok, W, bits, rows)
    gi, gw, got = idx.cpu().numpy(), w.cpu().numpy(), out.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        gi, gw, got = gi[rows], gw[rows], got[rows]
    assert not ((rr.group_margin < 1e-12) | (rr.expert_margin < 1e-12)).any()
    assert np.array_equal(gi, rr.topk_idx)
    assert np.abs(gw - rr.topk_w).max() <= W_TOL
    assert O.rel_l2(got, ref) <= REL_L2_TOL


@pytest.mark.parametrize("T", [16, 300])
def test_zero_shared_experts_equal_the_routed_layer(T):
    """All-zero shared weights add exact zeros in the fp32 sum, so the layer is
    moe_layer bit for bit, with and without a residual."""
    moe = _moe()
    W = layer0_weights()
    z = torch.zeros((2, 1536, 512), dtype=torch.bfloat16, device=DEV)
    zd = torch.zeros((2, 512, 1536), dtype=torch.bfloat16, device=DEV)
    packed0 = moe.moe_pack_shared(z, z, zd)
    tok = synth.make_tokens(T, 800 + T)
    x, lg, bias = tokens_dev(tok)
    for res in (None, x):
        a = moe.moe_layer_shared(x, lg, bias, packed0, 2, packed_w=W.packed, residual=res)
        b = moe.moe_layer(x, lg, bias, W.packed, residual=res)
        torch.cuda.synchronize()
        _status_ok()
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_shared_layer_residual_and_no_shared():
    """residual = x, and n_shared = 0 (moe_layer_shared = moe_layer)."""
    moe = _moe()
    W = layer0_weights()
    bits, packed = shared_pack(1)
    T = 40
    tok = synth.make_tokens(T, 901)
    x, lg, bias = tokens_dev(tok)
    out = moe.moe_layer_shared(x, lg, bias, packed, 1, packed_w=W.packed, residual=x)
    none = moe.moe_layer_shared(x, lg, bias, packed, 0, packed_w=W.packed)
    plain = moe.moe_layer(x, lg, bias, W.packed)
    torch.cuda.synchronize()
    _status_ok()
    assert torch.equal(none.view(torch.int16), plain.view(torch.int16))
    ref, _ = _oracle(tok, W, bits)
    ref = ref + O.bf16_bits_to_f64(tok.x_bits)
    assert O.rel_l2(out.float().cpu().numpy().astype(np.float64), ref) <= REL_L2_TOL


@pytest.mark.parametrize("T", [16, 300])
def test_shared_with_fp8_routed_experts(T):
    """Block-FP8 routed experts (power-of-two scales) with bf16 shared experts:
    bit for bit the layer with the bf16 pack of the dequantised routed weights."""
    from test_gpu_fp8 import pow2_bf16_packed, pow2_layer
    moe = _moe()
    L8 = pow2_layer()
    ref_packed = pow2_bf16_packed()
    bits, packed = shared_pack(2)
    tok = synth.make_tokens(T, 950 + T)
    x, lg, bias = tokens_dev(tok)
    a = moe.moe_layer_shared(x, lg, bias, packed, 2, packed_fp8=L8.packed)
    b = moe.moe_layer_shared(x, lg, bias, packed, 2, packed_w=ref_packed)
    torch.cuda.synchronize()
    _status_ok()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("T", [16, 300])
def test_shared_with_nvfp4_routed_experts(T):
    """NVFP4 routed experts (power-of-two tensor scales) with bf16 shared
    experts: bit for bit the layer with the bf16 pack of the dequantised routed
    weights; with no shared expert, bit for bit moe_layer_nvfp4."""
    from test_gpu_nvfp4 import pow2_bf16_packed as nv_bf16_packed
    from test_gpu_nvfp4 import pow2_layer as nv_layer
    moe = _moe()
    L4 = nv_layer()
    ref_packed = nv_bf16_packed()
    bits, packed = shared_pack(2)
    tok = synth.make_tokens(T, 1150 + T)
    x, lg, bias = tokens_dev(tok)
    a = moe.moe_layer_shared(x, lg, bias, packed, 2, packed_nvfp4=L4.packed, residual=x)
    b = moe.moe_layer_shared(x, lg, bias, packed, 2, packed_w=ref_packed, residual=x)
    c = moe.moe_layer_shared(x, lg, bias, packed, 0, packed_nvfp4=L4.packed)
    d = moe.moe_layer_nvfp4(x, lg, bias, L4.packed)
    torch.cuda.synchronize()
    _status_ok()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(c.view(torch.int16), d.view(torch.int16))
