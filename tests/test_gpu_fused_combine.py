"""The combine that the single-launch expert FFN runs itself for a single
token (the last CTA to retire writes the layer's output; no combine launch).

It must give what the separate combine gives, bit for bit: the same fp32 sum
in slot order, then the shared rows and the residual, rounded once.  Checked
two ways:
- against the step calls (moe_route, moe_permute, moe_expert_ffn[_fp8 |
  _nvfp4], moe_combine), which never fuse;
- against the rows of a three-token layer call, which does not fuse either
  (every token of the layer is independent, so rows agree bit for bit), for
  the routed, shared-expert and quantised layers, with and without an
  in-place residual.
Both orders of calls are repeated so that a counter left non-zero by the fused
path would show up as a wrong or timed-out next call."""
import numpy as np
import pytest
import torch

import oracle as O
from group_limited_routed_moe_b200 import synth
from gpu_helpers import DEV, REL_L2_TOL, layer0_weights, oracle_layer, to_dev_bf16, to_host_bits, tokens_dev

pytestmark = pytest.mark.gpu


def _moe():
    from group_limited_routed_moe_b200 import moe
    return moe


def _status_ok():
    moe = _moe()
    assert moe.get_device_status(0) == moe.MOE_OK, moe.last_error()


def _bits(t):
    return t.view(torch.int16)


@pytest.mark.parametrize("T", [1, 2, 3])
@pytest.mark.parametrize("with_residual", [False, True])
def test_layer_equals_step_calls(T, with_residual):
    moe = _moe()
    W = layer0_weights()
    tok = synth.make_tokens(T, 1300 + T)
    x, lg, bias = tokens_dev(tok)
    res = to_dev_bf16(synth.make_tokens(T, 1400 + T).x_bits) if with_residual else None
    for _ in range(2):
        idx, w = moe.moe_route(lg, bias)
        counts, offsets, perm, inv = moe.moe_permute(idx)
        _, y = moe.moe_expert_ffn(x, W.packed, offsets, perm)
        ref = moe.moe_combine(y, w, inv, residual=res)
        if with_residual:
            got = res.clone()
            moe.moe_layer(x, lg, bias, W.packed, residual=got, out=got)
        else:
            got = moe.moe_layer(x, lg, bias, W.packed)
        torch.cuda.synchronize()
        _status_ok()
        assert torch.equal(_bits(got), _bits(ref))


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
@pytest.mark.parametrize("T", [1, 2])
def test_quantised_layer_equals_step_calls(fmt, T):
    moe = _moe()
    if fmt == "fp8":
        from test_gpu_fp8 import pow2_layer
        packed, ffn, layer = pow2_layer().packed, moe.moe_expert_ffn_fp8, moe.moe_layer_fp8
    else:
        from test_gpu_nvfp4 import pow2_layer
        packed, ffn, layer = pow2_layer().packed, moe.moe_expert_ffn_nvfp4, moe.moe_layer_nvfp4
    tok = synth.make_tokens(T, 1500 + T)
    x, lg, bias = tokens_dev(tok)
    res = to_dev_bf16(synth.make_tokens(T, 1600 + T).x_bits)
    idx, w = moe.moe_route(lg, bias)
    counts, offsets, perm, inv = moe.moe_permute(idx)
    _, y = ffn(x, packed, offsets, perm)
    ref = moe.moe_combine(y, w, inv, residual=res)
    for _ in range(2):
        got = res.clone()
        layer(x, lg, bias, packed, residual=got, out=got)
        torch.cuda.synchronize()
        _status_ok()
        assert torch.equal(_bits(got), _bits(ref))


def _layer_call(kind, x, lg, bias, residual):
    """One layer call of the given kind on x (T rows), in place on a copy of
    residual when one is given."""
    moe = _moe()
    W = layer0_weights()
    out = residual.clone() if residual is not None else None
    if kind == "routed":
        return moe.moe_layer(x, lg, bias, W.packed, residual=out, out=out)
    if kind.startswith("shared"):
        from test_gpu_shared import shared_pack
        n = int(kind[-1])
        _, sp = shared_pack(n)
        return moe.moe_layer_shared(x, lg, bias, sp, n, packed_w=W.packed, residual=out, out=out)
    if kind == "fp8":
        from test_gpu_fp8 import pow2_layer
        return moe.moe_layer_fp8(x, lg, bias, pow2_layer().packed, residual=out, out=out)
    if kind == "nvfp4":
        from test_gpu_nvfp4 import pow2_layer
        return moe.moe_layer_nvfp4(x, lg, bias, pow2_layer().packed, residual=out, out=out)
    if kind == "fp8_shared1":
        from test_gpu_fp8 import pow2_layer
        from test_gpu_shared import shared_pack
        _, sp = shared_pack(1)
        return moe.moe_layer_shared(x, lg, bias, sp, 1, packed_fp8=pow2_layer().packed,
                                    residual=out, out=out)
    raise ValueError(kind)


@pytest.mark.parametrize("kind", ["routed", "shared1", "shared2", "fp8", "nvfp4", "fp8_shared1"])
@pytest.mark.parametrize("with_residual", [False, True])
def test_fused_rows_equal_unfused_batch(kind, with_residual):
    """Tokens 0..T-1 of a T = 3 call (separate combine launch) against T = 1
    calls (combine inside the FFN launch) and T = 2 calls, bit for bit."""
    tok = synth.make_tokens(3, 1700)
    x, lg, bias = tokens_dev(tok)
    res = to_dev_bf16(synth.make_tokens(3, 1701).x_bits) if with_residual else None
    full = _layer_call(kind, x, lg, bias, res)
    for T in (1, 2, 1):
        got = _layer_call(kind, x[:T].contiguous(), lg[:T].contiguous(), bias,
                          res[:T].contiguous() if res is not None else None)
        torch.cuda.synchronize()
        _status_ok()
        assert torch.equal(_bits(got), _bits(full[:T])), (kind, T)


@pytest.mark.parametrize("T", [1, 2])
def test_routed_from_x_equals_step_calls(T):
    """moe_layer_routed (router, routing and sort in one launch, then the FFN,
    with the combine inside at T = 1) against moe_route_from_x and the step
    calls."""
    from test_gpu_router import _router
    moe = _moe()
    W = layer0_weights()
    _, pr = _router()
    tok = synth.make_tokens(T, 1800 + T)
    x, _, bias = tokens_dev(tok)
    _, idx, w = moe.moe_route_from_x(x, pr, bias)
    counts, offsets, perm, inv = moe.moe_permute(idx)
    _, y = moe.moe_expert_ffn(x, W.packed, offsets, perm)
    ref = moe.moe_combine(y, w, inv)
    for _ in range(2):
        got = moe.moe_layer_routed(x, pr, bias, W.packed)
        torch.cuda.synchronize()
        _status_ok()
        assert torch.equal(_bits(got), _bits(ref))


@pytest.mark.parametrize("T", [1, 2])
def test_fused_layer_against_oracle(T):
    """The fused path's output against the float64 oracle (rel-L2 bound of the
    layer tests) and routing ids bit-exact."""
    moe = _moe()
    W = layer0_weights()
    tok = synth.make_tokens(T, 1900 + T)
    x, lg, bias = tokens_dev(tok)
    idx = torch.empty((T, 8), dtype=torch.int32, device=DEV)
    w = torch.empty((T, 8), dtype=torch.float32, device=DEV)
    out = moe.moe_layer(x, lg, bias, W.packed, topk_idx_out=idx, topk_w_out=w)
    torch.cuda.synchronize()
    _status_ok()
    ref, rr = oracle_layer(tok, W)
    assert np.array_equal(idx.cpu().numpy(), rr.topk_idx)
    err = O.rel_l2(O.bf16_bits_to_f64(to_host_bits(out)), ref)
    assert err <= REL_L2_TOL, f"T={T}: rel-L2 {err:.3e}"
