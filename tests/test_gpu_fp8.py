"""GPU parity of the block-FP8 expert path (moe_pack_weights_fp8,
moe_dequant_fp8, moe_layer_fp8) against the float64 oracle.

With power-of-two block scales every dequantised weight is exactly a bf16
value (and, for W_down, an fp16 value), so the FP8 layer must return bit for
bit what the bf16 layer returns on the oracle's dequantised weights: the
in-shared-memory dequantisation of the small-batch kernel and the expansion
pass of larger batches add no rounding.  Scales are jittered by powers of two
per block so that a transposed or mis-indexed scale changes the result.  With
arbitrary fp32 scales ("amax" mode) each weight gains one rounding to the
operand type, and the layer is compared with the oracle's exact-scale layer
under the same rel-L2 bound as the bf16 layer."""
import functools

import numpy as np
import pytest
import torch

import oracle as O
from group_limited_routed_moe_b200 import synth
from gpu_helpers import DEV, REL_L2_TOL, W_TOL, to_dev_bf16, tokens_dev

pytestmark = pytest.mark.gpu
NAMES = (("g", synth.W_GATE), ("u", synth.W_UP), ("d", synth.W_DOWN))


def _moe():
    from group_limited_routed_moe_b200 import moe
    return moe


class Fp8Layer:
    """One layer's block-FP8 experts: codes and scales made on the device by
    the seeded generator, packed, and fetched to the host for the oracle."""

    def __init__(self, seed: int, layer: int, mode: str, jitter: bool):
        moe = _moe()
        self.q, self.s = {}, {}
        for name, which in NAMES:
            q, s = synth.fp8_weights_torch(seed, layer, which, DEV, mode)
            if jitter:
                s = s * torch.from_numpy(synth.fp8_scale_jitter(tuple(s.shape), 10 + which)).to(DEV)
            self.q[name], self.s[name] = q.contiguous(), s.contiguous()
        self.packed = moe.moe_pack_weights_fp8(self.q["g"], self.s["g"], self.q["u"], self.s["u"],
                                               self.q["d"], self.s["d"])
        torch.cuda.synchronize()

    def host(self, experts):
        """Full-size host codes and scales with the given experts filled in."""
        experts = np.unique(np.asarray(experts))
        sel = torch.as_tensor(experts, device=DEV)
        out = []
        for name, _ in NAMES:
            q = np.zeros((128,) + tuple(self.q[name].shape[1:]), np.uint8)
            s = np.ones((128,) + tuple(self.s[name].shape[1:]), np.float32)
            q[experts] = self.q[name][sel].cpu().numpy()
            s[experts] = self.s[name][sel].cpu().numpy()
            out += [q, s]
        return out

    def oracle(self, tok):
        rr = O.route(tok.logits, tok.bias)
        qg, sg, qu, su, qd, sd = self.host(rr.topk_idx)
        return O.moe_layer_fp8(tok.x_bits, tok.logits, tok.bias, qg, sg, qu, su, qd, sd,
                               route_result=rr), rr


@functools.lru_cache(maxsize=1)
def pow2_layer() -> Fp8Layer:
    return Fp8Layer(0, 0, "pow2", jitter=True)


@functools.lru_cache(maxsize=1)
def pow2_bf16_packed() -> torch.Tensor:
    """moe_pack_weights of the oracle's dequantised weights of pow2_layer()
    (exact bf16 values; the oracle dequantises on the host, expert by expert)."""
    moe = _moe()
    L = pow2_layer()
    dense = {}
    for name, _ in NAMES:
        shape = tuple(L.q[name].shape)
        dst = torch.empty(shape, dtype=torch.bfloat16, device=DEV)
        for e0 in range(0, 128, 16):
            q = L.q[name][e0:e0 + 16].cpu().numpy()
            s = L.s[name][e0:e0 + 16].cpu().numpy()
            w = O.dequant_block_fp8(q, s)
            bits = O.f64_to_bf16_bits(w)
            assert np.array_equal(O.bf16_bits_to_f64(bits), w)  # power-of-two scales: exact
            dst[e0:e0 + 16] = to_dev_bf16(bits)
        dense[name] = dst
    packed = moe.moe_pack_weights(dense["g"], dense["u"], dense["d"])
    torch.cuda.synchronize()
    return packed


def _status_ok():
    moe = _moe()
    assert moe.get_device_status(0) == moe.MOE_OK, moe.last_error()


def test_dequant_equals_bf16_pack_of_the_oracle_weights():
    """moe_dequant_fp8(moe_pack_weights_fp8(q, s)) is, byte for byte, the bf16
    pack of value(q) * s: codes transposed to the operand order with the right
    scale on every 128 x 128 block, gate/up interleaved, W_down in fp16."""
    moe = _moe()
    L = pow2_layer()
    ref = pow2_bf16_packed()
    got = moe.moe_dequant_fp8(L.packed)
    torch.cuda.synchronize()
    _status_ok()
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))


@pytest.mark.parametrize("T", [1, 5, 16, 33, 64, 77, 200, 256, 257, 1000])
def test_layer_fp8_equals_bf16_layer_bit_for_bit(T):
    """Up to 256 tokens: the FP8 skinny kernel (codes dequantised in shared
    memory); from 257: expansion pass + bf16 kernel.  Both must reproduce the
    bf16 layer on the dequantised weights exactly, including the residual."""
    moe = _moe()
    L = pow2_layer()
    ref_packed = pow2_bf16_packed()
    tok = synth.make_tokens(T, 300 + T)
    x, lg, bias = tokens_dev(tok)
    res = x if T in (16, 257) else None
    idx_a = torch.empty((T, 8), dtype=torch.int32, device=DEV)
    w_a = torch.empty((T, 8), dtype=torch.float32, device=DEV)
    idx_b, w_b = torch.empty_like(idx_a), torch.empty_like(w_a)
    out_a = moe.moe_layer_fp8(x, lg, bias, L.packed, residual=res, topk_idx_out=idx_a, topk_w_out=w_a)
    out_b = moe.moe_layer(x, lg, bias, ref_packed, residual=res, topk_idx_out=idx_b, topk_w_out=w_b)
    torch.cuda.synchronize()
    _status_ok()
    assert torch.equal(idx_a, idx_b)
    assert torch.equal(w_a.view(torch.int32), w_b.view(torch.int32))
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))


@pytest.mark.parametrize("T", [16, 256])
def test_layer_fp8_against_oracle(T):
    moe = _moe()
    L = pow2_layer()
    tok = synth.make_tokens(T, 400 + T)
    x, lg, bias = tokens_dev(tok)
    idx = torch.empty((T, 8), dtype=torch.int32, device=DEV)
    w = torch.empty((T, 8), dtype=torch.float32, device=DEV)
    out = moe.moe_layer_fp8(x, lg, bias, L.packed, topk_idx_out=idx, topk_w_out=w)
    torch.cuda.synchronize()
    _status_ok()
    ref, rr = L.oracle(tok)
    assert not ((rr.group_margin < 1e-12) | (rr.expert_margin < 1e-12)).any()
    assert np.array_equal(idx.cpu().numpy(), rr.topk_idx)
    assert np.abs(w.cpu().numpy() - rr.topk_w).max() <= W_TOL
    got = out.float().cpu().numpy().astype(np.float64)
    assert O.rel_l2(got, ref) <= REL_L2_TOL


@pytest.mark.parametrize("T", [16, 300])
def test_layer_fp8_arbitrary_scales_against_oracle(T):
    """fp32 scales max|w|/448 (not powers of two): one extra rounding per
    weight, compared with the oracle's exact value(code) * scale."""
    moe = _moe()
    L = Fp8Layer(0, 1, "amax", jitter=False)
    tok = synth.make_tokens(T, 500 + T)
    x, lg, bias = tokens_dev(tok)
    out = moe.moe_layer_fp8(x, lg, bias, L.packed)
    torch.cuda.synchronize()
    _status_ok()
    ref, _ = L.oracle(tok)
    got = out.float().cpu().numpy().astype(np.float64)
    assert O.rel_l2(got, ref) <= REL_L2_TOL


def test_pack_fp8_flags_down_weights_beyond_fp16():
    """A W_down block scale that puts a dequantised weight above 65504 sets
    the range status at pack time (the fp16 operand could not hold it)."""
    moe = _moe()
    L = pow2_layer()
    _status_ok()
    sd = L.s["d"].clone()
    sd[3, 1, 5] = 2.0 ** 10  # codes up to ~350 -> values up to ~3.6e5
    tmp = moe.moe_pack_weights_fp8(L.q["g"], L.s["g"], L.q["u"], L.s["u"], L.q["d"], sd)
    torch.cuda.synchronize()
    assert moe.get_device_status(0) == moe.MOE_ERR_RANGE
    _status_ok()  # read-and-clear
    del tmp


@pytest.mark.parametrize("T", [3, 16, 256, 300])
def test_expert_ffn_fp8_step_equals_bf16_step(T):
    """moe_expert_ffn_fp8 (the step call) against moe_expert_ffn on the
    oracle's dequantised weights: h and y_perm bit for bit."""
    moe = _moe()
    L = pow2_layer()
    ref_packed = pow2_bf16_packed()
    tok = synth.make_tokens(T, 600 + T)
    x, lg, bias = tokens_dev(tok)
    idx, w = moe.moe_route(lg, bias)
    counts, offsets, perm, inv = moe.moe_permute(idx)
    h8, y8 = moe.moe_expert_ffn_fp8(x, L.packed, offsets, perm)
    h16, y16 = moe.moe_expert_ffn(x, ref_packed, offsets, perm)
    torch.cuda.synchronize()
    _status_ok()
    assert torch.equal(h8.view(torch.int16), h16.view(torch.int16))
    assert torch.equal(y8.view(torch.int16), y16.view(torch.int16))


def test_pack_fp8_flags_nan_codes():
    """A NaN code (0x7F / 0xFF) in gate/up weights sets the range status at
    pack time: the integer dequantisation route would read it as a number."""
    moe = _moe()
    L = pow2_layer()
    _status_ok()
    qg = L.q["g"].clone()
    qg[7, 100, 33] = 0xFF
    tmp = moe.moe_pack_weights_fp8(qg, L.s["g"], L.q["u"], L.s["u"], L.q["d"], L.s["d"])
    torch.cuda.synchronize()
    assert moe.get_device_status(0) == moe.MOE_ERR_RANGE
    assert "NaN" in moe.last_error()
    _status_ok()
    del tmp
