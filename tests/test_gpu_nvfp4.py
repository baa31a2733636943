"""GPU parity of the NVFP4 expert path (moe_pack_weights_nvfp4,
moe_dequant_nvfp4, moe_expert_ffn_nvfp4, moe_layer_nvfp4) against the float64
oracle.

With power-of-two tensor scales every dequantised weight is exactly a bf16
value (and, for W_down, an fp16 value), so the NVFP4 layer must return bit for
bit what the bf16 layer returns on the oracle's dequantised weights: the
dequantisation into tensor memory of the small-batch kernel and the expansion
pass of larger batches add no rounding.  The synthetic block scales differ
from block to block of 16 (each comes from its block's largest weight), so a
transposed or mis-indexed scale changes the result.  With fp32 tensor scales
that are not powers of two ("amax" mode) the block multiplier is rounded once,
and the layer is compared with the oracle's exact layer under the same rel-L2
bound as the bf16 layer."""
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


class Nvfp4Layer:
    """One layer's NVFP4 experts ([out, in] form): codes and scales made on the
    device by the seeded generator, packed, and fetched to the host for the
    oracle."""

    def __init__(self, seed: int, layer: int, mode: str):
        moe = _moe()
        self.q, self.s, self.g = {}, {}, {}
        for name, which in NAMES:
            q, s, g = synth.nvfp4_weights_torch(seed, layer, which, DEV, mode)
            self.q[name], self.s[name], self.g[name] = q.contiguous(), s.contiguous(), g.contiguous()
        self.packed = self.pack()
        torch.cuda.synchronize()

    def pack(self, **override):
        moe = _moe()
        a = {f"{k}{n}": getattr(self, k)[n] for k in "qsg" for n in "gud"}
        a.update(override)
        return moe.moe_pack_weights_nvfp4(a["qg"], a["sg"], a["gg"], a["qu"], a["su"], a["gu"],
                                          a["qd"], a["sd"], a["gd"])

    def host(self, experts):
        """Full-size host codes, block scales and tensor scales with the given
        experts filled in."""
        experts = np.unique(np.asarray(experts))
        sel = torch.as_tensor(experts, device=DEV)
        out = []
        for name, _ in NAMES:
            q = np.zeros((128,) + tuple(self.q[name].shape[1:]), np.uint8)
            s = np.full((128,) + tuple(self.s[name].shape[1:]), 0x38, np.uint8)
            g = np.ones(128, np.float32)
            q[experts] = self.q[name][sel].cpu().numpy()
            s[experts] = self.s[name][sel].cpu().numpy()
            g[experts] = self.g[name][sel].cpu().numpy()
            out += [q, s, g]
        return out

    def oracle(self, tok):
        rr = O.route(tok.logits, tok.bias)
        return O.moe_layer_nvfp4(tok.x_bits, tok.logits, tok.bias, *self.host(rr.topk_idx),
                                 route_result=rr), rr


@functools.lru_cache(maxsize=1)
def pow2_layer() -> Nvfp4Layer:
    return Nvfp4Layer(0, 0, "pow2")


@functools.lru_cache(maxsize=1)
def pow2_bf16_packed() -> torch.Tensor:
    """moe_pack_weights of the oracle's dequantised weights of pow2_layer()
    (exact bf16 values, transposed to the x W form; the oracle dequantises on
    the host, 16 experts at a time)."""
    moe = _moe()
    L = pow2_layer()
    dense = {}
    for name, _ in NAMES:
        n_out, n_in2 = L.q[name].shape[1:]
        dst = torch.empty((128, 2 * n_in2, n_out), dtype=torch.bfloat16, device=DEV)
        for e0 in range(0, 128, 16):
            w = O.dequant_nvfp4(L.q[name][e0:e0 + 16].cpu().numpy(),
                                L.s[name][e0:e0 + 16].cpu().numpy(),
                                L.g[name][e0:e0 + 16].cpu().numpy())
            bits = O.f64_to_bf16_bits(w)
            assert np.array_equal(O.bf16_bits_to_f64(bits), w)  # power-of-two tensor scales
            dst[e0:e0 + 16] = to_dev_bf16(np.ascontiguousarray(bits.transpose(0, 2, 1)))
        dense[name] = dst
    packed = moe.moe_pack_weights(dense["g"], dense["u"], dense["d"])
    torch.cuda.synchronize()
    return packed


def _status_ok():
    moe = _moe()
    assert moe.get_device_status(0) == moe.MOE_OK, moe.last_error()


def test_dequant_equals_bf16_pack_of_the_oracle_weights():
    """moe_dequant_nvfp4(moe_pack_weights_nvfp4(...)) is, byte for byte, the
    bf16 pack of value(code) * value(block scale) * tensor scale: codes in the
    operand order, the right multiplier on every block of 16, gate/up
    interleaved, W_down in fp16."""
    moe = _moe()
    L = pow2_layer()
    ref = pow2_bf16_packed()
    got = moe.moe_dequant_nvfp4(L.packed)
    torch.cuda.synchronize()
    _status_ok()
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))


@pytest.mark.parametrize("T", [1, 5, 16, 33, 64, 77, 200, 256, 257, 1000])
def test_layer_nvfp4_equals_bf16_layer_bit_for_bit(T):
    """Up to 256 tokens: the NVFP4 skinny kernel (codes dequantised into tensor
    memory); from 257: expansion pass + bf16 kernel.  Both must reproduce the
    bf16 layer on the dequantised weights exactly, including the residual."""
    moe = _moe()
    L = pow2_layer()
    ref_packed = pow2_bf16_packed()
    tok = synth.make_tokens(T, 700 + T)
    x, lg, bias = tokens_dev(tok)
    res = x if T in (16, 257) else None
    idx_a = torch.empty((T, 8), dtype=torch.int32, device=DEV)
    w_a = torch.empty((T, 8), dtype=torch.float32, device=DEV)
    idx_b, w_b = torch.empty_like(idx_a), torch.empty_like(w_a)
    out_a = moe.moe_layer_nvfp4(x, lg, bias, L.packed, residual=res, topk_idx_out=idx_a,
                                topk_w_out=w_a)
    out_b = moe.moe_layer(x, lg, bias, ref_packed, residual=res, topk_idx_out=idx_b,
                          topk_w_out=w_b)
    torch.cuda.synchronize()
    _status_ok()
    assert torch.equal(idx_a, idx_b)
    assert torch.equal(w_a.view(torch.int32), w_b.view(torch.int32))
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))


@pytest.mark.parametrize("T", [16, 256])
def test_layer_nvfp4_against_oracle(T):
    moe = _moe()
    L = pow2_layer()
    tok = synth.make_tokens(T, 800 + T)
    x, lg, bias = tokens_dev(tok)
    idx = torch.empty((T, 8), dtype=torch.int32, device=DEV)
    w = torch.empty((T, 8), dtype=torch.float32, device=DEV)
    out = moe.moe_layer_nvfp4(x, lg, bias, L.packed, topk_idx_out=idx, topk_w_out=w)
    torch.cuda.synchronize()
    _status_ok()
    ref, rr = L.oracle(tok)
    assert not ((rr.group_margin < 1e-12) | (rr.expert_margin < 1e-12)).any()
    assert np.array_equal(idx.cpu().numpy(), rr.topk_idx)
    assert np.abs(w.cpu().numpy() - rr.topk_w).max() <= W_TOL
    got = out.float().cpu().numpy().astype(np.float64)
    assert O.rel_l2(got, ref) <= REL_L2_TOL


@pytest.mark.parametrize("T", [16, 300])
def test_layer_nvfp4_arbitrary_tensor_scales_against_oracle(T):
    """fp32 tensor scales max|w| / (6 * 448) (not powers of two): the block
    multiplier is rounded to the operand type once; compared with the oracle's
    exact value(code) * value(block scale) * tensor scale."""
    moe = _moe()
    L = Nvfp4Layer(0, 1, "amax")
    tok = synth.make_tokens(T, 900 + T)
    x, lg, bias = tokens_dev(tok)
    out = moe.moe_layer_nvfp4(x, lg, bias, L.packed)
    torch.cuda.synchronize()
    _status_ok()
    ref, _ = L.oracle(tok)
    got = out.float().cpu().numpy().astype(np.float64)
    assert O.rel_l2(got, ref) <= REL_L2_TOL


@pytest.mark.parametrize("T", [3, 16, 256, 300])
def test_expert_ffn_nvfp4_step_equals_bf16_step(T):
    """moe_expert_ffn_nvfp4 (the step call) against moe_expert_ffn on the
    oracle's dequantised weights: h and y_perm bit for bit."""
    moe = _moe()
    L = pow2_layer()
    ref_packed = pow2_bf16_packed()
    tok = synth.make_tokens(T, 1000 + T)
    x, lg, bias = tokens_dev(tok)
    idx, w = moe.moe_route(lg, bias)
    counts, offsets, perm, inv = moe.moe_permute(idx)
    h4, y4 = moe.moe_expert_ffn_nvfp4(x, L.packed, offsets, perm)
    h16, y16 = moe.moe_expert_ffn(x, ref_packed, offsets, perm)
    torch.cuda.synchronize()
    _status_ok()
    assert torch.equal(h4.view(torch.int16), h16.view(torch.int16))
    assert torch.equal(y4.view(torch.int16), y16.view(torch.int16))


def test_expert_ffn_nvfp4_forced_experts():
    """Every token of a small batch forced onto the same 8 experts: 200 rows per
    expert, seven 32-token chunks with a ragged last one, through the NVFP4
    skinny kernel; bit for bit against the bf16 step on the dequantised weights."""
    moe = _moe()
    L = pow2_layer()
    ref_packed = pow2_bf16_packed()
    tok = synth.make_tokens(200, 1201)
    tok.bias[:] = 0
    tok.bias[[1, 2, 30, 31, 60, 61, 100, 127]] = 1000.0
    x, lg, bias = tokens_dev(tok)
    idx, w = moe.moe_route(lg, bias)
    counts, offsets, perm, inv = moe.moe_permute(idx)
    assert int(counts.max()) == 200
    h4, y4 = moe.moe_expert_ffn_nvfp4(x, L.packed, offsets, perm)
    h16, y16 = moe.moe_expert_ffn(x, ref_packed, offsets, perm)
    torch.cuda.synchronize()
    _status_ok()
    assert torch.equal(h4.view(torch.int16), h16.view(torch.int16))
    assert torch.equal(y4.view(torch.int16), y16.view(torch.int16))


def test_pack_nvfp4_flags_bad_scales():
    """A NaN block-scale code, a non-finite tensor scale, and a W_down block
    whose multiplier leaves the fp16 range each set the range status at pack
    time (read and cleared by moe_get_device_status)."""
    moe = _moe()
    L = pow2_layer()
    _status_ok()
    sg = L.s["g"].clone()
    sg[5, 10, 3] = 0x7F
    gd = L.g["d"].clone()
    gd[9] = float("inf")
    gu = L.g["u"].clone()
    gu[2] = 2.0 ** 20  # W_up multipliers of expert 2 overflow bf16
    for override in ({"sg": sg}, {"gd": gd}, {"gu": gu}):
        tmp = L.pack(**override)
        torch.cuda.synchronize()
        assert moe.get_device_status(0) == moe.MOE_ERR_RANGE, override.keys()
        assert "NVFP4" in moe.last_error()
        _status_ok()
        del tmp


def test_host_pipeline_nvfp4_outputs_equal_direct_calls():
    """moe.HostPipeline(nvfp4=True): four different batches from pinned host
    buffers, two in flight; each output equals moe_layer_nvfp4 on that batch."""
    moe = _moe()
    L = pow2_layer()
    T = 16
    pipe = moe.HostPipeline(T, DEV, 2, nvfp4=True)
    toks = [synth.make_tokens(T, 1300 + k) for k in range(4)]
    bias = torch.from_numpy(toks[0].bias).to(DEV)
    hosts = []
    for tok in toks:
        x_h = torch.from_numpy(tok.x_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
        lg_h = torch.from_numpy(tok.logits).pin_memory()
        out_h = torch.full((T, 1536), float("nan"), dtype=torch.bfloat16).pin_memory()
        hosts.append((x_h, lg_h, out_h))
    for x_h, lg_h, out_h in hosts:
        pipe.submit(x_h, lg_h, out_h, bias, L.packed)
    pipe.drain()
    _status_ok()
    for tok, (x_h, lg_h, out_h) in zip(toks, hosts):
        x, lg, _ = tokens_dev(tok)
        ref = moe.moe_layer_nvfp4(x, lg, bias, L.packed)
        torch.cuda.synchronize()
        assert torch.equal(out_h.view(torch.int16), ref.cpu().view(torch.int16))
