"""GPU parity of the fused layer (moe_layer) on every single-layer workload,
plus the invariances the layer must satisfy bit for bit on the device.

Tolerances: routing ids bit-exact, weights <= 1e-6, output rel-L2 <= 5e-3
against the float64 oracle (bf16 inputs, fp32 accumulation, bf16 h / y / out).
"""
import numpy as np
import pytest
import torch

import oracle as O
from group_limited_routed_moe_b200 import synth
from gpu_helpers import (DEV, REL_L2_TOL, W_TOL, layer0_weights, oracle_layer, to_dev_bf16,
                         to_host_bits, tokens_dev)

pytestmark = pytest.mark.gpu


def _moe():
    from group_limited_routed_moe_b200 import moe
    return moe


def _run_layer(tok, T_buf=None, residual=None):
    moe = _moe()
    W = layer0_weights()
    T = tok.x_bits.shape[0]
    x, lg, bias = tokens_dev(tok, T_buf)
    idx = torch.empty((T, 8), dtype=torch.int32, device=DEV)
    w = torch.empty((T, 8), dtype=torch.float32, device=DEV)
    out = torch.full((x.shape[0], 1536), float("nan"), dtype=torch.bfloat16, device=DEV)
    moe.moe_layer(x[:T], lg[:T], bias, W.packed, residual=residual, out=out[:T],
                  topk_idx_out=idx, topk_w_out=w)
    torch.cuda.synchronize()
    assert moe.get_device_status(0) == moe.MOE_OK, moe.last_error()
    return out, idx, w


@pytest.mark.parametrize("name", ["decode_T16"] + [f"decode_T4_seed{s}" for s in range(1, 9)] +
                         ["prefill_T2048_skewed"])
def test_layer_parity_full(name):
    wl = synth.WORKLOADS[name]
    tok = synth.make_tokens(wl.T, wl.seed, hot=wl.hot)
    out, idx, w = _run_layer(tok)
    ref, rr = oracle_layer(tok, layer0_weights())
    assert np.array_equal(idx.cpu().numpy(), rr.topk_idx)
    assert np.abs(w.cpu().numpy() - rr.topk_w).max() <= W_TOL
    err = O.rel_l2(O.bf16_bits_to_f64(to_host_bits(out)), ref)
    assert err <= REL_L2_TOL, f"{name}: rel-L2 {err:.3e}"
    if wl.hot:
        counts = np.bincount(rr.topk_idx.ravel(), minlength=128)
        assert counts[tok.hot_experts].mean() > 4 * counts.mean()


def test_layer_parity_prefill_T8189():
    """Long-prompt prefill: 8,189 real tokens in buffers of 8,192.  The oracle
    checks every token; rows 8189..8191 of the output buffer stay untouched."""
    wl = synth.WORKLOADS["prefill_T8189"]
    tok = synth.make_tokens(wl.T, wl.seed)
    out, idx, w = _run_layer(tok, T_buf=wl.T_buf)
    ref, rr = oracle_layer(tok, layer0_weights())
    assert np.array_equal(idx.cpu().numpy(), rr.topk_idx)
    assert np.abs(w.cpu().numpy() - rr.topk_w).max() <= W_TOL
    got = O.bf16_bits_to_f64(to_host_bits(out[:wl.T]))
    err = O.rel_l2(got, ref)
    assert err <= REL_L2_TOL, f"rel-L2 {err:.3e}"
    # token-wise: no single token far off
    per_tok = np.linalg.norm(got - ref, axis=1) / np.linalg.norm(ref, axis=1)
    assert per_tok.max() <= 4 * REL_L2_TOL
    assert torch.isnan(out[wl.T:].float()).all()


def test_layer_permutation_and_batch_invariance():
    """out(P x) = P out(x) and rows of a T=16 call equal T=4 + T=12 calls, bit
    for bit (the combine is deterministic, every token is independent)."""
    tok = synth.make_tokens(16, 0)
    out, _, _ = _run_layer(tok)
    perm = np.random.default_rng(0).permutation(16)
    tok_p = synth.TokenInputs(tok.x_bits[perm].copy(), tok.logits[perm].copy(), tok.bias)
    out_p, _, _ = _run_layer(tok_p)
    assert torch.equal(out_p.view(torch.int16), out[torch.as_tensor(perm, device=DEV)].view(torch.int16))
    a = synth.TokenInputs(tok.x_bits[:4].copy(), tok.logits[:4].copy(), tok.bias)
    b = synth.TokenInputs(tok.x_bits[4:].copy(), tok.logits[4:].copy(), tok.bias)
    oa, _, _ = _run_layer(a)
    ob, _, _ = _run_layer(b)
    assert torch.equal(torch.cat([oa, ob]).view(torch.int16), out.view(torch.int16))


def test_layer_deterministic():
    tok = synth.make_tokens(2048, 2, hot=16)
    o1, _, _ = _run_layer(tok)
    o2, _, _ = _run_layer(tok)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))


def test_layer_residual():
    """out = bf16(residual + moe(x)), in place on the residual buffer.

    The oracle's value is bf16(x + moe_exact).  The GPU rounds x + moe_fp32,
    and moe_fp32 differs from moe_exact by the layer's own error, so the two
    roundings agree except where a bf16 boundary lies between them: every
    element is within one bf16 ulp of the oracle and almost all are equal."""
    tok = synth.make_tokens(16, 0)
    x, lg, bias = tokens_dev(tok)
    moe = _moe()
    W = layer0_weights()
    h = x.clone()
    moe.moe_layer(x, lg, bias, W.packed, residual=h, out=h)
    torch.cuda.synchronize()
    upd, _ = oracle_layer(tok, W)
    exact = O.bf16_bits_to_f64(tok.x_bits) + upd
    ref_bits = O.f64_to_bf16_bits(exact)
    got_bits = to_host_bits(h)
    got, ref = O.bf16_bits_to_f64(got_bits), O.bf16_bits_to_f64(ref_bits)
    assert O.rel_l2(got, exact) <= REL_L2_TOL
    assert np.mean(got_bits == ref_bits) >= 0.9
    # one bf16 ulp of the sum plus the layer's own error (a few 1e-3 of the update)
    ulp = np.ldexp(1.0, np.frexp(np.abs(exact))[1] - 8)
    assert np.all(np.abs(got - exact) <= ulp + 0.02 * np.sqrt(np.mean(upd ** 2)))


@pytest.mark.parametrize("fmt", ["bf16", "fp8", "nvfp4"])
def test_layer_from_host_e2e(fmt):
    """moe_layer_host (C ABI, host buffers in and out) against the oracle, and
    bit for bit against the device-buffer layer call of the same format."""
    moe = _moe()
    W = layer0_weights()
    T = 16
    tok = synth.make_tokens(T, 0)
    x_h = torch.from_numpy(tok.x_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    lg_h = torch.from_numpy(tok.logits).pin_memory()
    out_h = torch.full((T, 1536), float("nan"), dtype=torch.bfloat16).pin_memory()
    bias = torch.from_numpy(tok.bias).to(DEV)
    f = moe.WEIGHT_FORMATS[fmt]
    if fmt == "bf16":
        packed, layer = W.packed, moe.moe_layer
    else:
        qs = []
        for which in (synth.W_GATE, synth.W_UP, synth.W_DOWN):
            if fmt == "fp8":
                q, sc = synth.fp8_weights_torch(0, 0, which, DEV, "pow2")
                qs += [q, sc]
            else:
                qs += list(synth.nvfp4_weights_torch(0, 0, which, DEV, "pow2"))
        packed = (moe.moe_pack_weights_fp8 if fmt == "fp8" else moe.moe_pack_weights_nvfp4)(*qs)
        layer = moe.moe_layer_fp8 if fmt == "fp8" else moe.moe_layer_nvfp4
        del qs
    ws = moe.alloc_layer_host_workspace(T, DEV, f)
    moe.moe_layer_host(x_h, lg_h, bias, packed, out_h, ws, f)
    x_d, lg_d, _ = tokens_dev(tok)
    direct = layer(x_d, lg_d, bias, packed)
    torch.cuda.synchronize()
    assert moe.get_device_status(0) == moe.MOE_OK, moe.last_error()
    assert torch.equal(out_h.view(torch.int16), direct.cpu().view(torch.int16))
    if fmt != "bf16":
        return  # the quantised layers' oracle parity is tested in their own files
    torch.cuda.synchronize()
    ref, _ = oracle_layer(tok, W)
    got = O.bf16_bits_to_f64(out_h.view(torch.int16).numpy().view(np.uint16))
    assert O.rel_l2(got, ref) <= REL_L2_TOL


def test_layer_graph_capture():
    """The layer is capturable in a CUDA graph and replays to the same bits."""
    moe = _moe()
    W = layer0_weights()
    tok = synth.make_tokens(16, 0)
    x, lg, bias = tokens_dev(tok)
    ws = moe.alloc_layer_workspace(16, DEV)
    out = torch.empty_like(x)
    moe.moe_layer(x, lg, bias, W.packed, out=out, workspace=ws)
    torch.cuda.synchronize()
    ref = out.clone()
    out.zero_()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            moe.moe_layer(x, lg, bias, W.packed, out=out, workspace=ws, stream=s)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    del g


@pytest.mark.parametrize("T,depth", [(16, 3), (1000, 2)])
def test_host_pipeline_outputs_equal_direct_calls(T, depth):
    """moe.HostPipeline keeps `depth` host-buffer calls in flight (copies of one
    overlapping the layer of another).  Six different batches go through it; each
    output must equal, bit for bit, moe_layer on that batch: no call may read or
    overwrite another call's buffers."""
    moe = _moe()
    W = layer0_weights()
    pipe = moe.HostPipeline(T, DEV, depth)
    toks = [synth.make_tokens(T, 300 + k) for k in range(6)]
    bias = torch.from_numpy(toks[0].bias).to(DEV)
    hosts = []
    for tok in toks:
        x_h = torch.from_numpy(tok.x_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
        lg_h = torch.from_numpy(tok.logits).pin_memory()
        out_h = torch.full((T, 1536), float("nan"), dtype=torch.bfloat16).pin_memory()
        hosts.append((x_h, lg_h, out_h))
    for x_h, lg_h, out_h in hosts:
        pipe.submit(x_h, lg_h, out_h, bias, W.packed)
    pipe.drain()
    assert moe.get_device_status(0) == moe.MOE_OK, moe.last_error()
    for tok, (x_h, lg_h, out_h) in zip(toks, hosts):
        x, lg, _ = tokens_dev(tok)
        ref = moe.moe_layer(x, lg, bias, W.packed)
        torch.cuda.synchronize()
        assert torch.equal(out_h.view(torch.int16), ref.cpu().view(torch.int16))
