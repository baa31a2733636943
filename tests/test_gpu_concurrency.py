"""Layers on unordered streams: the persistent expert-FFN kernels must finish
however many of their CTAs are resident at once.

A single-launch expert FFN makes a down tile wait for every gate/up tile of
its expert.  If a CTA that is not running owned such a gate/up tile (a first
tile assigned by block index), a running CTA could wait for it until the
bounded wait ran out.  Here three layers (T = 16, 2048 and 8189, each with its
own workspace) run on three streams with no ordering between them, so their
kernels compete for the SMs, and the wait limit is cut to 50 ms so that a
regression shows up as MOE_ERR_TIMEOUT rather than as a 2 s stall.  Each
output must equal, bit for bit, the same layer run alone.
"""
import pytest
import torch

from group_limited_routed_moe_b200 import synth
from gpu_helpers import DEV, layer0_weights, to_dev_bf16, tokens_dev

pytestmark = pytest.mark.gpu

CASES = (("decode_T16", 16, 16, 0), ("prefill_T2048_skewed", 2048, 2048, 16),
         ("prefill_T8189", 8189, 8192, 0))


def _inputs():
    out = []
    for name, T, T_buf, hot in CASES:
        wl = synth.WORKLOADS[name]
        tok = synth.make_tokens(T, wl.seed, hot=hot)
        out.append((T, tokens_dev(tok, T_buf)))
    return out


def test_layers_on_unordered_streams_equal_serial_calls():
    from group_limited_routed_moe_b200 import moe
    W = layer0_weights()
    ins = _inputs()
    wss = [moe.alloc_layer_workspace(T, DEV) for T, _ in ins]
    outs_serial = []
    for (T, (x, lg, b)), ws in zip(ins, wss):
        outs_serial.append(moe.moe_layer(x[:T], lg[:T], b, W.packed, workspace=ws).clone())
    torch.cuda.synchronize()
    assert moe.get_device_status(0) == moe.MOE_OK, moe.last_error()

    streams = [torch.cuda.Stream() for _ in ins]
    outs = [torch.empty_like(o) for o in outs_serial]
    moe.set_wait_timeout_ns(50_000_000)
    try:
        for rep in range(6):
            for o in outs:
                o.fill_(0)
            ev = torch.cuda.Event()
            ev.record()
            order = list(range(len(ins))) if rep % 2 == 0 else list(reversed(range(len(ins))))
            for i in order:
                T, (x, lg, b) = ins[i]
                streams[i].wait_event(ev)
                moe.moe_layer(x[:T], lg[:T], b, W.packed, out=outs[i], workspace=wss[i],
                              stream=streams[i])
            torch.cuda.synchronize()
            assert moe.get_device_status(0) == moe.MOE_OK, f"rep {rep}: {moe.last_error()}"
            for (name, *_), o, ref in zip(CASES, outs, outs_serial):
                assert torch.equal(o.view(torch.int16), ref.view(torch.int16)), (name, rep)
    finally:
        moe.set_wait_timeout_ns(2_000_000_000)


def _aligned_workspace(nbytes):
    raw = torch.empty(nbytes + 1024, dtype=torch.uint8, device=DEV)
    off = (-raw.data_ptr()) % 1024
    return raw[off:off + nbytes]


def test_weight_pack_launches_on_unordered_streams_equal_serial_calls():
    """The same with launches that run several weight packs: a layer with one
    shared expert (routed and shared packs in one launch) at T = 16 and 2048,
    and the 256-expert shape with 2 shared experts (three packs) at T = 16 and
    600, all on their own streams with no ordering between them."""
    from group_limited_routed_moe_b200 import moe
    from test_gpu_e256 import shared2, weights as e256_weights
    from test_gpu_shared import shared_pack
    W = layer0_weights()
    _, sp1 = shared_pack(1)
    W2 = e256_weights()
    _, sp2 = shared2()
    calls = []
    for T, seed in ((16, 31), (2048, 32)):
        x, lg, b = tokens_dev(synth.make_tokens(T, seed))
        ws = _aligned_workspace(moe.layer_shared_workspace_bytes(T, 1, False))
        calls.append(lambda out, s, x=x, lg=lg, b=b, ws=ws: moe.moe_layer_shared(
            x, lg, b, sp1, 1, packed_w=W.packed, out=out, workspace=ws, stream=s))
    for T, seed in ((16, 33), (600, 34)):
        tok = synth.make_tokens_e256(T, seed)
        x = to_dev_bf16(tok.x_bits)
        lg, b = torch.from_numpy(tok.logits).to(DEV), torch.from_numpy(tok.bias).to(DEV)
        ws = _aligned_workspace(moe.layer_e256_workspace_bytes(T, 2))
        calls.append(lambda out, s, x=x, lg=lg, b=b, ws=ws: moe.moe_layer_e256(
            x, lg, b, W2.packed[0], W2.packed[1], sp2, 2, out=out, workspace=ws, stream=s))
    sizes = (16, 2048, 16, 600)
    refs = []
    for call, T in zip(calls, sizes):
        o = torch.empty((T, 1536), dtype=torch.bfloat16, device=DEV)
        call(o, None)
        refs.append(o)
    torch.cuda.synchronize()
    assert moe.get_device_status(0) == moe.MOE_OK, moe.last_error()
    streams = [torch.cuda.Stream() for _ in calls]
    outs = [torch.empty_like(r) for r in refs]
    moe.set_wait_timeout_ns(50_000_000)
    try:
        for rep in range(4):
            for o in outs:
                o.fill_(0)
            ev = torch.cuda.Event()
            ev.record()
            order = range(len(calls)) if rep % 2 == 0 else reversed(range(len(calls)))
            for i in order:
                streams[i].wait_event(ev)
                calls[i](outs[i], streams[i])
            torch.cuda.synchronize()
            assert moe.get_device_status(0) == moe.MOE_OK, f"rep {rep}: {moe.last_error()}"
            for i, (o, r) in enumerate(zip(outs, refs)):
                assert torch.equal(o.view(torch.int16), r.view(torch.int16)), (i, rep)
    finally:
        moe.set_wait_timeout_ns(2_000_000_000)
