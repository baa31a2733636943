"""GPU parity of the second MoE shape (256 experts in 8 groups of 32, keep 4,
top-6, 2 shared experts: moe_route_e256, moe_layer_e256) against the float64
oracle.  The routing kernel must reproduce the oracle's ids bit for bit
(float64 decisions on both sides) and its weights within 1e-6; the layer,
which runs the 128-expert FFN kernels on each half of the experts, within the
layer tolerance."""
import functools

import numpy as np
import pytest
import torch

import oracle as O
from group_limited_routed_moe_b200 import synth
from gpu_helpers import DEV, REL_L2_TOL, W_TOL, to_dev_bf16, to_host_bits

pytestmark = pytest.mark.gpu


def _moe():
    from group_limited_routed_moe_b200 import moe
    return moe


class E256Weights:
    """Both halves made on the device, packed; host bits per expert on demand."""

    def __init__(self, seed=0, layer=0):
        moe = _moe()
        self.seed, self.layer = seed, layer
        self.dev = [[synth.e256_weight_bits_torch(seed, layer, w, half, DEV)
                     for w in (synth.W_GATE, synth.W_UP, synth.W_DOWN)] for half in (0, 1)]
        self.packed = [moe.moe_pack_weights(*self.dev[h]) for h in (0, 1)]
        torch.cuda.synchronize()

    def host(self, experts):
        experts = np.unique(np.asarray(experts))
        out = []
        for wi in range(3):
            shape = tuple(self.dev[0][wi].shape[1:])
            a = np.zeros((256,) + shape, np.uint16)
            for half in (0, 1):
                sel = experts[(experts >= 128 * half) & (experts < 128 * (half + 1))]
                if len(sel):
                    idx = torch.as_tensor(sel - 128 * half, device=DEV)
                    a[sel] = to_host_bits(self.dev[half][wi][idx])
            out.append(a)
        return tuple(out)


@functools.lru_cache(maxsize=1)
def weights() -> E256Weights:
    return E256Weights()


@functools.lru_cache(maxsize=1)
def shared2():
    moe = _moe()
    bits = synth.shared_weights_np(0, 0, 2)
    return bits, moe.moe_pack_shared(*(to_dev_bf16(b) for b in bits))


def _dev(tok):
    x = to_dev_bf16(tok.x_bits)
    return x, torch.from_numpy(tok.logits).to(DEV), torch.from_numpy(tok.bias).to(DEV)


def _status_ok():
    moe = _moe()
    assert moe.get_device_status(0) == moe.MOE_OK, moe.last_error()


@pytest.mark.parametrize("T", [1, 7, 300, 4096])
def test_route_e256_parity(T):
    moe = _moe()
    tok = synth.make_tokens_e256(T, 10 + T)
    _, lg, bias = _dev(tok)
    for b_np, b in ((tok.bias, bias), (None, None)):
        idx, w = moe.moe_route_e256(lg, b)
        torch.cuda.synchronize()
        _status_ok()
        rr = O.route_e256(tok.logits, b_np)
        assert not ((rr.group_margin < 1e-12) | (rr.expert_margin < 1e-12)).any()
        assert np.array_equal(idx.cpu().numpy(), rr.topk_idx)
        assert np.abs(w.cpu().numpy() - rr.topk_w).max() <= W_TOL


def test_route_e256_ties():
    """All-equal logits: groups 0-3 kept, experts 0..5 in index order, weights
    1/6; one saturated expert per group: ties broken by the float64 scores."""
    moe = _moe()
    lg = np.zeros((3, 256), np.float32)
    lg[1, ::32] = 60.0
    lg[2, 200:206] = 40.0
    idx, w = moe.moe_route_e256(torch.from_numpy(lg).to(DEV), None)
    torch.cuda.synchronize()
    rr = O.route_e256(lg, None)
    assert np.array_equal(idx.cpu().numpy(), rr.topk_idx)
    assert idx.cpu().numpy()[0].tolist() == [0, 1, 2, 3, 4, 5]
    assert np.abs(w.cpu().numpy() - rr.topk_w).max() <= W_TOL


@pytest.mark.parametrize("T", [1, 7, 16, 33, 64, 65])
def test_layer_e256_small_routing_equals_route_kernel(T):
    """Up to 64 tokens the layer routes and sorts in one block
    (route_sort_small_e256_kernel); its ids and weights must be the routing
    kernel's bit for bit (65 takes the multi-block path)."""
    moe = _moe()
    W = weights()
    tok = synth.make_tokens_e256(T, 40 + T)
    x, lg, bias = _dev(tok)
    idx = torch.empty((T, 6), dtype=torch.int32, device=DEV)
    wts = torch.empty((T, 6), dtype=torch.float32, device=DEV)
    moe.moe_layer_e256(x, lg, bias, W.packed[0], W.packed[1], None, 0, topk_idx_out=idx,
                       topk_w_out=wts)
    idx2, w2 = moe.moe_route_e256(lg, bias)
    torch.cuda.synchronize()
    _status_ok()
    assert torch.equal(idx, idx2)
    assert torch.equal(wts.view(torch.int32), w2.view(torch.int32))


def test_layer_e256_small_routing_ties():
    """The tie rows of test_route_e256_ties through the one-block routing."""
    moe = _moe()
    W = weights()
    lg = np.zeros((3, 256), np.float32)
    lg[1, ::32] = 60.0
    lg[2, 200:206] = 40.0
    x = to_dev_bf16(synth.make_tokens_e256(3, 5).x_bits)
    idx = torch.empty((3, 6), dtype=torch.int32, device=DEV)
    wts = torch.empty((3, 6), dtype=torch.float32, device=DEV)
    moe.moe_layer_e256(x, torch.from_numpy(lg).to(DEV), None, W.packed[0], W.packed[1], None, 0,
                       topk_idx_out=idx, topk_w_out=wts)
    torch.cuda.synchronize()
    _status_ok()
    rr = O.route_e256(lg, None)
    assert np.array_equal(idx.cpu().numpy(), rr.topk_idx)
    assert np.abs(wts.cpu().numpy() - rr.topk_w).max() <= W_TOL


@pytest.mark.parametrize("T,n_shared", [(1, 2), (16, 2), (64, 0), (300, 2), (2048, 2)])
def test_layer_e256_against_oracle(T, n_shared):
    moe = _moe()
    W = weights()
    sbits, spacked = shared2()
    tok = synth.make_tokens_e256(T, 20 + T)
    x, lg, bias = _dev(tok)
    idx = torch.empty((T, 6), dtype=torch.int32, device=DEV)
    wts = torch.empty((T, 6), dtype=torch.float32, device=DEV)
    out = moe.moe_layer_e256(x, lg, bias, W.packed[0], W.packed[1], spacked if n_shared else None,
                             n_shared, topk_idx_out=idx, topk_w_out=wts)
    torch.cuda.synchronize()
    _status_ok()
    rows = None if T <= 300 else np.sort(np.random.default_rng(T).choice(T, 64, replace=False))
    xb, lgs = (tok.x_bits, tok.logits) if rows is None else (tok.x_bits[rows], tok.logits[rows])
    rr = O.route_e256(lgs, tok.bias)
    wg, wu, wd = W.host(rr.topk_idx)
    sg, su, sd = (b[:n_shared] for b in sbits)
    ref = O.moe_layer_shared(xb, lgs, tok.bias, wg, wu, wd, sg, su, sd, route_result=rr)
    gi, gw, got = idx.cpu().numpy(), wts.cpu().numpy(), out.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        gi, gw, got = gi[rows], gw[rows], got[rows]
    assert np.array_equal(gi, rr.topk_idx)
    assert np.abs(gw - rr.topk_w).max() <= W_TOL
    assert O.rel_l2(got, ref) <= REL_L2_TOL


def test_layer_e256_residual_and_determinism():
    moe = _moe()
    W = weights()
    sbits, spacked = shared2()
    T = 40
    tok = synth.make_tokens_e256(T, 99)
    x, lg, bias = _dev(tok)
    a = moe.moe_layer_e256(x, lg, bias, W.packed[0], W.packed[1], spacked, 2, residual=x)
    b = moe.moe_layer_e256(x, lg, bias, W.packed[0], W.packed[1], spacked, 2, residual=x)
    torch.cuda.synchronize()
    _status_ok()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    rr = O.route_e256(tok.logits, tok.bias)
    wg, wu, wd = W.host(rr.topk_idx)
    ref = O.moe_layer_shared(tok.x_bits, tok.logits, tok.bias, wg, wu, wd, *sbits,
                             route_result=rr) + O.bf16_bits_to_f64(tok.x_bits)
    assert O.rel_l2(a.float().cpu().numpy().astype(np.float64), ref) <= REL_L2_TOL
