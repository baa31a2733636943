"""Large batches: the layer at 2^20 tokens, routing and the sort at the
maximum batch of 2^22 tokens.

At T = 2^20 the element offsets into y_perm (8T rows of 1536) and h (8T rows
of 512) pass 2^31, so a 32-bit product anywhere in the expert FFN, the
combine or the gather would show.  The tokens are copies of the 8,189 tokens
of prefill_T8189 (token i is base token src[i], src seeded), and the layer is
token-wise independent, so every output row, routing id and weight must equal
the T = 8189 call's for the same base token, bit for bit.  The T = 8189 call
is the one the oracle checks token by token in the layer tests.

At T = 2^22 (moe_max_tokens) the sort is checked against its definition: a
stable counting sort of the (token, slot) rows by expert, i.e. the order of
the keys expert * 8T + row, which a library sort computes independently."""
import numpy as np
import pytest
import torch

from group_limited_routed_moe_b200 import synth
from gpu_helpers import DEV, layer0_weights, to_dev_bf16

pytestmark = pytest.mark.gpu


def _moe():
    from group_limited_routed_moe_b200 import moe
    return moe


def _status_ok():
    moe = _moe()
    assert moe.get_device_status(0) == moe.MOE_OK, moe.last_error()


def _base():
    wl = synth.WORKLOADS["prefill_T8189"]
    tok = synth.make_tokens(wl.T, wl.seed)
    x = to_dev_bf16(tok.x_bits)
    lg = torch.from_numpy(tok.logits).to(DEV)
    bias = torch.from_numpy(tok.bias).to(DEV)
    return wl.T, x, lg, bias


def _sources(n_base, T, seed):
    src = np.random.default_rng(seed).integers(0, n_base, size=T)
    return torch.from_numpy(src).to(DEV)


def test_layer_two_to_the_20_tokens_equals_base_rows():
    moe = _moe()
    W = layer0_weights()
    n, x, lg, bias = _base()
    T = 1 << 20
    src = _sources(n, T, 2020)
    idx0 = torch.empty((n, 8), dtype=torch.int32, device=DEV)
    w0 = torch.empty((n, 8), dtype=torch.float32, device=DEV)
    out0 = moe.moe_layer(x, lg, bias, W.packed, topk_idx_out=idx0, topk_w_out=w0)
    xb = x.index_select(0, src)
    lgb = lg.index_select(0, src)
    idx = torch.empty((T, 8), dtype=torch.int32, device=DEV)
    w = torch.empty((T, 8), dtype=torch.float32, device=DEV)
    ws = moe.alloc_layer_workspace(T, DEV)
    assert 8 * T * 1536 > 1 << 31 and 8 * T * 512 > 1 << 31  # y_perm and h element offsets
    out = moe.moe_layer(xb, lgb, bias, W.packed, topk_idx_out=idx, topk_w_out=w, workspace=ws)
    torch.cuda.synchronize()
    _status_ok()
    del ws, xb, lgb
    assert torch.equal(idx, idx0.index_select(0, src))
    assert torch.equal(w.view(torch.int32), w0.view(torch.int32).index_select(0, src))
    assert torch.equal(out.view(torch.int16), out0.view(torch.int16).index_select(0, src))
    del out, idx, w
    torch.cuda.empty_cache()


def test_route_and_sort_at_the_maximum_batch():
    moe = _moe()
    n, _, lg, bias = _base()
    T = int(moe.lib.moe_max_tokens())
    assert T == 1 << 22
    src = _sources(n, T, 2022)
    idx0, w0 = moe.moe_route(lg, bias)
    lgb = lg.index_select(0, src)
    idx, w = moe.moe_route(lgb, bias)
    torch.cuda.synchronize()
    _status_ok()
    del lgb
    assert torch.equal(idx, idx0.index_select(0, src))
    assert torch.equal(w.view(torch.int32), w0.view(torch.int32).index_select(0, src))
    del w
    counts, offsets, perm_src, inv_perm = moe.moe_permute(idx)
    torch.cuda.synchronize()
    _status_ok()
    flat = idx.view(-1).long()
    rows = flat.numel()
    ref_counts = torch.bincount(flat, minlength=128)
    assert torch.equal(counts.long(), ref_counts)
    assert torch.equal(offsets.long(), torch.cat([ref_counts.new_zeros(1), ref_counts.cumsum(0)]))
    order = torch.argsort(flat * rows + torch.arange(rows, device=DEV))
    assert torch.equal(perm_src.long(), order)
    ref_inv = torch.empty_like(order)
    ref_inv[order] = torch.arange(rows, device=DEV)
    assert torch.equal(inv_perm.long(), ref_inv)
    del idx, counts, offsets, perm_src, inv_perm, flat, order, ref_inv
    torch.cuda.empty_cache()
