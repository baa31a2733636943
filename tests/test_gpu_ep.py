"""Expert parallelism on one GPU: W = 2, 4, 8 ranks run in lockstep by one
process (group_limited_routed_moe_b200.ep.forward_in_process), each rank with
its own tokens and its slice of the experts (moe_pack_experts), the owner's
compute through moe_permute (empty slots skipped) and moe_expert_ffn_slice,
the source's combine through moe_combine, the exchanges as copies.

Each rank's output is compared with the single-GPU step calls (moe_permute,
moe_expert_ffn on the whole layer, moe_combine) on the same routing: bit for
bit where both run the same expert-FFN kernel shape (the weights-as-M kernel
up to 256 rows on both sides), and against the float64 oracle within the
layer tolerance always.
"""
import numpy as np
import pytest
import torch

import oracle as O
from group_limited_routed_moe_b200 import ep, synth
from gpu_helpers import DEV, REL_L2_TOL, layer0_weights, oracle_layer, to_host_bits, tokens_dev

pytestmark = pytest.mark.gpu


def _slices(W, world):
    from group_limited_routed_moe_b200 import moe
    n = ep.experts_per_rank(world)
    return [moe.moe_pack_experts(W.wg[d * n:(d + 1) * n].contiguous(),
                                 W.wu[d * n:(d + 1) * n].contiguous(),
                                 W.wd[d * n:(d + 1) * n].contiguous()) for d in range(world)]


@pytest.mark.parametrize("world,T", [(2, 16), (4, 16), (8, 16), (2, 300), (8, 200)])
def test_expert_parallel_in_process_equals_single_gpu_layer(world, T):
    from group_limited_routed_moe_b200 import moe
    W = layer0_weights()
    packs = _slices(W, world)
    layers = [ep.ExpertParallelMoE(d, world, packs[d]) for d in range(world)]
    toks, xs, idxs, ws, refs = [], [], [], [], []
    for d in range(world):
        tok = synth.make_tokens(T, 40 + d)
        x, lg, b = tokens_dev(tok)
        idx, w = moe.moe_route(lg, b)
        toks.append(tok)
        xs.append(x)
        idxs.append(idx)
        ws.append(w)
        # the single-GPU step calls on the same routing
        _, offsets, perm_src, inv_perm = moe.moe_permute(idx)
        h = torch.empty((T * 8, 512), dtype=torch.float16, device=DEV)
        y = torch.empty((T * 8, 1536), dtype=torch.float16, device=DEV)
        moe.moe_expert_ffn(x, W.packed, offsets, perm_src, h, y)
        refs.append(moe.moe_combine(y, w, inv_perm))
    outs = ep.forward_in_process(layers, xs, idxs, ws)
    torch.cuda.synchronize()
    assert moe.get_device_status(0) == moe.MOE_OK, moe.last_error()
    for d in range(world):
        # the owners' row counts decide the kernel shape on each side
        rows_max = max(sum(L.recv_counts) for L in layers)
        if T <= 256 and rows_max <= 256:
            assert torch.equal(outs[d].view(torch.int16), refs[d].view(torch.int16)), d
        ref64, _ = oracle_layer(toks[d], W)
        err = O.rel_l2(O.bf16_bits_to_f64(to_host_bits(outs[d])), ref64)
        assert err <= REL_L2_TOL, (d, err)


def test_expert_parallel_fan_out_at_most_four_ranks():
    """Every token's row reaches at most 4 of 8 ranks (the group limit)."""
    from group_limited_routed_moe_b200 import moe
    tok = synth.make_tokens(2048, 7)
    _, lg, b = tokens_dev(tok)
    idx, _ = moe.moe_route(lg, b)
    p = ep.plan_dispatch(idx, 8)
    per_tok = torch.bincount(p.send_tok, minlength=2048)
    assert int(per_tok.max()) <= 4 and int(per_tok.min()) >= 1
    assert int(p.send_counts.sum()) == int(per_tok.sum())


@pytest.mark.parametrize("T", [5, 700, 3000])
def test_permute_skips_empty_slots(T):
    """moe_permute with some slots empty (-1): the stable counting sort of the
    non-empty items only (checked against the oracle's sort of those items),
    inv_perm = -1 at the empty ones, offsets[128] = the non-empty count."""
    from group_limited_routed_moe_b200 import moe
    rng = np.random.default_rng(T)
    idx = np.stack([rng.permutation(128)[:8] for _ in range(T)]).astype(np.int32)
    idx[rng.random((T, 8)) < 0.6] = -1
    counts, offsets, perm_src, inv_perm = moe.moe_permute(torch.from_numpy(idx).to(DEV))
    torch.cuda.synchronize()
    assert moe.get_device_status(0) == moe.MOE_OK, moe.last_error()
    flat = idx.reshape(-1)
    valid = np.nonzero(flat >= 0)[0]
    o = O.permute(flat[valid].reshape(-1, 1))  # one slot per item: the items' stable sort
    n = len(valid)
    np.testing.assert_array_equal(counts.cpu().numpy(), o.counts)
    np.testing.assert_array_equal(offsets.cpu().numpy(), o.offsets)
    np.testing.assert_array_equal(perm_src.cpu().numpy()[:n], valid[o.perm_src])
    inv = inv_perm.cpu().numpy()
    assert np.all(inv[flat < 0] == -1)
    np.testing.assert_array_equal(inv[valid], o.inv_perm)
