"""moe_permute_fixed_scratch (library-owned scratch, no device allocation)
against moe_permute and against the float64 oracle's permutation, called
through the C ABI.

Collected last so that it also runs after every other GPU test in one process;
it passes on its own in a fresh process as well.  Each case makes two calls in
a row on different routings: the second must not see anything the first left
in the shared scratch; one case goes from the largest T (512 histogram rows)
to a smaller multi-block T, whose call must never read the stale rows past
its own blocks.  Integer outputs, so the comparison is bit-exact."""

import ctypes

import numpy as np
import pytest
import torch

import oracle as O
from group_limited_routed_moe_b200 import moe as M

N_EXPERTS, TOPK, OFFSETS_LEN = M.N_EXPERTS, M.TOPK, M.OFFSETS_LEN


def _routing(T, seed, hot=0):
    """[T][8] distinct expert ids per token; `hot` > 0 sends most tokens to the
    first `hot` experts (a skewed load)."""
    g = torch.Generator().manual_seed(seed)
    score = torch.rand((T, N_EXPERTS), generator=g)
    if hot:
        score[:, :hot] += 0.9
    return score.argsort(dim=1, descending=True)[:, :TOPK].to(torch.int32).contiguous()


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _fixed(idx_dev, stream):
    T = idx_dev.shape[0]
    dev = idx_dev.device
    counts = torch.full((N_EXPERTS,), -7, dtype=torch.int32, device=dev)
    offsets = torch.full((OFFSETS_LEN,), -7, dtype=torch.int32, device=dev)
    perm = torch.full((max(T * TOPK, 1),), -7, dtype=torch.int32, device=dev)
    inv = torch.full((max(T * TOPK, 1),), -7, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    rc = M.lib.moe_permute_fixed_scratch(_p(idx_dev), T, _p(counts), _p(offsets), _p(perm),
                                         _p(inv), ctypes.c_void_p(stream.cuda_stream))
    assert rc == M.MOE_OK, M.last_error()
    return counts, offsets, perm[:T * TOPK], inv[:T * TOPK]


def _same(got, ref, idx):
    counts, offsets, perm, inv = got
    r_counts, r_offsets, r_perm, r_inv = ref
    assert torch.equal(counts.cpu(), r_counts.cpu())
    assert torch.equal(offsets[:N_EXPERTS + 1].cpu(), r_offsets.cpu())
    assert torch.equal(offsets[132:OFFSETS_LEN].cpu(), torch.zeros(OFFSETS_LEN - 132, dtype=torch.int32))
    assert torch.equal(perm.cpu(), r_perm.cpu())
    assert torch.equal(inv.cpu(), r_inv.cpu())
    # and against the oracle's stable counting sort of the same routing
    o = O.permute(idx.cpu().numpy())
    np.testing.assert_array_equal(counts.cpu().numpy(), o.counts)
    np.testing.assert_array_equal(offsets[:N_EXPERTS + 1].cpu().numpy(), o.offsets)
    np.testing.assert_array_equal(perm.cpu().numpy(), o.perm_src)
    np.testing.assert_array_equal(inv.cpu().numpy(), o.inv_perm)


@pytest.mark.gpu
@pytest.mark.parametrize("T,hot", [(0, 0), (700, 0), (8189, 16), (40000, 0), (65536, 4)])
def test_fixed_scratch_permute_matches_moe_permute(T, hot):
    assert M.lib.moe_permute_fixed_scratch_max_tokens() == 65536
    stream = torch.cuda.current_stream()
    for call, seed in enumerate((11 + T, 12 + T)):  # two calls in a row
        idx = _routing(T, seed, hot if call == 0 else 0).cuda()
        ref = M.moe_permute(idx)
        got = _fixed(idx, stream)
        torch.cuda.synchronize()
        _same(got, ref, idx)
        if T:
            rows = np.sort(got[2].cpu().numpy())
            assert np.array_equal(rows, np.arange(T * TOPK))
    torch.cuda.synchronize()
    assert M.lib.moe_get_device_status(torch.cuda.current_device()) == M.MOE_OK


@pytest.mark.gpu
def test_fixed_scratch_permute_large_then_small():
    """T = 65536 (512 blocks of 128 tokens) fills every histogram row; T = 2000
    (32 blocks of 64 tokens, the multi-block path) then runs on the same stream
    with rows 32..511 stale."""
    stream = torch.cuda.current_stream()
    for T, seed, hot in ((65536, 5, 0), (2000, 6, 16), (65536, 7, 8), (1100, 8, 0)):
        idx = _routing(T, seed, hot).cuda()
        ref = M.moe_permute(idx)
        got = _fixed(idx, stream)
        torch.cuda.synchronize()
        _same(got, ref, idx)
    assert M.lib.moe_get_device_status(torch.cuda.current_device()) == M.MOE_OK


@pytest.mark.gpu
def test_fixed_scratch_permute_rejects_too_many_tokens():
    T = M.lib.moe_permute_fixed_scratch_max_tokens() + 1
    dummy = torch.zeros(OFFSETS_LEN, dtype=torch.int32, device="cuda")
    rc = M.lib.moe_permute_fixed_scratch(_p(dummy), T, _p(dummy), _p(dummy), _p(dummy),
                                         _p(dummy), None)
    assert rc == M.MOE_ERR_INVALID_ARG
    assert "65536" in M.last_error()
