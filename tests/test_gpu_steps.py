"""GPU parity of each step through the C ABI against the float64 oracle.

Routing ids, per-expert counts and the permutation are compared bit for bit;
routing weights within 1e-6; expert outputs within the layer tolerance.
"""
import numpy as np
import pytest
import torch

import oracle as O
from group_limited_routed_moe_b200 import synth
from gpu_helpers import (DEV, REL_L2_TOL, W_TOL, extreme_logits, layer0_weights, to_dev_bf16,
                         to_host_bits, tokens_dev)

pytestmark = pytest.mark.gpu


def _moe():
    from group_limited_routed_moe_b200 import moe
    return moe


def _route_check(lg_np, bias_np, exact_ties=False):
    moe = _moe()
    T = lg_np.shape[0]
    lg = torch.from_numpy(lg_np).to(DEV)
    b = None if bias_np is None else torch.from_numpy(bias_np).to(DEV)
    idx, w = moe.moe_route(lg, b)
    torch.cuda.synchronize()
    rr = O.route(lg_np, bias_np)
    gi, gw = idx.cpu().numpy(), w.cpu().numpy()
    # audit: a float64 near-tie would be reported, not counted as a mismatch
    # (inputs built with exact ties are exempt: equal values are equal on both sides)
    ambiguous = (rr.group_margin < 1e-12) | (rr.expert_margin < 1e-12)
    if not exact_ties:
        assert not ambiguous.any(), f"{ambiguous.sum()} near-tied tokens in the inputs"
    assert np.array_equal(gi, rr.topk_idx), "routing ids differ"
    assert np.abs(gw - rr.topk_w).max() <= W_TOL
    return gi, gw, rr


@pytest.mark.parametrize("name", ["decode_T16", "decode_T4_seed1", "decode_T4_seed8",
                                  "prefill_T2048_skewed", "prefill_T8189"])
def test_route_parity_workloads(name):
    wl = synth.WORKLOADS[name]
    tok = synth.make_tokens(wl.T, wl.seed, hot=wl.hot)
    _route_check(tok.logits, tok.bias)


@pytest.mark.parametrize("T", [1, 7, 33, 257])
def test_route_ragged_and_no_bias(T):
    rng = np.random.default_rng(T)
    _route_check(rng.standard_normal((T, 128)).astype(np.float32), None)


def test_route_special_cases():
    moe = _moe()
    # all equal -> groups 0-3, experts 0..7, w = 1/8
    lg = torch.full((5, 128), 0.7, dtype=torch.float32, device=DEV)
    idx, w = moe.moe_route(lg, torch.zeros(128, device=DEV))
    assert idx.cpu().tolist() == [list(range(8))] * 5
    assert torch.all(w == 0.125)
    # exact ties between groups and experts resolve to the lower index
    a = np.full((1, 128), -3.0, np.float32)
    a[0, [32, 33, 80, 81]] = 2.0
    a[0, [34, 35, 82, 83]] = 1.0
    gi, _, _ = _route_check(a, None, exact_ties=True)
    assert gi[0].tolist() == [32, 33, 80, 81, 34, 35, 82, 83]
    # dominant expert and an excluded group
    rng = np.random.default_rng(3)
    lg2 = rng.standard_normal((16, 128)).astype(np.float32)
    b2 = (0.1 * rng.standard_normal(128)).astype(np.float32)
    lg2[:, 77] = 12.0
    b2[16:32] = -40.0
    gi, _, _ = _route_check(lg2, b2)
    assert np.all(gi[:, 0] == 77) and not np.any((gi >= 16) & (gi < 32))


def test_route_extreme_logits():
    """Scores at the ends of the sigmoid: z in (10, 36) (distinct, close to 1),
    z > 37 (float64 sigmoid == 1.0 exactly: ties broken by index), z < -745
    (sigmoid underflows to 0: ties), mixed with ordinary values."""
    lg, b = extreme_logits()
    _route_check(lg, None, exact_ties=True)
    _route_check(lg, b, exact_ties=True)


def _key_boundary_rows():
    """Logits and a bias that put scores on the edges of the routing keys: the
    float64 sum z = logit + bias rounding away a tiny bias (a float64 tie the
    exact sum would split), z = -0 against z = +0, z on either side of 10 and of
    -700 (the saturation tiers) by less than an fp32 ulp of the logit, and a
    bias 2^-40 times the logit that float64 still holds.  Other logits are -3
    (or -800 where the row tests the low tier)."""
    f = np.float32
    lg = np.full((6, 128), -3.0, f)
    b = np.zeros(128, f)
    b[5] = f(1e-30)                 # row 0: z = 2 + 1e-30 rounds to 2 = z of expert 6
    lg[0, [5, 6]] = 2.0
    b[8] = f(-0.0)                  # row 1: z = -0 (expert 8) and +0 (expert 9) are one score
    lg[1, 8], lg[1, 9] = f(-0.0), f(0.0)
    b[16], b[18] = f(-2.0 ** -20), f(2.0 ** -20)   # row 2: z just below / above 10, and 10
    lg[2, [16, 18, 19]] = 10.0
    lg[2, 17] = np.nextafter(f(10.0), f(0.0))      # equal to expert 16's z
    b[32], b[33] = f(1e-5), f(-1e-5)               # row 3: around -700 (33 drops to the low tier)
    lg[3, :] = -800.0
    lg[3, [32, 33, 34]] = -700.0
    lg[3, 35] = np.nextafter(f(-700.0), f(0.0))
    b[48] = f(2.0 ** -40)           # row 4: 0.5 + 2^-40 is exact in float64, above 0.5
    lg[4, [48, 49]] = 0.5
    lg[5, [5, 6, 8, 9, 48, 49]] = [2.0, 2.0, -0.0, 0.0, 0.5, 0.5]  # the same pairs together
    return lg, b


def test_route_key_boundaries():
    """The routing keys order scores exactly as the oracle's float64 sums do
    on the edges above, through moe_route and through the one-launch routing
    and sort of a small layer (whose ids must match too)."""
    moe = _moe()
    lg, b = _key_boundary_rows()
    gi, _, rr = _route_check(lg, b, exact_ties=True)
    assert list(gi[0, :2]) == [5, 6] and list(gi[1, :2]) == [8, 9]
    assert list(gi[2, :4]) == [18, 19, 16, 17] and list(gi[3, :4]) == [35, 32, 34, 33]
    assert list(gi[4, :2]) == [48, 49]
    W = layer0_weights()
    tok = synth.make_tokens(lg.shape[0], 5)
    x, _, _ = tokens_dev(tok)
    idx = torch.empty((lg.shape[0], 8), dtype=torch.int32, device=DEV)
    w = torch.empty((lg.shape[0], 8), dtype=torch.float32, device=DEV)
    moe.moe_layer(x, torch.from_numpy(lg).to(DEV), torch.from_numpy(b).to(DEV), W.packed,
                  topk_idx_out=idx, topk_w_out=w)
    torch.cuda.synchronize()
    assert moe.get_device_status(0) == moe.MOE_OK, moe.last_error()
    assert np.array_equal(idx.cpu().numpy(), rr.topk_idx)
    assert np.abs(w.cpu().numpy() - rr.topk_w).max() <= W_TOL


def test_route_key_fp32_overflow():
    """logit + bias above the fp32 range: the float64 sum decides (top tier)."""
    f = np.float32
    lg = np.full((2, 128), -3.0, f)
    b = np.zeros(128, f)
    b[70] = f(3e38)
    lg[0, 70] = f(3e38)
    lg[1, [70, 71]] = [f(-3e38), f(3e38)]   # z = 0 for expert 70, 3e38 for 71
    gi, _, _ = _route_check(lg, b, exact_ties=True)
    assert gi[0, 0] == 70 and gi[1, 0] == 71


@pytest.mark.parametrize("T", [1, 4, 16, 1000, 1024, 1025, 2048, 8189])
def test_permute_parity(T):
    moe = _moe()
    tok = synth.make_tokens(T, 100 + T)
    lg = torch.from_numpy(tok.logits).to(DEV)
    idx, _ = moe.moe_route(lg, torch.from_numpy(tok.bias).to(DEV))
    counts, offsets, perm_src, inv_perm = moe.moe_permute(idx)
    torch.cuda.synchronize()
    ref = O.permute(idx.cpu().numpy().astype(np.int64))
    assert np.array_equal(counts.cpu().numpy(), ref.counts)
    assert np.array_equal(offsets.cpu().numpy(), ref.offsets)
    assert np.array_equal(perm_src.cpu().numpy(), ref.perm_src)
    assert np.array_equal(inv_perm.cpu().numpy(), ref.inv_perm)
    # and the routing that fed it is the oracle's
    assert np.array_equal(idx.cpu().numpy(), O.route(tok.logits, tok.bias).topk_idx)


def test_permute_skewed_and_forced():
    """All tokens on the same 8 experts (counts 8T on 8 experts, 0 elsewhere)."""
    moe = _moe()
    T = 3000
    idx = torch.tensor([[5, 6, 7, 40, 41, 100, 101, 127]] * T, dtype=torch.int32, device=DEV)
    counts, offsets, perm_src, inv_perm = moe.moe_permute(idx)
    ref = O.permute(idx.cpu().numpy().astype(np.int64))
    assert np.array_equal(counts.cpu().numpy(), ref.counts)
    assert np.array_equal(perm_src.cpu().numpy(), ref.perm_src)
    assert np.array_equal(inv_perm.cpu().numpy(), ref.inv_perm)


def _ffn_check(T, seed, forced=None):
    """Runs route -> permute -> expert_ffn and compares every computed y_perm
    row with the oracle's expert FFN of that (token, expert)."""
    moe = _moe()
    W = layer0_weights()
    tok = synth.make_tokens(T, seed)
    if forced is not None:
        tok.bias[:] = 0
        tok.bias[forced] = 1000.0
    x, lg, bias = tokens_dev(tok)
    idx, w = moe.moe_route(lg, bias)
    counts, offsets, perm_src, inv_perm = moe.moe_permute(idx)
    h, y = moe.moe_expert_ffn(x, W.packed, offsets, perm_src)
    torch.cuda.synchronize()
    assert moe.get_device_status(0) == moe.MOE_OK, moe.last_error()
    rr = O.route(tok.logits, tok.bias)
    assert np.array_equal(idx.cpu().numpy(), rr.topk_idx)
    wg, wu, wd = W.host(rr.topk_idx)
    ps = perm_src.cpu().numpy()
    yh = y.double().cpu().numpy()                 # fp16 -> float64 is exact
    xh = O.bf16_bits_to_f64(tok.x_bits)
    ref = np.empty_like(yh)
    for e in np.unique(rr.topk_idx):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        toks = ps[r0:r1] // 8
        ref[r0:r1] = O.expert_ffn(xh[toks], O.bf16_bits_to_f64(wg[e]), O.bf16_bits_to_f64(wu[e]),
                                  O.bf16_bits_to_f64(wd[e]))
    err = O.rel_l2(yh, ref)
    assert err <= REL_L2_TOL, f"y_perm rel-L2 {err:.3e}"
    # per-expert check too, so that one bad tile cannot hide in the total
    for e in np.unique(rr.topk_idx):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        assert O.rel_l2(yh[r0:r1], ref[r0:r1]) <= 2 * REL_L2_TOL, f"expert {e}"
    return err


@pytest.mark.parametrize("T,seed", [(1, 11), (4, 1), (16, 0), (300, 5)])
def test_expert_ffn_parity(T, seed):
    _ffn_check(T, seed)


def test_expert_ffn_dense_special_case():
    """Every token forced onto the same 8 experts: each expert runs a dense
    [T, 1536] x [1536, 1024] GEMM over several 128-row tiles and a ragged tail."""
    _ffn_check(333, 21, forced=[3, 4, 21, 22, 40, 41, 90, 91])


def test_expert_ffn_forced_small_batch():
    """Small batch (weights-as-M kernels) with every token forced onto the same 8
    experts: 200 rows per expert = seven 32-token chunks, the last one ragged."""
    _ffn_check(200, 22, forced=[0, 1, 16, 17, 32, 33, 48, 49])


def test_expert_ffn_forced_large_batch():
    """Large batch (128-row token tiles, no padding zeroing) with every token
    forced onto the same 8 experts: 1500 rows per expert = 12 tiles, the last ragged."""
    _ffn_check(1500, 24, forced=[2, 3, 50, 51, 64, 65, 126, 127])


def test_combine_parity():
    moe = _moe()
    rng = np.random.default_rng(9)
    T = 37
    y16 = rng.standard_normal((T * 8, 1536)).astype(np.float16)
    w = rng.random((T, 8)).astype(np.float32)
    inv = rng.permutation(T * 8).astype(np.int32)
    res_bits = synth.f32_to_bf16_bits(rng.standard_normal((T, 1536)).astype(np.float32))
    out = moe.moe_combine(torch.from_numpy(y16).to(DEV), torch.from_numpy(w).to(DEV),
                          torch.from_numpy(inv).to(DEV), residual=to_dev_bf16(res_bits))
    torch.cuda.synchronize()
    yv = y16.astype(np.float64)
    ref = O.bf16_bits_to_f64(res_bits) + np.einsum("ts,tsh->th", w.astype(np.float64),
                                                   yv[inv.reshape(T, 8)])
    got = O.bf16_bits_to_f64(to_host_bits(out))
    # fp32 accumulation then one bf16 rounding: within one bf16 ulp (2**-8 relative)
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-6)


def test_generator_device_bytes_equal_host_bytes():
    """The oracle reads expert weights made on the device by the input
    generator; they are the same bytes as the host generator's."""
    W = layer0_weights()
    for which, t in ((synth.W_GATE, W.wg), (synth.W_DOWN, W.wd)):
        host = synth.weight_bits_np(0, 0, which, experts=[0, 77, 127])
        assert np.array_equal(to_host_bits(t[[0, 77, 127]]), host)


@pytest.mark.parametrize("T,seed,forced", [(1, 31, None), (16, 32, None), (77, 33, None),
                                           (200, 34, [0, 1, 16, 17, 32, 33, 48, 49]),
                                           (256, 35, None), (333, 36, None),
                                           (1500, 37, [2, 3, 50, 51, 64, 65, 126, 127]),
                                           (2048, 38, None), (8189, 39, None)])
def test_expert_ffn_single_launch_equals_two_launches(T, seed, forced):
    """moe_expert_ffn runs gate/up and down in one launch (weights-as-M tiles
    for T <= 256, 128-row token tiles above), a down tile starting when its
    expert's gate/up tiles have stored h.  Its h and y_perm must equal, bit for
    bit, those of the two separate launches (moe_expert_gate_up then
    moe_expert_down), on repeated calls: a down tile that read h too early
    would differ."""
    moe = _moe()
    W = layer0_weights()
    tok = synth.make_tokens(T, seed)
    if forced is not None:
        tok.bias[:] = 0
        tok.bias[forced] = 1000.0
    x, lg, bias = tokens_dev(tok)
    idx, w = moe.moe_route(lg, bias)
    counts, offsets, perm_src, inv_perm = moe.moe_permute(idx)
    h2 = moe.moe_expert_gate_up(x, W.packed, offsets, perm_src)
    y2 = moe.moe_expert_down(h2, W.packed, offsets)
    for _ in range(3):
        h1 = torch.full_like(h2, float("nan"))
        y1 = torch.full_like(y2, float("nan"))
        moe.moe_expert_ffn(x, W.packed, offsets, perm_src, h1, y1)
        torch.cuda.synchronize()
        assert moe.get_device_status(0) == moe.MOE_OK, moe.last_error()
        assert torch.equal(h1.view(torch.int16), h2.view(torch.int16))
        assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
