"""Pins of the oracle on the second MoE shape (route_e256 and the layer with
256 experts and 6 slots):

* the kept groups by exhaustive search over all 70 four-group subsets, with
  group scores from an independent top-2 (sorting each group), and the
  chosen experts by dominance (each chosen score >= every unchosen
  candidate's, ties to the lower index), slot order and weights from their
  definitions;
* the all-equal special case (groups 0-3, experts 0-5, weights 1/6);
* a token driven to one expert above index 127, whose layer output is that
  expert's dense FFN times its weight (experts above 128 are indexed
  correctly)."""
import itertools

import numpy as np

import oracle as O
from group_limited_routed_moe_b200 import synth

E, G, KEEP, K = 256, 8, 4, 6


def _sig(z):
    return 1.0 / (1.0 + np.exp(-z))


def test_route_e256_groups_by_search_and_experts_by_dominance():
    rng = np.random.default_rng(5)
    T = 24
    lg = rng.standard_normal((T, E)).astype(np.float32)
    b = (0.1 * rng.standard_normal(E)).astype(np.float32)
    rr = O.route_e256(lg, b)
    assert rr.topk_idx.shape == (T, K) and rr.kept_groups.shape == (T, KEEP)
    s = _sig(lg.astype(np.float64) + b.astype(np.float64))
    for t in range(T):
        gs = [np.sort(s[t, 32 * j:32 * j + 32])[-2:].sum() for j in range(G)]
        best = max(itertools.combinations(range(G), KEEP), key=lambda sub: (sum(gs[j] for j in sub),
                                                                           [-j for j in sub]))
        assert sorted(rr.kept_groups[t].tolist()) == sorted(best)
        cand = [e for j in best for e in range(32 * j, 32 * j + 32)]
        chosen = rr.topk_idx[t].tolist()
        assert len(set(chosen)) == K and set(chosen) <= set(cand)
        rest = [e for e in cand if e not in chosen]
        assert min(s[t, chosen]) >= max(s[t, rest])
        assert all(s[t, chosen[i]] >= s[t, chosen[i + 1]] for i in range(K - 1))
        w = _sig(lg[t, chosen].astype(np.float64))
        assert np.allclose(rr.topk_w[t], w / w.sum(), rtol=1e-12)


def test_route_e256_all_equal():
    rr = O.route_e256(np.zeros((3, E), np.float32), None)
    assert rr.kept_groups.tolist() == [[0, 1, 2, 3]] * 3
    assert rr.topk_idx.tolist() == [[0, 1, 2, 3, 4, 5]] * 3
    assert np.allclose(rr.topk_w, 1.0 / 6.0, rtol=1e-15)


def test_layer_e256_expert_above_127():
    tok = synth.make_tokens(1, 77)
    lg = np.full((1, E), -30.0, np.float32)
    lg[0, 200] = 30.0                      # expert 200 (group 6) first
    lg[0, 192:224] = np.maximum(lg[0, 192:224], 1.0)
    bits = synth.layer_weights_np(0, 0, [5])  # any bf16 weights, placed at expert 200 only
    wg = np.zeros((E, 1536, 512), np.uint16); wu = np.zeros_like(wg)
    wd = np.zeros((E, 512, 1536), np.uint16)
    wg[200], wu[200], wd[200] = bits[0][0], bits[1][0], bits[2][0]
    rr = O.route_e256(lg, None)
    assert rr.topk_idx[0, 0] == 200
    out = O.moe_layer(tok.x_bits, lg, None, wg, wu, wd, route_result=rr)
    x = O.bf16_bits_to_f64(tok.x_bits)
    dense = O.expert_ffn(x, O.bf16_bits_to_f64(wg[200]), O.bf16_bits_to_f64(wu[200]),
                         O.bf16_bits_to_f64(wd[200]))
    assert np.allclose(out, rr.topk_w[0, 0] * dense, rtol=1e-12, atol=1e-15)
    assert np.abs(dense).max() > 1e-2
