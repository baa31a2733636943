"""Pins for the oracle's routing (no GPU).

The oracle's ``route`` is checked against things other than itself:
brute-force enumeration of group subsets and expert subsets on reduced grids,
an exhaustive group-subset check plus a swap-dominance check on the real grid,
a hand-worked example (tests/golden/route_worked_example.json), and closed-form
special cases (all-equal scores, a dominant expert, an excluded group, ties).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _draw(rng, T, E):
    lg = rng.standard_normal((T, E)).astype(np.float32)
    b = (0.1 * rng.standard_normal(E)).astype(np.float32)
    return lg, b


@pytest.mark.parametrize("grid", [(16, 4, 2, 3), (24, 4, 2, 4), (32, 8, 3, 5), (12, 3, 1, 2)])
def test_route_matches_bruteforce_on_small_grids(grid):
    """Every token's routing equals exhaustive search over all group subsets
    and all expert subsets (skipping tokens whose margins are float-ties)."""
    E, G, keep, k = grid
    rng = np.random.default_rng(1234 + E)
    lg, b = _draw(rng, 60, E)
    rr = O.route(lg, b, n_groups=G, keep=keep, topk=k)
    checked = 0
    for t in range(lg.shape[0]):
        if rr.group_margin[t] < 1e-12 or rr.expert_margin[t] < 1e-12:
            continue
        kept, chosen, w = O.route_bruteforce(lg[t], b, G, keep, k)
        assert sorted(rr.kept_groups[t].tolist()) == kept
        assert rr.topk_idx[t].tolist() == chosen
        np.testing.assert_allclose(rr.topk_w[t], w, rtol=0, atol=1e-15)
        checked += 1
    assert checked >= 55


def test_route_full_grid_group_enumeration_and_dominance():
    """Real grid (128 experts, 8 groups of 16, keep 4, top 8): the kept groups
    maximise the summed group score over all C(8,4)=70 subsets, each group
    score being the best pair sum found by scanning all member pairs; every
    chosen expert scores at least as much as every unchosen candidate."""
    rng = np.random.default_rng(7)
    lg, b = _draw(rng, 40, 128)
    rr = O.route(lg, b)
    z = lg.astype(np.float64) + b.astype(np.float64)
    s = 1.0 / (1.0 + np.exp(-z))
    for t in range(40):
        gs = []
        for j in range(8):
            mem = s[t, 16 * j:16 * (j + 1)]
            gs.append(max(mem[a] + mem[c] for a in range(16) for c in range(a + 1, 16)))
        best = max(itertools.combinations(range(8), 4), key=lambda sub: sum(gs[j] for j in sub))
        assert sorted(rr.kept_groups[t].tolist()) == sorted(best)
        cand = [e for j in best for e in range(16 * j, 16 * (j + 1))]
        chosen = rr.topk_idx[t].tolist()
        assert len(set(chosen)) == 8 and set(chosen) <= set(cand)
        rest = [e for e in cand if e not in chosen]
        assert min(s[t, chosen]) >= max(s[t, rest])
        # slot order: descending score
        assert all(s[t, chosen[i]] >= s[t, chosen[i + 1]] for i in range(7))
        # at most 4 groups touched
        assert len({e // 16 for e in chosen}) <= 4


def test_route_worked_example():
    """Hand-worked example: bias steers selection, weights ignore the bias."""
    g = json.load(open(os.path.join(GOLDEN, "route_worked_example.json")))
    grid = g["grid"]
    rr = O.route(np.array([g["logits"]], np.float32), np.array(g["bias"], np.float32),
                 n_groups=grid["n_groups"], keep=grid["keep"], topk=grid["topk"])
    assert rr.kept_groups[0].tolist() == g["kept_groups"]
    assert rr.topk_idx[0].tolist() == g["topk_idx"]
    np.testing.assert_allclose(rr.topk_w[0], g["topk_w"], rtol=0, atol=1e-15)
    assert abs(rr.topk_w[0][0] - g["topk_w_if_bias_were_included"][0]) > 1e-3


def test_route_all_equal_scores():
    """All logits and biases equal: groups 0-3 kept, experts 0..7 in order, w = 1/8."""
    lg = np.full((3, 128), 0.3, np.float32)
    b = np.full(128, -0.2, np.float32)
    rr = O.route(lg, b)
    for t in range(3):
        assert rr.kept_groups[t].tolist() == [0, 1, 2, 3]
        assert rr.topk_idx[t].tolist() == list(range(8))
        assert np.all(rr.topk_w[t] == 0.125)


def test_route_dominant_expert_and_excluded_group():
    rng = np.random.default_rng(3)
    lg, b = _draw(rng, 16, 128)
    lg[:, 77] = 12.0                    # dominant expert -> slot 0
    b[16:32] = -40.0                    # group 1 can never win a slot
    rr = O.route(lg, b)
    assert np.all(rr.topk_idx[:, 0] == 77)
    assert not np.any((rr.topk_idx >= 16) & (rr.topk_idx < 32))
    assert not np.any(rr.kept_groups == 1)


def test_route_ties_prefer_lower_index():
    """Exactly equal expert scores and exactly equal group scores are ordered
    by index."""
    lg = np.full((1, 128), -3.0, np.float32)
    # groups 2 and 5 get identical top pairs; 6 more experts in group 2/5 tie
    for e in (32, 33, 80, 81):
        lg[0, e] = 2.0
    for e in (34, 35, 82, 83):
        lg[0, e] = 1.0
    rr = O.route(lg, None)
    assert rr.kept_groups[0].tolist()[:2] == [2, 5]
    assert rr.topk_idx[0].tolist() == [32, 33, 80, 81, 34, 35, 82, 83]


def test_route_weights_sum_to_one_and_positive():
    rng = np.random.default_rng(11)
    lg, b = _draw(rng, 500, 128)
    rr = O.route(lg, b)
    assert np.all(rr.topk_w > 0)
    np.testing.assert_allclose(rr.topk_w.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    # weights are sigmoid(logit) ratios: w_i / w_j == sig(l_i) / sig(l_j)
    sig = 1.0 / (1.0 + np.exp(-lg.astype(np.float64)))
    ratio = rr.topk_w[:, 0] / rr.topk_w[:, 1]
    ref = sig[np.arange(500), rr.topk_idx[:, 0]] / sig[np.arange(500), rr.topk_idx[:, 1]]
    np.testing.assert_allclose(ratio, ref, rtol=1e-13)


def test_route_token_independence():
    """Routing of a token does not depend on the other tokens."""
    rng = np.random.default_rng(5)
    lg, b = _draw(rng, 64, 128)
    full = O.route(lg, b)
    perm = rng.permutation(64)
    part = O.route(lg[perm], b)
    assert np.array_equal(part.topk_idx, full.topk_idx[perm])
    assert np.array_equal(part.topk_w, full.topk_w[perm])


def test_sigmoid_closed_forms():
    assert O.sigmoid(np.array([0.0]))[0] == 0.5
    z = np.linspace(-20, 20, 401)
    np.testing.assert_allclose(O.sigmoid(z) + O.sigmoid(-z), 1.0, atol=1e-15)
    assert abs(O.sigmoid(np.array([1.0]))[0] - 1 / (1 + math.e ** -1)) < 1e-16


def test_combine_weights_against_plain_formula_and_limit():
    """The weights equal sigmoid(l)/sum sigmoid(l) wherever that is finite, and
    when every sigmoid underflows they tend to the softmax of the logits."""
    rng = np.random.default_rng(21)
    for scale, shift in ((1.0, 0.0), (5.0, -20.0), (3.0, 15.0), (0.5, -3.0)):
        l = rng.standard_normal((200, 8)) * scale + shift
        plain = O.sigmoid(l) / O.sigmoid(l).sum(axis=1, keepdims=True)
        np.testing.assert_allclose(O.combine_weights(l), plain, rtol=1e-13, atol=1e-16)
    l = -800.0 - rng.random((20, 8)) * 30.0
    soft = np.exp(l - l.max(axis=1, keepdims=True))
    soft /= soft.sum(axis=1, keepdims=True)
    w = O.combine_weights(l)
    assert np.all(np.isfinite(w))
    np.testing.assert_allclose(w, soft, rtol=1e-12, atol=1e-300)
