"""Noise floor of the 23-layer stack's accumulated update, from the oracle alone.

Both the GPU and the oracle round the residual stream to bf16 after every
layer, h <- bf16(h + moe(h)), but they round slightly different values: the
GPU's MoE output carries a small relative error (fp16 intermediates, bf16
inputs of the tensor-core GEMMs, fp32 accumulation order).  Whenever that
error moves a value across a bf16 rounding boundary, the two streams differ by
one bf16 ulp of h from then on, and those flips add up over the layers.  How
much they add up to is a property of the stack, not of any implementation, so
it is measured here on the oracle itself: the oracle stack is run once as it
stands and once with every layer's float64 update multiplied element-wise by
(1 + EPS * N(0, 1)) (seeded) before the bf16 rounding.  The rel-L2 between
the two accumulated updates h_23 - x is the floor that an implementation with
a per-layer relative error of EPS on the update cannot get under.

EPS = 2e-3 is the layer tolerance's expected error (about 2e-3 against the
float64 layer).  The floor hardly depends on EPS: measured on this stack (max
of two seeds, 2 tokens) it is 0.73e-2 at EPS = 1e-6, 0.88e-2 at 1e-5, 1.1e-2
at 1e-4, 1.33e-2 at 5e-4, 1.47e-2 at 1e-3, 1.72e-2 at 2e-3 and 1.97e-2 at
4e-3.  A single early flip is enough: the one-ulp difference it leaves in h
moves later layers' sums across further rounding boundaries, so the two
streams part by about 1% of the update whatever the size of the first
difference.  The stack test bounds the GPU's update error by UPDATE_FACTOR x
the floor at EPS = 2e-3; a wrong expert, weight or sign in any layer would
be off by O(1).

The routing of every layer comes from given per-layer logits (it does not
depend on the activations), so both runs route identically and the floor is
purely numerical.  Only the experts a layer's tokens touch are generated.
"""
from __future__ import annotations

import dataclasses

import numpy as np

import oracle as O
from group_limited_routed_moe_b200 import synth

N_LAYERS = 23
SEED = 4            # the stack's weight and logit seed
EPS = 2e-3          # per-layer relative error of the update in the perturbed run
FLOOR_TOKENS = 2    # tokens of the floor run (2 x 1536 update elements per run)
PERT_SEEDS = (101, 102)

# The floor as computed by update_noise_floor() (pinned by
# tests/test_oracle_layer.py::test_stack_update_noise_floor), and the factor
# the GPU stack test allows above it.
UPDATE_FLOOR = 1.72e-2
UPDATE_FACTOR = 1.5


def _compact(rr: O.RouteResult):
    """The layer's touched experts and the routing re-indexed onto them."""
    experts = np.unique(rr.topk_idx)
    return experts, dataclasses.replace(rr, topk_idx=np.searchsorted(experts, rr.topk_idx))


def update_noise_floor(T: int = FLOOR_TOKENS, seeds=PERT_SEEDS, eps: float = EPS):
    """Returns (floor, per-seed rel-L2 list, the unperturbed h_23 bits).

    floor = max over the perturbation seeds of rel_l2(h_23' - x, h_23 - x).
    """
    x_bits = synth.make_tokens(T, SEED).x_bits
    h_ref = x_bits
    h_pert = [x_bits for _ in seeds]
    rngs = [np.random.default_rng(s) for s in seeds]
    for layer in range(N_LAYERS):
        lg, b = synth.layer_logits(T, SEED, layer)
        experts, rr = _compact(O.route(lg, b))
        wg, wu, wd = synth.layer_weights_np(SEED, layer, experts)
        upd = O.moe_layer(h_ref, lg, b, wg, wu, wd, route_result=rr)
        h_ref = O.f64_to_bf16_bits(O.bf16_bits_to_f64(h_ref) + upd)
        for i, rng in enumerate(rngs):
            u = O.moe_layer(h_pert[i], lg, b, wg, wu, wd, route_result=rr)
            u = u * (1.0 + eps * rng.standard_normal(u.shape))
            h_pert[i] = O.f64_to_bf16_bits(O.bf16_bits_to_f64(h_pert[i]) + u)
    x = O.bf16_bits_to_f64(x_bits)
    ref_upd = O.bf16_bits_to_f64(h_ref) - x
    errs = [O.rel_l2(O.bf16_bits_to_f64(h) - x, ref_upd) for h in h_pert]
    return max(errs), errs, h_ref
