"""Shared set-up for the GPU parity tests: seeded inputs on the device, packed
weights, and host copies for the float64 oracle.

Inputs come only from ``group_limited_routed_moe_b200.synth`` (the seeded
generator); expected values come only from ``oracle``.  Nothing here reads a
result of the CUDA path back as an oracle input.
"""
from __future__ import annotations

import functools

import numpy as np
import torch

import oracle as O
from group_limited_routed_moe_b200 import synth

DEV = torch.device("cuda:0")

# Layer-output tolerance: rel-L2 against the float64 oracle.  bf16 rounding of
# h, y_perm and the output each add about 2**-9/sqrt(3) = 1.1e-3 relative
# (RMS), so about 2e-3 is expected; the bound is 5e-3.
REL_L2_TOL = 5e-3
# Routing weights: fp32 output of a float64 ratio.
W_TOL = 1e-6


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(DEV).view(torch.bfloat16)


def to_host_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class LayerWeights:
    """One layer's expert weights: generated on the device, packed, and
    fetched to the host per expert on demand for the oracle."""

    def __init__(self, seed: int, layer: int):
        self.seed, self.layer = seed, layer
        self.wg = synth.weight_bits_torch(seed, layer, synth.W_GATE, DEV)
        self.wu = synth.weight_bits_torch(seed, layer, synth.W_UP, DEV)
        self.wd = synth.weight_bits_torch(seed, layer, synth.W_DOWN, DEV)
        from group_limited_routed_moe_b200 import moe
        self.packed = moe.moe_pack_weights(self.wg, self.wu, self.wd)
        torch.cuda.synchronize()

    def host(self, experts) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
        """Full-size [128,...] host arrays with the given experts filled in."""
        experts = np.unique(np.asarray(experts))
        sel = torch.as_tensor(experts, device=DEV)
        out = []
        for t in (self.wg, self.wu, self.wd):
            a = np.zeros((128,) + tuple(t.shape[1:]), np.uint16)
            a[experts] = to_host_bits(t[sel])
            out.append(a)
        return tuple(out)

    def drop_unpacked(self):
        self.wg = self.wu = self.wd = None


@functools.lru_cache(maxsize=1)
def layer0_weights() -> LayerWeights:
    return LayerWeights(0, 0)


def extreme_logits():
    """Router logits at the ends of the sigmoid, with a bias: 8 tokens.

    z in (10, 36): distinct scores close to 1; z > 37: float64 sigmoid == 1.0
    exactly, so ties are broken by index; z < -745: the sigmoid underflows to 0
    (ties, and weights that only the shifted ratio keeps finite); mixed with
    ordinary values."""
    rng = np.random.default_rng(17)
    lg = rng.standard_normal((8, 128)).astype(np.float32)
    lg[0, [5, 9, 70, 71]] = [40.0, 45.0, 50.0, 38.0]              # saturated ties in slot order
    lg[1, [3, 4, 20, 21, 22]] = [12.0, 12.5, 30.0, 29.0, 35.5]     # large but distinct
    lg[2, :] = -800.0                                              # everything underflows
    lg[2, [100, 101]] = [-1.0, 0.5]
    lg[3, :64] = -760.0
    lg[3, 64:] = -900.0
    lg[4, [0, 16, 32, 48, 64, 80, 96, 112]] = 60.0                 # one saturated expert per group
    lg[5, 16:32] = 11.0                                            # a whole group tied above 10
    lg[6, ::2] = 37.5
    lg[7, :] = 0.0
    b = (0.1 * rng.standard_normal(128)).astype(np.float32)
    return lg, b


def tokens_dev(tok: synth.TokenInputs, T_buf: int | None = None):
    T = tok.x_bits.shape[0]
    T_buf = T_buf or T
    x = torch.zeros((T_buf, 1536), dtype=torch.bfloat16, device=DEV)
    x[:T] = to_dev_bf16(tok.x_bits)
    lg = torch.zeros((T_buf, 128), dtype=torch.float32, device=DEV)
    lg[:T] = torch.from_numpy(tok.logits).to(DEV)
    bias = torch.from_numpy(tok.bias).to(DEV)
    return x, lg, bias


def oracle_layer(tok: synth.TokenInputs, weights: LayerWeights, rows=None):
    """Oracle output (float64) for all tokens or for ``rows``."""
    x, lg = tok.x_bits, tok.logits
    if rows is not None:
        x, lg = x[rows], lg[rows]
    rr = O.route(lg, tok.bias)
    wg, wu, wd = weights.host(rr.topk_idx)
    return O.moe_layer(x, lg, tok.bias, wg, wu, wd, route_result=rr), rr
