"""Seeded synthetic inputs for the routed MoE layer.

This module holds no arithmetic of the method: only random draws and dtype
packing.  It is the one piece of code that both the CUDA path (tests, bench,
smoke) and the float64 oracle consume, so that both see identical bytes.  It
never imports the CUDA binding or the oracle.

Recipe (the distributions of the layer's workloads):

* activations x ~ N(0, 1), stored as bf16 [T, 1536];
* router logits ~ N(0, 1) fp32 [T, 128], per-expert bias ~ N(0, 0.1) fp32 [128];
* the skewed prefill adds +2.0 to the logits of 16 "hot" experts drawn
  without replacement (Zipf-like load imbalance);
* expert weights ~ N(0, 0.02), bf16: W_gate, W_up [128, 1536, 512] and
  W_down [128, 512, 1536] per layer, used as x @ W.

Shared experts (when a layer has them) come from the same generator under
seed + 1000, expert indices 0, 1, ...

Activations, logits and bias are drawn with NumPy's PCG64 (host).  Expert
weights (up to 23 x 604 MB) come from a counter-based generator so that the
same bytes can be produced on the device in bulk or on the host for any
single expert: a 32-bit integer hash of (seed, layer, matrix, expert, element)
picks one of 65,536 normal quantiles Phi^-1((k + 1/2) / 65536), scaled by
0.02 and rounded once to bf16.  After bf16 rounding this is indistinguishable
from N(0, 0.02) except that the tails are cut at 4.33 sigma.

Block-FP8 expert weights (the synthetic counterpart of a block-FP8
checkpoint) are those bf16 weights written the way such a file is written:
per 128 x 128 block a scale s, and every weight stored as the FP8 E4M3 code
nearest to w / s (round to nearest even, by PyTorch's float8_e4m3fn cast).
Scale modes: "pow2" takes the smallest power of two with max|w| <= 448 s (the
power-of-two block scales of UE8M0-style checkpoints); "amax" takes
s = fp32(max|w| / 448).  This is input synthesis: the layer only reads codes
and scales.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

HIDDEN = 1536
INTER = 512
N_EXPERTS = 128
TOPK = 8
WEIGHT_STD = 0.02

# matrix ids inside a layer
W_GATE, W_UP, W_DOWN, W_ROUTER = 0, 1, 2, 3
_W_SHAPES = {W_GATE: (HIDDEN, INTER), W_UP: (HIDDEN, INTER), W_DOWN: (INTER, HIDDEN),
             W_ROUTER: (HIDDEN, N_EXPERTS)}


# ----------------------------------------------------------------------------
# dtype packing
# ----------------------------------------------------------------------------

def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> raw bf16 bits (uint16), round to nearest even (finite input)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (r >> np.uint32(16)).astype(np.uint16)


# ----------------------------------------------------------------------------
# counter-based weight generator
# ----------------------------------------------------------------------------

_M1 = 0x7FEB352D
_M2 = 0x846CA68B
_TABLE_BITS: np.ndarray | None = None


def _quantile_table_bits() -> np.ndarray:
    """65,536 bf16 values: bf16(float32(Phi^-1((k + 0.5) / 65536)) * 0.02)."""
    global _TABLE_BITS
    if _TABLE_BITS is None:
        from scipy.special import ndtri
        q = ndtri((np.arange(65536, dtype=np.float64) + 0.5) / 65536.0).astype(np.float32)
        _TABLE_BITS = f32_to_bf16_bits(q * np.float32(WEIGHT_STD))
    return _TABLE_BITS


def _mix32_np(x: np.ndarray) -> np.ndarray:
    """32-bit avalanche hash (xorshift-multiply, 'lowbias32' constants), uint32."""
    x = x.astype(np.uint32, copy=True)
    x ^= x >> np.uint32(16)
    x *= np.uint32(_M1)
    x ^= x >> np.uint32(15)
    x *= np.uint32(_M2)
    x ^= x >> np.uint32(16)
    return x


def _stream_keys(seed: int, layer: int, which: int, experts: np.ndarray):
    sid = ((np.uint64(seed) * np.uint64(64) + np.uint64(layer)) * np.uint64(4)
           + np.uint64(which)) * np.uint64(128) + experts.astype(np.uint64)
    sid = (sid & np.uint64(0xFFFFFFFF)).astype(np.uint32)
    k1 = _mix32_np(sid ^ np.uint32(0xA511E9B3))
    k2 = _mix32_np(sid ^ np.uint32(0x63D83595))
    return k1, k2


def weight_bits_np(seed: int, layer: int, which: int,
                   experts=None) -> np.ndarray:
    """Expert matrix ``which`` of ``layer`` as bf16 bits [len(experts), rows, cols]."""
    experts = np.arange(N_EXPERTS) if experts is None else np.asarray(experts)
    rows, cols = _W_SHAPES[which]
    n = rows * cols
    k1, k2 = _stream_keys(seed, layer, which, experts)
    i = np.arange(n, dtype=np.uint32)
    table = _quantile_table_bits()
    out = np.empty((len(experts), n), dtype=np.uint16)
    for j in range(len(experts)):
        u = _mix32_np(_mix32_np(i ^ k1[j]) ^ k2[j])
        out[j] = table[u >> np.uint32(16)]
    return out.reshape(len(experts), rows, cols)


def router_weight_bits_np(seed: int, layer: int) -> np.ndarray:
    """Router matrix W_router [1536, 128] of ``layer`` as bf16 bits (one matrix,
    from the same counter generator as the expert weights: N(0, 0.02))."""
    return weight_bits_np(seed, layer, W_ROUTER, experts=[0])[0]


def layer_weights_np(seed: int, layer: int, experts=None):
    """(W_gate, W_up, W_down) bf16 bits of one layer on the host."""
    return tuple(weight_bits_np(seed, layer, w, experts) for w in (W_GATE, W_UP, W_DOWN))


SHARED_SEED_OFFSET = 1000


def shared_weights_np(seed: int, layer: int, n_shared: int):
    """(W_gate, W_up, W_down) bf16 bits of ``n_shared`` shared experts of
    ``layer``: the generator's expert matrices 0 .. n_shared-1 of seed
    seed + 1000 (a stream no routed expert uses)."""
    ex = np.arange(n_shared)
    return tuple(weight_bits_np(seed + SHARED_SEED_OFFSET, layer, w, ex)
                 for w in (W_GATE, W_UP, W_DOWN))


def _mix32_torch(x):
    """Same hash as ``_mix32_np`` on int64 tensors holding values < 2**32.

    Multiplication modulo 2**32 is split into 16-bit halves so that no
    intermediate leaves the int64 range on any device.
    """
    def mul32(v, c):
        lo = (v & 0xFFFF) * c
        hi = (((v >> 16) * c) & 0xFFFF) << 16
        return (lo + hi) & 0xFFFFFFFF
    x = x ^ (x >> 16)
    x = mul32(x, _M1)
    x = x ^ (x >> 15)
    x = mul32(x, _M2)
    x = x ^ (x >> 16)
    return x


def weight_bits_torch(seed: int, layer: int, which: int, device, out=None):
    """Same bytes as ``weight_bits_np`` for all 128 experts, made on ``device``.

    Returns (or fills) a torch.bfloat16 tensor [128, rows, cols].
    """
    import torch
    rows, cols = _W_SHAPES[which]
    n = rows * cols
    k1, k2 = _stream_keys(seed, layer, which, np.arange(N_EXPERTS))
    table = torch.from_numpy(_quantile_table_bits().view(np.int16)).to(device)
    if out is None:
        out = torch.empty((N_EXPERTS, rows, cols), dtype=torch.bfloat16, device=device)
    flat = out.view(N_EXPERTS, n).view(torch.int16)
    i = torch.arange(n, dtype=torch.int64, device=device)[None, :]
    k1t = torch.from_numpy(k1.astype(np.int64)).to(device)[:, None]
    k2t = torch.from_numpy(k2.astype(np.int64)).to(device)[:, None]
    step = 16
    for e0 in range(0, N_EXPERTS, step):
        u = _mix32_torch(_mix32_torch(i ^ k1t[e0:e0 + step]) ^ k2t[e0:e0 + step])
        flat[e0:e0 + step].copy_(table[u >> 16])
    return out


# ----------------------------------------------------------------------------
# block-FP8 expert weights
# ----------------------------------------------------------------------------

FP8_BLOCK = 128
FP8_MAX = 448.0


def _quantize_block_fp8(w, mode: str):
    """torch float32 [n, R, C] -> (uint8 codes [n, R, C], fp32 scales [n, R/128, C/128])."""
    import torch
    n, R, C = w.shape
    blk = w.reshape(n, R // FP8_BLOCK, FP8_BLOCK, C // FP8_BLOCK, FP8_BLOCK)
    amax = blk.abs().amax(dim=(2, 4))
    if mode == "pow2":
        # smallest e with amax <= 448 * 2**e; amax = m * 2**k, 0.5 <= m < 1, 448 = 0.875 * 2**9
        m, k = torch.frexp(amax)
        e = k - 9 + (m > 0.875).to(k.dtype)
        scale = torch.ldexp(torch.ones_like(amax), e)
    elif mode == "amax":
        scale = amax / FP8_MAX
    else:
        raise ValueError(f"unknown scale mode {mode!r}")
    scale = torch.where(amax > 0, scale, torch.ones_like(scale)).to(torch.float32)
    q = (blk / scale[:, :, None, :, None]).to(torch.float8_e4m3fn)
    return q.reshape(n, R, C).view(torch.uint8), scale


def fp8_weights_np(seed: int, layer: int, which: int, experts=None, mode: str = "pow2"):
    """Block-FP8 form of expert matrix ``which`` of ``layer`` on the host:
    (codes uint8 [len(experts), R, C], scales float32 [len(experts), R/128, C/128])."""
    import torch
    bits = weight_bits_np(seed, layer, which, experts)
    w = (torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)).to(torch.float32)
    q, s = _quantize_block_fp8(w, mode)
    return q.numpy(), s.numpy()


def fp8_weights_torch(seed: int, layer: int, which: int, device, mode: str = "pow2"):
    """Same bytes as ``fp8_weights_np`` for all 128 experts, made on ``device``."""
    import torch
    w = weight_bits_torch(seed, layer, which, device)
    codes = torch.empty(w.shape, dtype=torch.uint8, device=device)
    scales = []
    for e0 in range(0, N_EXPERTS, 16):  # bounded float32 temporaries
        q, s = _quantize_block_fp8(w[e0:e0 + 16].to(torch.float32), mode)
        codes[e0:e0 + 16].copy_(q)
        scales.append(s)
    return codes, torch.cat(scales)


def fp8_scale_jitter(shape, seed: int) -> np.ndarray:
    """Per-block factors 2**j, j uniform in {-2, ..., 2}, from PCG64(seed):
    multiplied into power-of-two scales they give blocks of different scales
    (the generator's own scales are nearly uniform, since every block of
    N(0, 0.02) weights has about the same max |w|)."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 77])))
    return np.exp2(rng.integers(-2, 3, size=shape)).astype(np.float32)


# NVFP4 form of the synthetic experts, as ModelOpt quantises a linear weight
# [out, in]: tensor scale g from the matrix's max |w| (so that the largest
# block scale is at most 448), block scale = E4M3(max |w| of 16 / 6 / g)
# rounded to nearest even, code = E2M1(w / (block scale * g)) rounded to
# nearest even and saturated at 6.  mode "pow2" rounds g up to a power of two
# (the dequantised weights are then bf16 values), "amax" keeps it as is.
FP4_BLOCK = 16
E2M1_MAX = 6.0
_E2M1_MIDS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)  # between the 8 magnitudes


def _encode_e2m1(q):
    """torch float32 (|q| <= 6) -> uint8 E2M1 codes, nearest, ties to even."""
    import torch
    mids = torch.tensor(_E2M1_MIDS, dtype=torch.float32, device=q.device)
    a = q.abs()
    idx = torch.bucketize(a, mids)  # mids[idx-1] < a <= mids[idx]: ties go down
    tie = (idx < len(_E2M1_MIDS)) & (a == mids[idx.clamp(max=len(_E2M1_MIDS) - 1)])
    idx = idx + (tie & (idx % 2 == 1)).to(idx.dtype)  # ...unless that magnitude is odd
    sign = ((q < 0) & (idx > 0)).to(idx.dtype) << 3
    return (idx | sign).to(torch.uint8)


def _quantize_nvfp4(w, mode: str):
    """torch float32 [n, out, in] -> (packed uint8 [n, out, in/2], block-scale
    E4M3 codes uint8 [n, out, in/16], tensor scales float32 [n])."""
    import torch
    n, R, C = w.shape
    amax = w.abs().amax(dim=(1, 2))
    g = amax / torch.tensor(E2M1_MAX * FP8_MAX, dtype=torch.float32, device=w.device)
    if mode == "pow2":
        m, k = torch.frexp(g)  # g = m * 2**k, 0.5 <= m < 1: the next power of two is 2**k
        g = torch.ldexp(torch.ones_like(g), k - (m == 0.5).to(k.dtype))
    elif mode != "amax":
        raise ValueError(f"unknown scale mode {mode!r}")
    g = torch.where(amax > 0, g, torch.ones_like(g)).to(torch.float32)
    blk = w.reshape(n, R, C // FP4_BLOCK, FP4_BLOCK)
    bmax = blk.abs().amax(dim=-1)
    sc = (bmax / E2M1_MAX / g[:, None, None]).to(torch.float8_e4m3fn)
    sc = torch.where(sc.to(torch.float32) > 0, sc,
                     torch.full_like(sc, 0x01, dtype=torch.uint8).view(torch.float8_e4m3fn))
    den = sc.to(torch.float32) * g[:, None, None]
    q = (blk / den[..., None]).clamp(-E2M1_MAX, E2M1_MAX)
    codes = _encode_e2m1(q).reshape(n, R, C)
    packed = codes[..., 0::2] | (codes[..., 1::2] << 4)
    return packed, sc.view(torch.uint8), g


def _linear_form(w):
    """[n, K, N] (x W form) -> [n, N, K] (a linear layer's [out, in] form)."""
    return w.transpose(1, 2).contiguous()


def nvfp4_weights_np(seed: int, layer: int, which: int, experts=None, mode: str = "pow2"):
    """NVFP4 form of expert matrix ``which`` of ``layer`` on the host, [out, in]:
    (packed codes uint8 [n, out, in/2], block scales uint8 [n, out, in/16],
    tensor scales float32 [n])."""
    import torch
    bits = weight_bits_np(seed, layer, which, experts)
    w = (torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)).to(torch.float32)
    q, s, g = _quantize_nvfp4(_linear_form(w), mode)
    return q.numpy(), s.numpy(), g.numpy()


def nvfp4_weights_torch(seed: int, layer: int, which: int, device, mode: str = "pow2"):
    """Same bytes as ``nvfp4_weights_np`` for all 128 experts, made on ``device``."""
    import torch
    w = weight_bits_torch(seed, layer, which, device)
    K, N = w.shape[1], w.shape[2]
    packed = torch.empty((N_EXPERTS, N, K // 2), dtype=torch.uint8, device=device)
    scales = torch.empty((N_EXPERTS, N, K // FP4_BLOCK), dtype=torch.uint8, device=device)
    gs = torch.empty(N_EXPERTS, dtype=torch.float32, device=device)
    for e0 in range(0, N_EXPERTS, 16):  # bounded float32 temporaries
        q, s, g = _quantize_nvfp4(_linear_form(w[e0:e0 + 16].to(torch.float32)), mode)
        packed[e0:e0 + 16].copy_(q)
        scales[e0:e0 + 16].copy_(s)
        gs[e0:e0 + 16].copy_(g)
    return packed, scales, gs


# ----------------------------------------------------------------------------
# token-side inputs
# ----------------------------------------------------------------------------

@dataclass
class TokenInputs:
    x_bits: np.ndarray        # [T, 1536] uint16 (bf16 bits)
    logits: np.ndarray        # [T, 128] float32
    bias: np.ndarray          # [128] float32
    hot_experts: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int64))


def make_tokens(T: int, seed: int, hot: int = 0, hot_boost: float = 2.0,
                layer: int = 0) -> TokenInputs:
    """x, router logits and bias for ``T`` tokens from PCG64(seed, layer)."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, layer])))
    x = rng.standard_normal((T, HIDDEN), dtype=np.float32)
    logits = rng.standard_normal((T, N_EXPERTS), dtype=np.float32)
    bias = (rng.standard_normal(N_EXPERTS, dtype=np.float32) * np.float32(0.1)).astype(np.float32)
    hot_ids = np.zeros(0, np.int64)
    if hot:
        hot_ids = np.sort(rng.choice(N_EXPERTS, size=hot, replace=False)).astype(np.int64)
        logits[:, hot_ids] += np.float32(hot_boost)
    return TokenInputs(f32_to_bf16_bits(x), logits, bias, hot_ids)


def layer_logits(T: int, seed: int, layer: int):
    """Router logits [T,128] and bias [128] of one layer of the stack."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 1000 + layer])))
    logits = rng.standard_normal((T, N_EXPERTS), dtype=np.float32)
    bias = (rng.standard_normal(N_EXPERTS, dtype=np.float32) * np.float32(0.1)).astype(np.float32)
    return logits, bias


# ----------------------------------------------------------------------------
# second MoE shape: 256 experts
# ----------------------------------------------------------------------------

E256_SEED_OFFSET = (2000, 3000)  # generator seeds of experts 0..127 and 128..255


def e256_weight_bits_np(seed: int, layer: int, which: int, experts) -> np.ndarray:
    """Expert matrix ``which`` of the 256-expert shape for the given expert ids
    (0..255): experts 0..127 are the generator's under seed + 2000, experts
    128..255 its experts 0..127 under seed + 3000.  [len(experts), rows, cols]."""
    experts = np.asarray(experts)
    rows, cols = _W_SHAPES[which]
    out = np.zeros((len(experts), rows, cols), np.uint16)
    for half in (0, 1):
        sel = np.nonzero((experts >= 128 * half) & (experts < 128 * (half + 1)))[0]
        if len(sel):
            out[sel] = weight_bits_np(seed + E256_SEED_OFFSET[half], layer, which,
                                      experts[sel] - 128 * half)
    return out


def e256_weight_bits_torch(seed: int, layer: int, which: int, half: int, device):
    """The 128 experts of one half (0: experts 0..127, 1: 128..255) on ``device``."""
    return weight_bits_torch(seed + E256_SEED_OFFSET[half], layer, which, device)


def make_tokens_e256(T: int, seed: int) -> TokenInputs:
    """x [T, 1536] bf16 bits, router logits [T, 256] ~ N(0, 1) and bias [256]
    ~ N(0, 0.1), from PCG64(seed, 256)."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 256])))
    x = rng.standard_normal((T, HIDDEN), dtype=np.float32)
    logits = rng.standard_normal((T, 256), dtype=np.float32)
    bias = (rng.standard_normal(256, dtype=np.float32) * np.float32(0.1)).astype(np.float32)
    return TokenInputs(f32_to_bf16_bits(x), logits, bias)


# ----------------------------------------------------------------------------
# named workloads
# ----------------------------------------------------------------------------

@dataclass(frozen=True)
class Workload:
    name: str
    T: int                 # tokens actually processed
    T_buf: int             # rows allocated (>= T)
    seed: int
    hot: int = 0
    layers: int = 1
    weight_seed: int = 0


WORKLOADS = {
    "decode_T16": Workload("decode_T16", 16, 16, 0),
    **{f"decode_T4_seed{s}": Workload(f"decode_T4_seed{s}", 4, 4, s) for s in range(1, 9)},
    "prefill_T2048_skewed": Workload("prefill_T2048_skewed", 2048, 2048, 2, hot=16),
    "prefill_T8189": Workload("prefill_T8189", 8189, 8192, 3),
    "stack23_T1": Workload("stack23_T1", 1, 1, 4, layers=23, weight_seed=4),
    "stack23_T8189": Workload("stack23_T8189", 8189, 8192, 4, layers=23, weight_seed=4),
}
