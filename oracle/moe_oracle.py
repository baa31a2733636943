"""Float64 CPU oracle for the group-limited routed MoE layer of Ling-3.0-tiny.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
link this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA library (no kernels, headers, helpers or tables) and
imports nothing from the ``group_limited_routed_moe_b200`` package.

What it computes is the plain definition of the layer, evaluated in float64
from the exact bf16 / fp32 input values, with no blocking, fusion or
reordering beyond what the definition states:

* Grid.  128 routed experts per layer in 8 groups of 16; each token keeps 4
  groups and then uses 8 experts; hidden size 1536.  Sources: "Ling-3.0-tiny
  on a Qualcomm board" (TensorFold issue #1247), first comment, opening
  paragraph (tiny's config: "128 experts in 8 groups of 16 keeping 4",
  hidden 1536); "HelloSun/ling30tiny", table "模型與路由" (model and
  routing): 128 experts per layer, 8 experts active per token.
* Routing is group-limited (issue #1247, "What it does not cover", the bullet
  that lists the CUDA C kernels).  The pages name the rule but not its
  arithmetic; the reading used here (and in the CUDA path) is:
  score s_e = sigmoid(logit_e + bias_e); group score = sum of the group's two
  largest s; keep the 4 groups with the largest score (ties: lower group
  index); pick the 8 largest s among the 64 experts of the kept groups (ties:
  lower expert index), in that order; combine weight
  w_i = sigmoid(logit_{e_i}) / sum_j sigmoid(logit_{e_j}) (bias excluded).
* Expert FFN: each expert has gate, up and down matrices ("HelloSun/
  ling30tiny", table "模型與路由", row "expert 權重": gate/up and down), i.e.
  a SwiGLU FFN  y = (silu(x W_gate) * (x W_up)) W_down  with silu(a) =
  a * sigmoid(a) and no clamp (issue #1247, opening paragraph: "null SwiGLU
  limit lists").  Intermediate size 512.
* Layer output: out_t = sum_i w_i * FFN_{e_i}(x_t) -- the "real MoE routing
  + weighted layer" of "HelloSun/ling30tiny", section "數值檢查摘要"
  (numeric check summary).
* Expert row sets: each expert runs on exactly the rows that picked it
  (issue #1247, "What it does not cover", bullet on bf16 experts).  The
  permutation below is the stable (token-ascending) counting sort of those
  rows, which the CUDA path must reproduce bit for bit.
* Stack: 23 MoE layers (24 layers with dense layer 0 -- issue #1247, opening
  paragraph), residual stream kept in bf16: h <- bf16(h + moe(h)).
* A second shape, 256 experts top-6 with 2 shared experts ("Add TML Inkling
  architecture", model description), with tiny's group rule scaled to 8
  groups of 32 keeping 4 (``route_e256``).
* Shared experts ("khronnuz/Ling-3.0-flash-exl3", table of quants; "Add TML
  Inkling architecture", model description): SwiGLU FFNs of the routed
  shape applied to every token with weight 1 (``moe_layer_shared``).
* Block-FP8 experts (issue #1247, "What it does not cover", third bullet: the
  CUDA path reads bf16, block FP8 and NVFP4 experts): E4M3 codes with one fp32
  scale per 128 x 128 block, weight = value(code) * scale; the layer is the
  definition above with those weights (``moe_layer_fp8``).
* NVFP4 experts (same bullet): E2M1 codes, one E4M3 scale per 16 weights
  along the input dimension and one fp32 scale per matrix, weight =
  value(code) * value(block scale) * tensor scale (``moe_layer_nvfp4``).

Every function is pinned by tests in ``tests/test_oracle_*.py`` against
brute force, closed forms and invariants (see each test's docstring).
"""

from __future__ import annotations

import itertools
from dataclasses import dataclass

import numpy as np

HIDDEN = 1536
INTER = 512
N_EXPERTS = 128
N_GROUPS = 8
KEEP_GROUPS = 4
TOPK = 8
N_MOE_LAYERS = 23


# ----------------------------------------------------------------------------
# bf16 <-> float64 (the oracle's own conversions; exact / round-to-nearest-even)
# ----------------------------------------------------------------------------

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of raw bfloat16 bits (uint16) as float64."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round float64 values to bfloat16 (round to nearest, ties to even).

    Rounds directly from float64 to 8 significant bits (no intermediate
    float32 rounding, which could round twice).  Finite normal-range values
    only; zero is kept.
    """
    v = np.asarray(v, dtype=np.float64)
    mant, expo = np.frexp(v)                  # v = mant * 2**expo, 0.5 <= |mant| < 1
    q = np.rint(mant * 256.0)                 # 8 significant bits, half to even
    r = np.ldexp(q, expo - 8)                 # exactly representable in bf16
    return (r.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# ----------------------------------------------------------------------------
# Routing
# ----------------------------------------------------------------------------

def router_logits(x_bits: np.ndarray, w_router_bits: np.ndarray) -> np.ndarray:
    """Router projection: logits[t, e] = sum_k x[t, k] * W_router[k, e], float64.

    x_bits [T, 1536] and w_router_bits [1536, 128] are bf16 bits; the result is
    the exact product of their values up to float64 rounding.  The pages name
    the routing kernel this feeds ("Ling-3.0-tiny on a Qualcomm board", issue
    #1247, "What it does not cover", first bullet) but not the projection
    itself; the reading here is the usual bias-free linear gate of the hidden
    state onto the 128 experts (the bias of the routing rule is added after it).
    """
    return bf16_bits_to_f64(x_bits) @ bf16_bits_to_f64(w_router_bits)


def sigmoid(z: np.ndarray) -> np.ndarray:
    """Logistic function in float64."""
    return 1.0 / (1.0 + np.exp(-z))


@dataclass
class RouteResult:
    topk_idx: np.ndarray      # [T, k] int64, slot order = descending score, ties -> lower index
    topk_w: np.ndarray        # [T, k] float64 combine weights
    kept_groups: np.ndarray   # [T, keep] int64, descending group score, ties -> lower index
    group_margin: np.ndarray  # [T] float64: (keep-th best group score) - (next one)
    expert_margin: np.ndarray  # [T] float64: (k-th best candidate score) - (next one)


def route(logits: np.ndarray, bias: np.ndarray | None,
          n_groups: int = N_GROUPS, keep: int = KEEP_GROUPS,
          topk: int = TOPK) -> RouteResult:
    """Group-limited top-k routing of every token (float64).

    Steps, per token (the reading stated in the module docstring):
      1. z_e = logit_e + bias_e and s_e = sigmoid(z_e);
      2. group score g_j = s_(1) + s_(2), the two largest s inside group j;
      3. kept groups = the ``keep`` largest g_j, ties to the lower group index;
      4. the ``topk`` largest s among the experts of the kept groups, ties to
         the lower expert index, in that order (the slot order);
      5. w_i = sigmoid(logit_{e_i}) / sum_i' sigmoid(logit_{e_i'}).
    The grid sizes are parameters so that tests can brute-force small grids.
    """
    lg = np.asarray(logits, dtype=np.float64)
    T, n_exp = lg.shape
    if n_exp % n_groups:
        raise ValueError("experts must split evenly into groups")
    gsize = n_exp // n_groups
    z = lg + (np.asarray(bias, dtype=np.float64)[None, :] if bias is not None else 0.0)
    s = sigmoid(z)

    two_best = np.sort(s.reshape(T, n_groups, gsize), axis=2)[:, :, -2:]
    gscore = two_best[:, :, 0] + two_best[:, :, 1]
    g_order = np.argsort(-gscore, axis=1, kind="stable")      # ties keep lower index first
    kept = g_order[:, :keep]
    rows = np.arange(T)[:, None]
    g_sorted = gscore[rows, g_order]
    group_margin = (g_sorted[:, keep - 1] - g_sorted[:, keep]) if keep < n_groups \
        else np.full(T, np.inf)

    in_kept = np.zeros((T, n_groups), dtype=bool)
    in_kept[rows, kept] = True
    cand = np.where(np.repeat(in_kept, gsize, axis=1), s, -np.inf)
    e_order = np.argsort(-cand, axis=1, kind="stable")
    idx = e_order[:, :topk]
    c_sorted = cand[rows, e_order]
    n_cand = keep * gsize
    expert_margin = (c_sorted[:, topk - 1] - c_sorted[:, topk]) if topk < n_cand \
        else np.full(T, np.inf)

    w = combine_weights(lg[rows, idx])
    return RouteResult(idx.astype(np.int64), w, kept.astype(np.int64),
                       group_margin, expert_margin)


def combine_weights(l: np.ndarray) -> np.ndarray:
    """w_i = sigmoid(l_i) / sum_j sigmoid(l_j) over each row of chosen raw logits.

    Evaluated as r_i / sum_j r_j with r_i = sigmoid(l_i) / sigmoid(m), m the
    row's largest logit -- the same quantity, but for m < 0 written as
    exp(l_i - m) (1 + exp(m)) / (1 + exp(l_i)), whose terms stay finite and
    non-zero when every sigmoid(l_i) underflows (logits below about -745).
    """
    l = np.asarray(l, dtype=np.float64)
    m = l.max(axis=1, keepdims=True)
    with np.errstate(over="ignore"):
        direct = sigmoid(l) / sigmoid(m)
        shifted = np.exp(l - m) * (1.0 + np.exp(m)) / (1.0 + np.exp(l))
    r = np.where(m >= 0.0, direct, shifted)
    return r / r.sum(axis=1, keepdims=True)


def route_bruteforce(logits_row: np.ndarray, bias_row: np.ndarray | None,
                     n_groups: int, keep: int, topk: int):
    """Routing of ONE token by exhaustive enumeration (pure Python, tiny grids).

    Enumerates every subset of ``keep`` groups and keeps the one with the
    largest total group score (a group's score being the sum of its two
    largest member scores, found here by scanning all member pairs); then
    enumerates every ``topk``-subset of the kept groups' experts and keeps the
    one with the largest total score.  Exact ties are broken by preferring the
    lexicographically smaller index tuple.  Returns (kept groups sorted,
    chosen experts sorted by descending score then index, weights).
    """
    n_exp = len(logits_row)
    gsize = n_exp // n_groups
    b = [0.0] * n_exp if bias_row is None else [float(v) for v in bias_row]
    s = [1.0 / (1.0 + np.exp(-(float(logits_row[e]) + b[e]))) for e in range(n_exp)]

    def gscore(j):
        mem = range(j * gsize, (j + 1) * gsize)
        return max(s[a] + s[c] for a in mem for c in mem if a < c)

    gs = [gscore(j) for j in range(n_groups)]
    best_g, best_val = None, None
    for sub in itertools.combinations(range(n_groups), keep):
        val = sum(sorted((gs[j] for j in sub), reverse=True))
        if best_val is None or val > best_val:
            best_g, best_val = sub, val
    cands = [e for j in best_g for e in range(j * gsize, (j + 1) * gsize)]
    best_e, best_v = None, None
    for sub in itertools.combinations(sorted(cands), topk):
        val = sum(sorted((s[e] for e in sub), reverse=True))
        if best_v is None or val > best_v:
            best_e, best_v = sub, val
    chosen = sorted(best_e, key=lambda e: (-s[e], e))
    sig = [1.0 / (1.0 + np.exp(-float(logits_row[e]))) for e in chosen]
    tot = sum(sig)
    return sorted(best_g), chosen, [v / tot for v in sig]


# ----------------------------------------------------------------------------
# Permutation (rows that picked each expert)
# ----------------------------------------------------------------------------

@dataclass
class PermuteResult:
    counts: np.ndarray    # [E] int64
    offsets: np.ndarray   # [E+1] int64, exclusive prefix of counts
    perm_src: np.ndarray  # [T*k] int64: permuted row r holds item t*k + slot
    inv_perm: np.ndarray  # [T*k] int64: item t*k + slot sits at permuted row inv_perm[...]


def permute(topk_idx: np.ndarray, n_experts: int = N_EXPERTS) -> PermuteResult:
    """Stable counting sort of the (token, slot) items by expert id.

    Items are numbered t*k + slot; rows are grouped expert-major and, inside
    an expert, kept in item order (token ascending, since a token picks an
    expert at most once).
    """
    flat = np.asarray(topk_idx, dtype=np.int64).reshape(-1)
    counts = np.bincount(flat, minlength=n_experts).astype(np.int64)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    perm_src = np.argsort(flat, kind="stable").astype(np.int64)
    inv_perm = np.empty_like(perm_src)
    inv_perm[perm_src] = np.arange(flat.size, dtype=np.int64)
    return PermuteResult(counts, offsets, perm_src, inv_perm)


# ----------------------------------------------------------------------------
# Expert FFN, layer, stack
# ----------------------------------------------------------------------------

def silu(a: np.ndarray) -> np.ndarray:
    """silu(a) = a * sigmoid(a), float64, no clamp."""
    return a * sigmoid(a)


def expert_ffn(x: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray,
               w_down: np.ndarray) -> np.ndarray:
    """SwiGLU expert on rows x [M, H] (float64): (silu(x Wg) * (x Wu)) Wd."""
    return (silu(x @ w_gate) * (x @ w_up)) @ w_down


def moe_layer(x_bits: np.ndarray, logits: np.ndarray, bias: np.ndarray | None,
              w_gate_bits: np.ndarray, w_up_bits: np.ndarray,
              w_down_bits: np.ndarray, route_result: RouteResult | None = None
              ) -> np.ndarray:
    """Routed MoE layer output [T, H] in float64 (no intermediate rounding).

    x_bits: [T, H] bf16 bits; logits [T, E] fp32; bias [E] fp32 or None;
    w_gate_bits, w_up_bits: [E, H, I] bf16 bits; w_down_bits: [E, I, H].
    Each token only depends on its own row, so calling this on a subset of
    rows gives those rows of the full result.
    """
    rr = route_result if route_result is not None else route(logits, bias)
    x = bf16_bits_to_f64(x_bits)
    T = x.shape[0]
    out = np.zeros((T, w_down_bits.shape[2]), dtype=np.float64)
    for e in np.unique(rr.topk_idx):
        tok, slot = np.nonzero(rr.topk_idx == e)
        y = expert_ffn(x[tok], bf16_bits_to_f64(w_gate_bits[e]),
                       bf16_bits_to_f64(w_up_bits[e]), bf16_bits_to_f64(w_down_bits[e]))
        out[tok] += rr.topk_w[tok, slot][:, None] * y
    return out


def moe_stack(x_bits: np.ndarray, layers) -> np.ndarray:
    """Stack of MoE layers with a bf16 residual stream.

    ``layers`` yields (logits, bias, w_gate_bits, w_up_bits, w_down_bits) per
    layer; the router logits of every layer are given (they do not depend on
    the activations in this reading).  After each layer the residual stream is
    rounded to bf16: h <- bf16(h + moe(h)).  Returns the final bf16 bits.
    """
    h = np.asarray(x_bits, dtype=np.uint16)
    for (lg, b, wg, wu, wd) in layers:
        upd = moe_layer(h, lg, b, wg, wu, wd)
        h = f64_to_bf16_bits(bf16_bits_to_f64(h) + upd)
    return h


# ----------------------------------------------------------------------------
# Block-FP8 expert weights
# ----------------------------------------------------------------------------
# The CUDA path of "Ling-3.0-tiny on a Qualcomm board" (TensorFold issue
# #1247, first comment, "What it does not cover", third bullet) reads expert
# weights in bf16, in block FP8 and in NVFP4, and the issue mentions an
# official FP8 release of tiny.  The pages do not spell the block-FP8 format
# out; the reading here is the usual one for block-FP8 checkpoints: every
# weight is an FP8 E4M3 code (OCP 8-bit floating point, the "FN" variant
# without infinities), and every 128 x 128 block of a matrix carries one fp32
# scale, the weight being  value(code) * scale  exactly.  The layer is then the
# bf16 layer's definition with those weights.

FP8_BLOCK = 128


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    """Exact value of FP8 E4M3 codes (uint8) as float64.

    Bit 7 is the sign, bits 6..3 the exponent field E (bias 7), bits 2..0 the
    mantissa m.  E = 0 encodes the subnormals m/8 * 2**-6; otherwise the value
    is (1 + m/8) * 2**(E - 7).  The two codes with every exponent and mantissa
    bit set (0x7F, 0xFF) are NaN; there are no infinities, so the largest
    finite magnitude is 1.75 * 2**8 = 448.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c & 0x80) != 0, -1.0, 1.0)
    E = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(E == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(E - 7.0))
    v = sign * mag
    return np.where((c & 0x7F) == 0x7F, np.nan, v)


def dequant_block_fp8(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Weights of a block-FP8 matrix (or stack of matrices) in float64.

    codes [..., R, C] uint8 E4M3 codes; scales [..., R/128, C/128] fp32, one per
    128 x 128 block.  W[..., r, c] = value(codes[..., r, c]) * scales[..., r // 128,
    c // 128], exact in float64 (a 4-bit significand times a 24-bit one).
    """
    v = e4m3_to_f64(codes)
    s = np.asarray(scales, dtype=np.float64)
    R, C = v.shape[-2:]
    if s.shape[-2:] != (R // FP8_BLOCK, C // FP8_BLOCK) or R % FP8_BLOCK or C % FP8_BLOCK:
        raise ValueError(f"scales {s.shape} do not tile codes {v.shape} in {FP8_BLOCK}-blocks")
    full = np.repeat(np.repeat(s, FP8_BLOCK, axis=-2), FP8_BLOCK, axis=-1)
    return v * full


def moe_layer_f64(x_bits: np.ndarray, logits: np.ndarray, bias: np.ndarray | None,
                  expert_weights, route_result: RouteResult | None = None) -> np.ndarray:
    """The routed layer of ``moe_layer`` with float64 expert weights.

    ``expert_weights(e)`` returns (W_gate [H, I], W_up [H, I], W_down [I, H]) of
    expert e in float64; it is called once for every expert some token uses.
    """
    rr = route_result if route_result is not None else route(logits, bias)
    x = bf16_bits_to_f64(x_bits)
    out = np.zeros((x.shape[0], HIDDEN), dtype=np.float64)
    for e in np.unique(rr.topk_idx):
        tok, slot = np.nonzero(rr.topk_idx == e)
        wg, wu, wd = expert_weights(int(e))
        out[tok] += rr.topk_w[tok, slot][:, None] * expert_ffn(x[tok], wg, wu, wd)
    return out


def moe_layer_fp8(x_bits: np.ndarray, logits: np.ndarray, bias: np.ndarray | None,
                  q_gate: np.ndarray, s_gate: np.ndarray, q_up: np.ndarray, s_up: np.ndarray,
                  q_down: np.ndarray, s_down: np.ndarray,
                  route_result: RouteResult | None = None) -> np.ndarray:
    """Routed layer with block-FP8 experts, float64, no intermediate rounding.

    q_gate, q_up: [E, 1536, 512] uint8 codes, s_gate, s_up: [E, 12, 4] fp32;
    q_down: [E, 512, 1536] codes, s_down: [E, 4, 12].  Only the experts that
    some token uses are read.
    """
    def weights(e):
        return (dequant_block_fp8(q_gate[e], s_gate[e]), dequant_block_fp8(q_up[e], s_up[e]),
                dequant_block_fp8(q_down[e], s_down[e]))
    return moe_layer_f64(x_bits, logits, bias, weights, route_result)


# ----------------------------------------------------------------------------
# NVFP4 expert weights
# ----------------------------------------------------------------------------
# The same bullet of issue #1247 names ModelOpt NVFP4 as the third expert
# format the CUDA path reads.  The format, as ModelOpt writes it for a linear
# layer's weight [out, in]: every weight is a 4-bit E2M1 code (OCP
# microscaling FP4: sign, 2-bit exponent with bias 1, 1-bit mantissa; no
# infinities or NaN), two codes per byte along the input dimension with the
# even element in the low nibble; every 16 consecutive weights along the input
# dimension share one FP8 E4M3 block scale; the whole matrix shares one fp32
# tensor scale.  weight = value(code) * value(block scale) * tensor scale,
# exactly.  The matrices are held here in that [out, in] orientation (W_gate
# and W_up of an expert as [512, 1536], W_down as [1536, 512]); the layer uses
# their transposes in the x W form above.

NVFP4_BLOCK = 16


def e2m1_to_f64(codes: np.ndarray) -> np.ndarray:
    """Exact value of FP4 E2M1 codes (uint8 holding 0..15) as float64.

    Bit 3 is the sign, bits 2..1 the exponent field E (bias 1), bit 0 the
    mantissa m.  E = 0 encodes the subnormals 0 and 0.5 (m/2); otherwise the
    value is (1 + m/2) * 2**(E - 1).  Magnitudes: 0, 0.5, 1, 1.5, 2, 3, 4, 6.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    if np.any(c > 15):
        raise ValueError("E2M1 codes are 4-bit values")
    sign = np.where((c & 0x8) != 0, -1.0, 1.0)
    E = (c >> 1) & 0x3
    m = (c & 0x1).astype(np.float64)
    mag = np.where(E == 0, m / 2.0, (1.0 + m / 2.0) * np.exp2(E - 1.0))
    return sign * mag


def unpack_fp4(packed: np.ndarray) -> np.ndarray:
    """[..., C/2] bytes -> [..., C] codes: element 2i is the low nibble of byte i,
    element 2i + 1 the high nibble."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def dequant_nvfp4(packed: np.ndarray, scales: np.ndarray, tensor_scale) -> np.ndarray:
    """Weights of an NVFP4 matrix (or stack of matrices) in float64, [out, in] form.

    packed [..., R, C/2] uint8 (two E2M1 codes per byte, see unpack_fp4);
    scales [..., R, C/16] uint8 E4M3 codes, one per 16 consecutive weights of a
    row; tensor_scale: fp32, one per matrix (shape [...]).
    W[..., r, c] = value(code[..., r, c]) * value(scales[..., r, c // 16]) * tensor_scale[...],
    exact in float64 (2 + 4 + 24 significant bits).
    """
    v = e2m1_to_f64(unpack_fp4(packed))
    s = e4m3_to_f64(scales)
    R, C = v.shape[-2:]
    if s.shape[-2:] != (R, C // NVFP4_BLOCK) or C % NVFP4_BLOCK:
        raise ValueError(f"scales {s.shape} do not tile codes {v.shape} in 1 x {NVFP4_BLOCK} blocks")
    g = np.asarray(tensor_scale, dtype=np.float64)
    if g.shape != v.shape[:-2]:
        raise ValueError(f"tensor scales {g.shape} do not match the matrices {v.shape[:-2]}")
    return v * np.repeat(s, NVFP4_BLOCK, axis=-1) * g[..., None, None]


def moe_layer_nvfp4(x_bits: np.ndarray, logits: np.ndarray, bias: np.ndarray | None,
                    q_gate: np.ndarray, s_gate: np.ndarray, g_gate: np.ndarray,
                    q_up: np.ndarray, s_up: np.ndarray, g_up: np.ndarray,
                    q_down: np.ndarray, s_down: np.ndarray, g_down: np.ndarray,
                    route_result: RouteResult | None = None) -> np.ndarray:
    """Routed layer with NVFP4 experts, float64, no intermediate rounding.

    q_gate, q_up: [E, 512, 768] packed codes ([out, in] form), s_gate, s_up:
    [E, 512, 96] E4M3 codes, g_gate, g_up: [E] fp32; q_down: [E, 1536, 256],
    s_down: [E, 1536, 32], g_down: [E].  Only the experts some token uses are read.
    """
    def weights(e):
        return (dequant_nvfp4(q_gate[e], s_gate[e], g_gate[e]).T,
                dequant_nvfp4(q_up[e], s_up[e], g_up[e]).T,
                dequant_nvfp4(q_down[e], s_down[e], g_down[e]).T)
    return moe_layer_f64(x_bits, logits, bias, weights, route_result)


# ----------------------------------------------------------------------------
# Second MoE shape: 256 experts, top-6
# ----------------------------------------------------------------------------
# The Inkling model has "256 experts top-6 plus 2 shared" ("Add TML Inkling
# architecture", llama.cpp PR #25731, model description); the pages give no
# group structure, hidden or intermediate size for it.  Read with tiny's group
# rule scaled to 256 experts (8 groups of 32, 4 kept) and tiny's expert shape
# (1536 -> 512 -> 1536), so that the same layer definition applies with 256
# experts and 6 slots; the two shared experts are those of moe_layer_shared.

E256_EXPERTS, E256_GROUPS, E256_KEEP, E256_TOPK = 256, 8, 4, 6


def route_e256(logits: np.ndarray, bias: np.ndarray | None) -> RouteResult:
    """route() on the second shape: logits [T, 256], 8 groups of 32, keep 4, top-6."""
    return route(logits, bias, n_groups=E256_GROUPS, keep=E256_KEEP, topk=E256_TOPK)


# ----------------------------------------------------------------------------
# Shared experts
# ----------------------------------------------------------------------------
# The Ling family's flash model has shared experts (its EXL3 card lists them
# beside attention among the parts kept at higher precision: "khronnuz/
# Ling-3.0-flash-exl3", table of quants), and the Inkling model has "256
# experts top-6 plus 2 shared" ("Add TML Inkling architecture", llama.cpp PR
# #25731, model description).  The pages give neither their size nor how they
# enter the sum; the reading here is the usual one: each shared expert is a
# SwiGLU FFN of the routed experts' shape that every token passes through
# with weight 1, added to the routed sum.

def moe_layer_shared(x_bits: np.ndarray, logits: np.ndarray, bias: np.ndarray | None,
                     w_gate_bits: np.ndarray, w_up_bits: np.ndarray, w_down_bits: np.ndarray,
                     s_gate_bits: np.ndarray, s_up_bits: np.ndarray, s_down_bits: np.ndarray,
                     route_result: RouteResult | None = None) -> np.ndarray:
    """Routed layer plus shared experts, float64, no intermediate rounding:
    out_t = sum_i w_i FFN_{e_i}(x_t) + sum_s FFN_s(x_t).

    s_gate_bits, s_up_bits: [S, 1536, 512] bf16 bits; s_down_bits: [S, 512, 1536]
    (S shared experts, S = 0 allowed); the routed arguments as in moe_layer.
    """
    out = moe_layer(x_bits, logits, bias, w_gate_bits, w_up_bits, w_down_bits,
                    route_result=route_result)
    x = bf16_bits_to_f64(x_bits)
    for s in range(np.asarray(s_gate_bits).shape[0]):
        out += expert_ffn(x, bf16_bits_to_f64(s_gate_bits[s]), bf16_bits_to_f64(s_up_bits[s]),
                          bf16_bits_to_f64(s_down_bits[s]))
    return out


def rel_l2(a: np.ndarray, ref: np.ndarray) -> float:
    """||a - ref||_2 / ||ref||_2 in float64."""
    a = np.asarray(a, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(a - ref) / den) if den > 0 else float(np.linalg.norm(a))
