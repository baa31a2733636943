"""Thin ctypes binding of libmoe (the C ABI in include/moe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch supplies device memory (tensors) and the current CUDA
stream.  Loading fails loudly when ``libmoe.so`` has not been built -- there is
no fallback path.
"""

from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "moe.h")

HIDDEN, INTER, N_EXPERTS, N_GROUPS, KEEP_GROUPS, TOPK = 1536, 512, 128, 8, 4, 8
OFFSETS_LEN = 264  # 129 expert offsets + scratch words used by the expert-FFN kernels
MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_TIMEOUT, \
    MOE_ERR_UNSUPPORTED, MOE_ERR_RANGE = range(7)


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed with status {code}: {msg}")
        self.code = code


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -c 'import __graft_entry__ as g; g.build()'`"
            " (there is no CPU or Python fallback for the MoE layer)")
    return ctypes.CDLL(LIB_PATH)


lib = _load()

_p, _i64, _sz, _i32, _u64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int, ctypes.c_uint64
_SIGS = {
    "moe_abi_version": ([], _i32),
    "moe_max_tokens": ([], _i64),
    "moe_last_error_string": ([], ctypes.c_char_p),
    "moe_get_device_status": ([_i32], _i32),
    "moe_init_device": ([], _i32),
    "moe_set_ffn_trace": ([_p, _i64], _i32),
    "moe_set_wait_timeout_ns": ([_u64], _i32),
    "moe_selftest_wait_timeout": ([_p], _i32),
    "moe_packed_weight_bytes": ([], _sz),
    "moe_pack_weights": ([_p, _p, _p, _p, _p], _i32),
    "moe_route": ([_p, _p, _i64, _p, _p, _p], _i32),
    "moe_permute_workspace_bytes": ([_i64], _sz),
    "moe_permute": ([_p, _i64, _p, _p, _p, _p, _p, _sz, _p], _i32),
    "moe_expert_ffn": ([_p, _p, _p, _p, _i64, _p, _p, _p], _i32),
    "moe_expert_gate_up": ([_p, _p, _p, _p, _i64, _p, _p], _i32),
    "moe_expert_down": ([_p, _p, _p, _i64, _p, _p], _i32),
    "moe_combine": ([_p, _p, _p, _i64, _p, _p, _p], _i32),
    "moe_layer_workspace_bytes": ([_i64], _sz),
    "moe_layer": ([_p, _p, _p, _p, _i64, _p, _p, _p, _p, _p, _sz, _p], _i32),
    "moe_router_packed_bytes": ([], _sz),
    "moe_layer_host_workspace_bytes": ([_i64, _i32], _sz),
    "moe_layer_host": ([_p, _p, _p, _p, _i32, _i64, _p, _p, _sz, _p, _p, _p], _i32),
    "moe_pack_router": ([_p, _p, _p], _i32),
    "moe_router": ([_p, _p, _i64, _p, _p], _i32),
    "moe_layer_routed": ([_p, _p, _p, _p, _i64, _p, _p, _p, _p, _p, _sz, _p], _i32),
    "moe_route_from_x": ([_p, _p, _p, _i64, _p, _p, _p, _p], _i32),
    "moe_permute_fixed_scratch_max_tokens": ([], _i64),
    "moe_permute_fixed_scratch": ([_p, _i64, _p, _p, _p, _p, _p], _i32),
    "moe_packed_fp8_bytes": ([], _sz),
    "moe_pack_weights_fp8": ([_p, _p, _p, _p, _p, _p, _p, _p], _i32),
    "moe_dequant_fp8": ([_p, _p, _p], _i32),
    "moe_layer_fp8_workspace_bytes": ([_i64], _sz),
    "moe_expert_ffn_fp8_workspace_bytes": ([_i64], _sz),
    "moe_expert_ffn_fp8": ([_p, _p, _p, _p, _i64, _p, _p, _p, _sz, _p], _i32),
    "moe_packed_shared_bytes": ([_i32], _sz),
    "moe_pack_shared": ([_p, _p, _p, _i32, _p, _p], _i32),
    "moe_layer_shared_workspace_bytes": ([_i64, _i32, _i32], _sz),
    "moe_layer_shared": ([_p, _p, _p, _p, _p, _p, _i32, _i64, _p, _p, _p, _p, _p, _sz, _p], _i32),
    "moe_layer_shared_nvfp4": ([_p, _p, _p, _p, _p, _i32, _i64, _p, _p, _p, _p, _p, _sz, _p], _i32),
    "moe_packed_experts_bytes": ([_i32], _sz),
    "moe_pack_experts": ([_p, _p, _p, _i32, _p, _p], _i32),
    "moe_expert_ffn_slice": ([_p, _p, _i32, _p, _p, _i64, _p, _p, _p], _i32),
    "moe_route_e256": ([_p, _p, _i64, _p, _p, _p], _i32),
    "moe_layer_e256_workspace_bytes": ([_i64, _i32], _sz),
    "moe_layer_e256": ([_p, _p, _p, _p, _p, _p, _i32, _i64, _p, _p, _p, _p, _p, _sz, _p], _i32),
    "moe_layer_fp8": ([_p, _p, _p, _p, _i64, _p, _p, _p, _p, _p, _sz, _p], _i32),
    "moe_packed_nvfp4_bytes": ([], _sz),
    "moe_pack_weights_nvfp4": ([_p] * 10 + [_p], _i32),
    "moe_dequant_nvfp4": ([_p, _p, _p], _i32),
    "moe_layer_nvfp4_workspace_bytes": ([_i64], _sz),
    "moe_expert_ffn_nvfp4_workspace_bytes": ([_i64], _sz),
    "moe_expert_ffn_nvfp4": ([_p, _p, _p, _p, _i64, _p, _p, _p, _sz, _p], _i32),
    "moe_layer_nvfp4": ([_p, _p, _p, _p, _i64, _p, _p, _p, _p, _p, _sz, _p], _i32),
}
for _name, (_args, _ret) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.argtypes = _args
    _f.restype = _ret


def header_functions() -> list[str]:
    """Names of the functions include/moe.h declares."""
    src = open(HEADER_PATH).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def _check(fn: str, rc: int) -> None:
    if rc != MOE_OK:
        raise MoeError(fn, rc, lib.moe_last_error_string().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def last_error() -> str:
    return lib.moe_last_error_string().decode()


# ----------------------------------------------------------------- weights

def packed_weight_bytes() -> int:
    return int(lib.moe_packed_weight_bytes())


def moe_pack_weights(w_gate: torch.Tensor, w_up: torch.Tensor, w_down: torch.Tensor,
                     packed: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Re-layout one layer's bf16 expert weights (see include/moe.h)."""
    for t, shp in ((w_gate, (N_EXPERTS, HIDDEN, INTER)), (w_up, (N_EXPERTS, HIDDEN, INTER)),
                   (w_down, (N_EXPERTS, INTER, HIDDEN))):
        if t.dtype != torch.bfloat16 or tuple(t.shape) != shp or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"expected contiguous CUDA bf16 {shp}, got {t.dtype} {tuple(t.shape)}")
    if packed is None:
        packed = torch.empty(packed_weight_bytes() // 2, dtype=torch.bfloat16, device=w_gate.device)
    _check("moe_pack_weights", lib.moe_pack_weights(_ptr(w_gate), _ptr(w_up), _ptr(w_down),
                                                    _ptr(packed), _stream(stream)))
    return packed


# ----------------------------------------------------------------- steps

def moe_route(logits: torch.Tensor, bias: torch.Tensor | None, topk_idx=None, topk_w=None,
              stream=None):
    T = logits.shape[0]
    dev = logits.device
    if topk_idx is None:
        topk_idx = torch.empty((T, TOPK), dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty((T, TOPK), dtype=torch.float32, device=dev)
    _check("moe_route", lib.moe_route(_ptr(logits), _ptr(bias), T, _ptr(topk_idx), _ptr(topk_w),
                                      _stream(stream)))
    return topk_idx, topk_w


def permute_workspace_bytes(T: int) -> int:
    return int(lib.moe_permute_workspace_bytes(T))


def moe_permute(topk_idx: torch.Tensor, counts=None, offsets=None, perm_src=None, inv_perm=None,
                workspace=None, stream=None):
    """Returns (counts[128], offsets[129], perm_src[8T], inv_perm[8T]) int32.

    ``offsets`` is a view of the first 129 words of an OFFSETS_LEN-word buffer;
    pass it on unchanged to the expert-FFN calls (they use the trailing words)."""
    T = topk_idx.shape[0]
    dev = topk_idx.device
    if counts is None:
        counts = torch.empty(N_EXPERTS, dtype=torch.int32, device=dev)
    if offsets is None:
        offsets = torch.empty(OFFSETS_LEN, dtype=torch.int32, device=dev)
    if offsets.numel() < OFFSETS_LEN:
        raise ValueError(f"offsets needs {OFFSETS_LEN} int32 words")
    if perm_src is None:
        perm_src = torch.empty(max(T * TOPK, 1), dtype=torch.int32, device=dev)
    if inv_perm is None:
        inv_perm = torch.empty(max(T * TOPK, 1), dtype=torch.int32, device=dev)
    wsb = permute_workspace_bytes(T)
    if workspace is None and wsb:
        workspace = torch.empty(wsb, dtype=torch.uint8, device=dev)
    _check("moe_permute", lib.moe_permute(_ptr(topk_idx), T, _ptr(counts), _ptr(offsets),
                                          _ptr(perm_src), _ptr(inv_perm),
                                          _ptr(workspace) if wsb else None,
                                          workspace.numel() if wsb else 0, _stream(stream)))
    return counts, offsets[:N_EXPERTS + 1], perm_src[:T * TOPK], inv_perm[:T * TOPK]


def moe_permute_fixed_scratch(topk_idx: torch.Tensor, counts: torch.Tensor, offsets: torch.Tensor,
                              perm_src: torch.Tensor, inv_perm: torch.Tensor, stream=None):
    """moe_permute with the library's fixed scratch (T <= 65536): every output is
    caller-provided, and the call allocates no device memory."""
    T = topk_idx.shape[0]
    if offsets.numel() < OFFSETS_LEN or counts.numel() < N_EXPERTS:
        raise ValueError(f"counts needs {N_EXPERTS} and offsets {OFFSETS_LEN} int32 words")
    if perm_src.numel() < T * TOPK or inv_perm.numel() < T * TOPK:
        raise ValueError(f"perm_src and inv_perm need {T * TOPK} int32 words")
    _check("moe_permute_fixed_scratch",
           lib.moe_permute_fixed_scratch(_ptr(topk_idx), T, _ptr(counts), _ptr(offsets),
                                         _ptr(perm_src), _ptr(inv_perm), _stream(stream)))
    return counts, offsets[:N_EXPERTS + 1], perm_src[:T * TOPK], inv_perm[:T * TOPK]


def moe_expert_ffn(x: torch.Tensor, packed_w: torch.Tensor, offsets: torch.Tensor,
                   perm_src: torch.Tensor, h=None, y_perm=None, stream=None):
    """Returns (h [8T,512], y_perm [8T,1536]) fp16."""
    T = x.shape[0]
    dev = x.device
    if h is None:
        h = torch.empty((T * TOPK, INTER), dtype=torch.float16, device=dev)
    if y_perm is None:
        y_perm = torch.empty((T * TOPK, HIDDEN), dtype=torch.float16, device=dev)
    _check("moe_expert_ffn", lib.moe_expert_ffn(_ptr(x), _ptr(packed_w), _ptr(offsets),
                                                _ptr(perm_src), T, _ptr(h), _ptr(y_perm),
                                                _stream(stream)))
    return h, y_perm


def moe_expert_gate_up(x: torch.Tensor, packed_w: torch.Tensor, offsets: torch.Tensor,
                       perm_src: torch.Tensor, h=None, stream=None):
    T = x.shape[0]
    if h is None:
        h = torch.empty((T * TOPK, INTER), dtype=torch.float16, device=x.device)
    _check("moe_expert_gate_up", lib.moe_expert_gate_up(_ptr(x), _ptr(packed_w), _ptr(offsets),
                                                        _ptr(perm_src), T, _ptr(h),
                                                        _stream(stream)))
    return h


def moe_expert_down(h: torch.Tensor, packed_w: torch.Tensor, offsets: torch.Tensor,
                    y_perm=None, stream=None):
    T = h.shape[0] // TOPK
    if y_perm is None:
        y_perm = torch.empty((T * TOPK, HIDDEN), dtype=torch.float16, device=h.device)
    _check("moe_expert_down", lib.moe_expert_down(_ptr(h), _ptr(packed_w), _ptr(offsets), T,
                                                  _ptr(y_perm), _stream(stream)))
    return y_perm


def moe_combine(y_perm: torch.Tensor, topk_w: torch.Tensor, inv_perm: torch.Tensor,
                residual=None, out=None, stream=None):
    T = topk_w.shape[0]
    if out is None:
        out = torch.empty((T, HIDDEN), dtype=torch.bfloat16, device=topk_w.device)
    _check("moe_combine", lib.moe_combine(_ptr(y_perm), _ptr(topk_w), _ptr(inv_perm), T,
                                          _ptr(residual), _ptr(out), _stream(stream)))
    return out


# ----------------------------------------------------------------- fused layer

def layer_workspace_bytes(T: int) -> int:
    return int(lib.moe_layer_workspace_bytes(T))


def alloc_layer_workspace(T: int, device, fp8: bool = False) -> torch.Tensor:
    """A uint8 view of at least layer_workspace_bytes(T) bytes, 1024-byte
    aligned.  fp8=True sizes it for a quantised layer (moe_layer_fp8 or
    moe_layer_nvfp4: layer_fp8_workspace_bytes(T), which
    layer_nvfp4_workspace_bytes(T) equals)."""
    n = layer_fp8_workspace_bytes(T) if fp8 else layer_workspace_bytes(T)
    raw = torch.empty(n + 1024, dtype=torch.uint8, device=device)
    off = (-raw.data_ptr()) % 1024
    return raw[off:off + n]


def moe_layer(x: torch.Tensor, logits: torch.Tensor, bias: torch.Tensor | None,
              packed_w: torch.Tensor, residual=None, out=None, topk_idx_out=None,
              topk_w_out=None, workspace: torch.Tensor | None = None, stream=None):
    """out = bf16(residual + MoE(x)) for x [T,1536] bf16 (see include/moe.h)."""
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, HIDDEN), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = alloc_layer_workspace(T, x.device)
    _check("moe_layer", lib.moe_layer(_ptr(x), _ptr(logits), _ptr(bias), _ptr(packed_w), T,
                                      _ptr(residual), _ptr(out), _ptr(topk_idx_out),
                                      _ptr(topk_w_out), _ptr(workspace), workspace.numel(),
                                      _stream(stream)))
    return out


def moe_pack_router(w_router: torch.Tensor, packed=None, stream=None) -> torch.Tensor:
    """W_router [1536,128] bf16 -> packed K-major [128,1536] (see include/moe.h)."""
    if w_router.dtype != torch.bfloat16 or tuple(w_router.shape) != (HIDDEN, N_EXPERTS) \
            or not w_router.is_contiguous() or not w_router.is_cuda:
        raise ValueError(f"expected contiguous CUDA bf16 ({HIDDEN}, {N_EXPERTS})")
    if packed is None:
        packed = torch.empty((N_EXPERTS, HIDDEN), dtype=torch.bfloat16, device=w_router.device)
    _check("moe_pack_router", lib.moe_pack_router(_ptr(w_router), _ptr(packed), _stream(stream)))
    return packed


def moe_router(x: torch.Tensor, packed_router: torch.Tensor, logits=None, stream=None):
    """logits [T,128] fp32 = x [T,1536] bf16 @ W_router."""
    T = x.shape[0]
    if logits is None:
        logits = torch.empty((T, N_EXPERTS), dtype=torch.float32, device=x.device)
    _check("moe_router", lib.moe_router(_ptr(x), _ptr(packed_router), T, _ptr(logits),
                                        _stream(stream)))
    return logits


def moe_route_from_x(x: torch.Tensor, packed_router: torch.Tensor, bias: torch.Tensor | None,
                     logits=None, topk_idx=None, topk_w=None, stream=None):
    """Router projection and routing from x [T,1536] bf16: returns (logits [T,128]
    fp32, topk_idx [T,8] int32, topk_w [T,8] fp32)."""
    T = x.shape[0]
    dev = x.device
    if logits is None:
        logits = torch.empty((T, N_EXPERTS), dtype=torch.float32, device=dev)
    if topk_idx is None:
        topk_idx = torch.empty((T, TOPK), dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty((T, TOPK), dtype=torch.float32, device=dev)
    _check("moe_route_from_x", lib.moe_route_from_x(_ptr(x), _ptr(packed_router), _ptr(bias), T,
                                                    _ptr(logits), _ptr(topk_idx), _ptr(topk_w),
                                                    _stream(stream)))
    return logits, topk_idx, topk_w


def moe_layer_routed(x: torch.Tensor, packed_router: torch.Tensor, bias: torch.Tensor | None,
                     packed_w: torch.Tensor, residual=None, out=None, topk_idx_out=None,
                     topk_w_out=None, workspace: torch.Tensor | None = None, stream=None):
    """moe_layer with the router projection of x in front (see include/moe.h)."""
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, HIDDEN), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = alloc_layer_workspace(T, x.device)
    _check("moe_layer_routed", lib.moe_layer_routed(
        _ptr(x), _ptr(packed_router), _ptr(bias), _ptr(packed_w), T, _ptr(residual), _ptr(out),
        _ptr(topk_idx_out), _ptr(topk_w_out), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


# ----------------------------------------------------------------- block-FP8 experts

def packed_fp8_bytes() -> int:
    return int(lib.moe_packed_fp8_bytes())


def layer_fp8_workspace_bytes(T: int) -> int:
    return int(lib.moe_layer_fp8_workspace_bytes(T))


def moe_pack_weights_fp8(q_gate: torch.Tensor, s_gate: torch.Tensor, q_up: torch.Tensor,
                         s_up: torch.Tensor, q_down: torch.Tensor, s_down: torch.Tensor,
                         packed: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Re-layout one layer's block-FP8 experts: uint8 E4M3 codes and fp32
    128 x 128 block scales (see include/moe.h)."""
    nb_h, nb_i = HIDDEN // 128, INTER // 128
    for t, shp, dt in ((q_gate, (N_EXPERTS, HIDDEN, INTER), torch.uint8),
                       (q_up, (N_EXPERTS, HIDDEN, INTER), torch.uint8),
                       (q_down, (N_EXPERTS, INTER, HIDDEN), torch.uint8),
                       (s_gate, (N_EXPERTS, nb_h, nb_i), torch.float32),
                       (s_up, (N_EXPERTS, nb_h, nb_i), torch.float32),
                       (s_down, (N_EXPERTS, nb_i, nb_h), torch.float32)):
        if t.dtype != dt or tuple(t.shape) != shp or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"expected contiguous CUDA {dt} {shp}, got {t.dtype} {tuple(t.shape)}")
    if packed is None:
        packed = torch.empty(packed_fp8_bytes(), dtype=torch.uint8, device=q_gate.device)
    _check("moe_pack_weights_fp8",
           lib.moe_pack_weights_fp8(_ptr(q_gate), _ptr(s_gate), _ptr(q_up), _ptr(s_up),
                                    _ptr(q_down), _ptr(s_down), _ptr(packed), _stream(stream)))
    return packed


def moe_dequant_fp8(packed_fp8: torch.Tensor, packed: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
    """The packed bf16/fp16 layer (moe_pack_weights layout) of a packed FP8 layer."""
    if packed is None:
        packed = torch.empty(packed_weight_bytes() // 2, dtype=torch.bfloat16,
                             device=packed_fp8.device)
    _check("moe_dequant_fp8", lib.moe_dequant_fp8(_ptr(packed_fp8), _ptr(packed), _stream(stream)))
    return packed


def moe_expert_ffn_fp8(x: torch.Tensor, packed_fp8: torch.Tensor, offsets: torch.Tensor,
                       perm_src: torch.Tensor, h=None, y_perm=None, workspace=None, stream=None):
    """Step 3 with block-FP8 experts (see include/moe.h); returns (h, y_perm)."""
    T = x.shape[0]
    n = T * TOPK
    if h is None:
        h = torch.empty((n, INTER), dtype=torch.float16, device=x.device)
    if y_perm is None:
        y_perm = torch.empty((n, HIDDEN), dtype=torch.float16, device=x.device)
    need = int(lib.moe_expert_ffn_fp8_workspace_bytes(T))
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    _check("moe_expert_ffn_fp8",
           lib.moe_expert_ffn_fp8(_ptr(x), _ptr(packed_fp8), _ptr(offsets), _ptr(perm_src), T,
                                  _ptr(h), _ptr(y_perm), _ptr(workspace),
                                  workspace.numel() if workspace is not None else 0,
                                  _stream(stream)))
    return h, y_perm


def moe_layer_fp8(x: torch.Tensor, logits: torch.Tensor, bias: torch.Tensor | None,
                  packed_fp8: torch.Tensor, residual=None, out=None, topk_idx_out=None,
                  topk_w_out=None, workspace: torch.Tensor | None = None, stream=None):
    """moe_layer with block-FP8 experts (see include/moe.h)."""
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, HIDDEN), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = alloc_layer_workspace(T, x.device, fp8=True)
    _check("moe_layer_fp8", lib.moe_layer_fp8(_ptr(x), _ptr(logits), _ptr(bias), _ptr(packed_fp8),
                                              T, _ptr(residual), _ptr(out), _ptr(topk_idx_out),
                                              _ptr(topk_w_out), _ptr(workspace), workspace.numel(),
                                              _stream(stream)))
    return out


# ----------------------------------------------------------------- NVFP4 experts

def packed_nvfp4_bytes() -> int:
    return int(lib.moe_packed_nvfp4_bytes())


def layer_nvfp4_workspace_bytes(T: int) -> int:
    return int(lib.moe_layer_nvfp4_workspace_bytes(T))


def moe_pack_weights_nvfp4(q_gate, s_gate, g_gate, q_up, s_up, g_up, q_down, s_down, g_down,
                           packed: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Re-layout one layer's NVFP4 experts ([out, in] form: uint8 codes two per
    byte, uint8 E4M3 block scales per 16 inputs, fp32 tensor scales; see
    include/moe.h)."""
    for t, shp, dt in ((q_gate, (N_EXPERTS, INTER, HIDDEN // 2), torch.uint8),
                       (q_up, (N_EXPERTS, INTER, HIDDEN // 2), torch.uint8),
                       (q_down, (N_EXPERTS, HIDDEN, INTER // 2), torch.uint8),
                       (s_gate, (N_EXPERTS, INTER, HIDDEN // 16), torch.uint8),
                       (s_up, (N_EXPERTS, INTER, HIDDEN // 16), torch.uint8),
                       (s_down, (N_EXPERTS, HIDDEN, INTER // 16), torch.uint8),
                       (g_gate, (N_EXPERTS,), torch.float32), (g_up, (N_EXPERTS,), torch.float32),
                       (g_down, (N_EXPERTS,), torch.float32)):
        if t.dtype != dt or tuple(t.shape) != shp or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"expected contiguous CUDA {dt} {shp}, got {t.dtype} {tuple(t.shape)}")
    if packed is None:
        packed = torch.empty(packed_nvfp4_bytes(), dtype=torch.uint8, device=q_gate.device)
    _check("moe_pack_weights_nvfp4",
           lib.moe_pack_weights_nvfp4(_ptr(q_gate), _ptr(s_gate), _ptr(g_gate), _ptr(q_up),
                                      _ptr(s_up), _ptr(g_up), _ptr(q_down), _ptr(s_down),
                                      _ptr(g_down), _ptr(packed), _stream(stream)))
    return packed


def moe_dequant_nvfp4(packed_nvfp4: torch.Tensor, packed: torch.Tensor | None = None,
                      stream=None) -> torch.Tensor:
    """The packed bf16/fp16 layer (moe_pack_weights layout) of a packed NVFP4 layer."""
    if packed is None:
        packed = torch.empty(packed_weight_bytes() // 2, dtype=torch.bfloat16,
                             device=packed_nvfp4.device)
    _check("moe_dequant_nvfp4",
           lib.moe_dequant_nvfp4(_ptr(packed_nvfp4), _ptr(packed), _stream(stream)))
    return packed


def moe_expert_ffn_nvfp4(x: torch.Tensor, packed_nvfp4: torch.Tensor, offsets: torch.Tensor,
                         perm_src: torch.Tensor, h=None, y_perm=None, workspace=None,
                         stream=None):
    """Step 3 with NVFP4 experts (see include/moe.h); returns (h, y_perm)."""
    T = x.shape[0]
    n = T * TOPK
    if h is None:
        h = torch.empty((n, INTER), dtype=torch.float16, device=x.device)
    if y_perm is None:
        y_perm = torch.empty((n, HIDDEN), dtype=torch.float16, device=x.device)
    need = int(lib.moe_expert_ffn_nvfp4_workspace_bytes(T))
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    _check("moe_expert_ffn_nvfp4",
           lib.moe_expert_ffn_nvfp4(_ptr(x), _ptr(packed_nvfp4), _ptr(offsets), _ptr(perm_src),
                                    T, _ptr(h), _ptr(y_perm), _ptr(workspace),
                                    workspace.numel() if workspace is not None else 0,
                                    _stream(stream)))
    return h, y_perm


def moe_layer_nvfp4(x: torch.Tensor, logits: torch.Tensor, bias: torch.Tensor | None,
                    packed_nvfp4: torch.Tensor, residual=None, out=None, topk_idx_out=None,
                    topk_w_out=None, workspace: torch.Tensor | None = None, stream=None):
    """moe_layer with NVFP4 experts (see include/moe.h)."""
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, HIDDEN), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = alloc_layer_workspace(T, x.device, fp8=True)
    _check("moe_layer_nvfp4",
           lib.moe_layer_nvfp4(_ptr(x), _ptr(logits), _ptr(bias), _ptr(packed_nvfp4), T,
                               _ptr(residual), _ptr(out), _ptr(topk_idx_out), _ptr(topk_w_out),
                               _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


# ----------------------------------------------------------------- shared experts

def moe_pack_experts(w_gate: torch.Tensor, w_up: torch.Tensor, w_down: torch.Tensor,
                     packed: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Pack a slice of n experts ([n,1536,512], [n,1536,512], [n,512,1536] bf16),
    renumbered 0..n-1 (see include/moe.h)."""
    n = w_gate.shape[0]
    for t, shp in ((w_gate, (n, HIDDEN, INTER)), (w_up, (n, HIDDEN, INTER)),
                   (w_down, (n, INTER, HIDDEN))):
        if t.dtype != torch.bfloat16 or tuple(t.shape) != shp or not t.is_contiguous() \
                or not t.is_cuda:
            raise ValueError(f"expected contiguous CUDA bf16 {shp}")
    nbytes = int(lib.moe_packed_experts_bytes(n))
    if packed is None:
        packed = torch.empty(nbytes // 2, dtype=torch.bfloat16, device=w_gate.device)
    _check("moe_pack_experts", lib.moe_pack_experts(_ptr(w_gate), _ptr(w_up), _ptr(w_down), n,
                                                    _ptr(packed), _stream(stream)))
    return packed


def moe_expert_ffn_slice(x: torch.Tensor, packed: torch.Tensor, n_experts: int,
                         offsets: torch.Tensor, perm_src: torch.Tensor, h: torch.Tensor,
                         y_perm: torch.Tensor, stream=None) -> torch.Tensor:
    """moe_expert_ffn over a packed slice of n_experts experts (local ids)."""
    _check("moe_expert_ffn_slice",
           lib.moe_expert_ffn_slice(_ptr(x), _ptr(packed), n_experts, _ptr(offsets),
                                    _ptr(perm_src), x.shape[0], _ptr(h), _ptr(y_perm),
                                    _stream(stream)))
    return y_perm


def packed_shared_bytes(n_shared: int) -> int:
    return int(lib.moe_packed_shared_bytes(n_shared))


def layer_shared_workspace_bytes(T: int, n_shared: int, fp8_routed: bool) -> int:
    return int(lib.moe_layer_shared_workspace_bytes(T, n_shared, int(bool(fp8_routed))))


def moe_pack_shared(w_gate: torch.Tensor, w_up: torch.Tensor, w_down: torch.Tensor,
                    packed: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Re-layout n_shared shared experts ([n, 1536, 512], [n, 1536, 512],
    [n, 512, 1536] bf16; see include/moe.h)."""
    n = w_gate.shape[0]
    for t, shp in ((w_gate, (n, HIDDEN, INTER)), (w_up, (n, HIDDEN, INTER)),
                   (w_down, (n, INTER, HIDDEN))):
        if t.dtype != torch.bfloat16 or tuple(t.shape) != shp or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"expected contiguous CUDA bf16 {shp}, got {t.dtype} {tuple(t.shape)}")
    if packed is None:
        packed = torch.empty(packed_shared_bytes(n) // 2, dtype=torch.bfloat16,
                             device=w_gate.device)
    _check("moe_pack_shared", lib.moe_pack_shared(_ptr(w_gate), _ptr(w_up), _ptr(w_down), n,
                                                  _ptr(packed), _stream(stream)))
    return packed


def moe_layer_shared(x: torch.Tensor, logits: torch.Tensor, bias: torch.Tensor | None,
                     packed_shared: torch.Tensor, n_shared: int, packed_w=None, packed_fp8=None,
                     residual=None, out=None, topk_idx_out=None, topk_w_out=None,
                     workspace: torch.Tensor | None = None, stream=None, packed_nvfp4=None):
    """moe_layer (packed_w), moe_layer_fp8 (packed_fp8) or moe_layer_nvfp4
    (packed_nvfp4) plus n_shared shared experts (see include/moe.h)."""
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, HIDDEN), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        quant = packed_fp8 is not None or packed_nvfp4 is not None
        n = layer_shared_workspace_bytes(T, n_shared, quant)
        raw = torch.empty(n + 1024, dtype=torch.uint8, device=x.device)
        off = (-raw.data_ptr()) % 1024
        workspace = raw[off:off + n]
    if packed_nvfp4 is not None:
        if packed_w is not None or packed_fp8 is not None:
            raise ValueError("exactly one of packed_w, packed_fp8, packed_nvfp4")
        _check("moe_layer_shared_nvfp4",
               lib.moe_layer_shared_nvfp4(_ptr(x), _ptr(logits), _ptr(bias), _ptr(packed_nvfp4),
                                          _ptr(packed_shared), n_shared, T, _ptr(residual),
                                          _ptr(out), _ptr(topk_idx_out), _ptr(topk_w_out),
                                          _ptr(workspace), workspace.numel(), _stream(stream)))
        return out
    _check("moe_layer_shared",
           lib.moe_layer_shared(_ptr(x), _ptr(logits), _ptr(bias), _ptr(packed_w),
                                _ptr(packed_fp8), _ptr(packed_shared), n_shared, T,
                                _ptr(residual), _ptr(out), _ptr(topk_idx_out), _ptr(topk_w_out),
                                _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


# ----------------------------------------------------------------- second shape (256 experts)

E256_EXPERTS, E256_TOPK = 256, 6


def layer_e256_workspace_bytes(T: int, n_shared: int) -> int:
    return int(lib.moe_layer_e256_workspace_bytes(T, n_shared))


def moe_route_e256(logits: torch.Tensor, bias: torch.Tensor | None, topk_idx=None, topk_w=None,
                   stream=None):
    """Routing on the second shape: logits [T, 256] -> ([T, 6] int32, [T, 6] fp32)."""
    T = logits.shape[0]
    if topk_idx is None:
        topk_idx = torch.empty((T, E256_TOPK), dtype=torch.int32, device=logits.device)
    if topk_w is None:
        topk_w = torch.empty((T, E256_TOPK), dtype=torch.float32, device=logits.device)
    _check("moe_route_e256", lib.moe_route_e256(_ptr(logits), _ptr(bias), T, _ptr(topk_idx),
                                                _ptr(topk_w), _stream(stream)))
    return topk_idx, topk_w


def moe_layer_e256(x: torch.Tensor, logits: torch.Tensor, bias: torch.Tensor | None,
                   packed_lo: torch.Tensor, packed_hi: torch.Tensor, packed_shared=None,
                   n_shared: int = 0, residual=None, out=None, topk_idx_out=None,
                   topk_w_out=None, workspace: torch.Tensor | None = None, stream=None):
    """The layer on the second shape (256 experts top-6, see include/moe.h)."""
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, HIDDEN), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        n = layer_e256_workspace_bytes(T, n_shared)
        raw = torch.empty(n + 1024, dtype=torch.uint8, device=x.device)
        off = (-raw.data_ptr()) % 1024
        workspace = raw[off:off + n]
    _check("moe_layer_e256",
           lib.moe_layer_e256(_ptr(x), _ptr(logits), _ptr(bias), _ptr(packed_lo), _ptr(packed_hi),
                              _ptr(packed_shared), n_shared, T, _ptr(residual), _ptr(out),
                              _ptr(topk_idx_out), _ptr(topk_w_out), _ptr(workspace),
                              workspace.numel(), _stream(stream)))
    return out


WEIGHT_FORMATS = {"bf16": 0, "fp8": 1, "nvfp4": 2}


def alloc_layer_host_workspace(T: int, device, weight_format: int = 0) -> torch.Tensor:
    n = int(lib.moe_layer_host_workspace_bytes(T, weight_format))
    raw = torch.empty(n + 1024, dtype=torch.uint8, device=device)
    off = (-raw.data_ptr()) % 1024
    return raw[off:off + n]


def _event(ev):
    return None if ev is None else ctypes.c_void_p(ev.cuda_event)


def moe_layer_host(x_host: torch.Tensor, logits_host: torch.Tensor, bias: torch.Tensor | None,
                   packed: torch.Tensor, out_host: torch.Tensor, workspace: torch.Tensor,
                   weight_format: int = 0, wait_event=None, done_event=None, stream=None):
    """The layer from host buffers through the C ABI (moe_layer_host): x and
    the router logits copied in, the layer, the output copied out, all on
    `stream`.  wait_event / done_event: recorded torch.cuda.Event objects, or
    None (see include/moe.h)."""
    for t, shp, dt in ((x_host, (None, HIDDEN), torch.bfloat16), (logits_host, (None, N_EXPERTS),
                       torch.float32), (out_host, (None, HIDDEN), torch.bfloat16)):
        if t.is_cuda or t.dtype != dt or t.dim() != 2 or t.shape[1] != shp[1] \
                or not t.is_contiguous():
            raise ValueError("host buffers: contiguous CPU tensors of the layer's shapes")
    T = x_host.shape[0]
    _check("moe_layer_host",
           lib.moe_layer_host(_ptr(x_host), _ptr(logits_host), _ptr(bias), _ptr(packed),
                              weight_format, T, _ptr(out_host), _ptr(workspace),
                              workspace.numel(), _event(wait_event), _event(done_event),
                              _stream(stream)))
    return out_host


def moe_layer_from_host(x_host: torch.Tensor, logits_host: torch.Tensor, bias: torch.Tensor | None,
                        packed_w: torch.Tensor, out_host: torch.Tensor,
                        workspace: torch.Tensor, stream=None) -> torch.Tensor:
    """End-to-end call from pinned host buffers (bf16 experts): moe_layer_host
    with a workspace from alloc_layer_host_workspace."""
    return moe_layer_host(x_host, logits_host, bias, packed_w, out_host, workspace, 0,
                          stream=stream)


class HostPipeline:
    """Layer calls from pinned host buffers with `depth` calls in flight.

    Each slot owns a device workspace and a stream; call k uses slot k % depth
    and goes through the C ABI's moe_layer_host (copies in, layer, copy out)
    unless shared experts are given (their layer call has no host-buffer
    form: then the copies are torch copies around moe_layer_shared).  Its host-to-device copies may overlap the previous
    call's layer, and its device-to-host copy the next call's layer, but the
    layers themselves run one after another (each waits for the previous
    call's layer), so two calls never share the weights they stream through
    L2.  Stream order keeps a slot's buffers from being reused before its
    previous call has finished.  The output of call k lands in the `out_host`
    passed to submit(); it is complete once `drain()` returns.  With fp8=True
    the weights passed to submit() are a packed block-FP8 layer and every call
    runs moe_layer_fp8; with nvfp4=True a packed NVFP4 layer (moe_layer_nvfp4).  With shared = (packed_shared, n_shared) every call
    also runs the shared experts (moe_layer_shared).
    """

    def __init__(self, T: int, device, depth: int = 2, fp8: bool = False, shared=None,
                 nvfp4: bool = False):
        if nvfp4 and fp8:
            raise ValueError("one routed-expert format: fp8 or nvfp4")
        self.T, self.depth, self.k, self.shared = T, depth, 0, shared
        self.fp8, self.nvfp4 = fp8 or nvfp4, nvfp4
        self.last_layer = None
        self.fmt = 2 if nvfp4 else 1 if fp8 else 0
        self.slots = []
        for _ in range(depth):
            st = torch.cuda.Stream(device)
            done = torch.cuda.Event()
            done.record(st)  # creates the event before the library records it
            self.slots.append({
                "stream": st, "done": done,
                "x": torch.empty((T, HIDDEN), dtype=torch.bfloat16, device=device),
                "logits": torch.empty((T, N_EXPERTS), dtype=torch.float32, device=device),
                "out": torch.empty((T, HIDDEN), dtype=torch.bfloat16, device=device),
                "ws": (self._workspace(T, device) if shared is not None else
                       alloc_layer_host_workspace(T, device, self.fmt)),
            })

    def _workspace(self, T, device):
        if self.shared is None:
            return alloc_layer_workspace(T, device, fp8=self.fp8)
        n = layer_shared_workspace_bytes(T, self.shared[1], self.fp8)
        raw = torch.empty(n + 1024, dtype=torch.uint8, device=device)
        off = (-raw.data_ptr()) % 1024
        return raw[off:off + n]

    def submit(self, x_host, logits_host, out_host, bias, packed_w):
        slot = self.slots[self.k % self.depth]
        self.k += 1
        st = slot["stream"]
        if self.shared is None:
            moe_layer_host(x_host, logits_host, bias, packed_w, out_host, slot["ws"], self.fmt,
                           wait_event=self.last_layer, done_event=slot["done"], stream=st)
            self.last_layer = slot["done"]
            return out_host
        with torch.cuda.stream(st):
            slot["x"].copy_(x_host, non_blocking=True)
            slot["logits"].copy_(logits_host, non_blocking=True)
            if self.last_layer is not None:
                st.wait_event(self.last_layer)
            if self.shared is not None:
                kw = ({"packed_nvfp4": packed_w} if self.nvfp4 else
                      {"packed_fp8": packed_w} if self.fp8 else {"packed_w": packed_w})
                moe_layer_shared(slot["x"], slot["logits"], bias, self.shared[0], self.shared[1],
                                 out=slot["out"], workspace=slot["ws"], stream=st, **kw)
            else:
                (moe_layer_nvfp4 if self.nvfp4 else moe_layer_fp8 if self.fp8 else moe_layer)(
                    slot["x"], slot["logits"], bias, packed_w, out=slot["out"],
                    workspace=slot["ws"], stream=st)
            self.last_layer = torch.cuda.Event()
            self.last_layer.record(st)
            out_host.copy_(slot["out"], non_blocking=True)
        return out_host

    def streams(self):
        return [slot["stream"] for slot in self.slots]

    def drain(self):
        for st in self.streams():
            st.synchronize()


# ----------------------------------------------------------------- status

def get_device_status(device: int = 0) -> int:
    return int(lib.moe_get_device_status(device))


def init_device() -> None:
    """Per-device set-up of the library on the current device (do it before
    capturing library calls into a CUDA graph)."""
    _check("moe_init_device", lib.moe_init_device())


def set_ffn_trace(buf: torch.Tensor | None) -> None:
    """Per-CTA timing record of the expert-FFN launches into buf (int64 [n, 3]:
    start ns, end ns, tiles), or off with None (see include/moe.h)."""
    if buf is None:
        _check("moe_set_ffn_trace", lib.moe_set_ffn_trace(None, 0))
        return
    if buf.dtype != torch.int64 or buf.dim() != 2 or buf.shape[1] != 3 or not buf.is_cuda \
            or not buf.is_contiguous():
        raise ValueError("expected a contiguous CUDA int64 tensor [n, 3]")
    _check("moe_set_ffn_trace", lib.moe_set_ffn_trace(_ptr(buf), buf.shape[0]))


def set_wait_timeout_ns(ns: int) -> None:
    _check("moe_set_wait_timeout_ns", lib.moe_set_wait_timeout_ns(ns))


def selftest_wait_timeout(stream=None) -> None:
    _check("moe_selftest_wait_timeout", lib.moe_selftest_wait_timeout(_stream(stream)))
