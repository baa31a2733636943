"""The C-ABI library loads on a CPU-only machine, exports every function that
include/moe.h declares, and rejects bad arguments on the host before any
CUDA call (no GPU needed)."""
import ctypes

import pytest

from group_limited_routed_moe_b200 import moe


def test_exports_every_declared_symbol():
    names = moe.header_functions()
    assert len(names) >= 15
    missing = [n for n in names if not hasattr(moe.lib, n)]
    assert missing == []
    assert moe.lib.moe_abi_version() == 6


def test_sizes():
    assert moe.packed_weight_bytes() == 128 * 3 * 1536 * 512 * 2
    assert moe.lib.moe_max_tokens() == 1 << 22
    assert moe.lib.moe_permute_workspace_bytes(1024) == 0
    # one histogram row of 128 experts per block: blocks of 64 tokens up to
    # 16384 tokens, of 128 above; rounded up to 256 bytes
    def ws(blocks):
        return blocks * 128 * 4 + (256 - (blocks * 128 * 4) % 256) % 256
    assert moe.lib.moe_permute_workspace_bytes(1025) == ws(17)
    assert moe.lib.moe_permute_workspace_bytes(16384) == ws(256)
    assert moe.lib.moe_permute_workspace_bytes(16385) == ws(129)
    assert moe.lib.moe_permute_workspace_bytes(-1) == 0
    prev = 0
    for T in (1, 4, 16, 2048, 8192):
        b = moe.layer_workspace_bytes(T)
        # h and y_perm dominate: 8T rows of (512 + 1536) bf16
        assert b >= T * 8 * (512 + 1536) * 2 and b % 1024 == 0 and b > prev
        prev = b


def _p(v):
    return ctypes.c_void_p(v)


def test_host_validation_without_gpu():
    L = moe.lib
    # T out of range
    assert L.moe_route(_p(256), None, -1, _p(256), _p(256), None) == moe.MOE_ERR_INVALID_ARG
    assert "outside" in moe.last_error()
    assert L.moe_route(_p(256), None, (1 << 22) + 1, _p(256), _p(256), None) == moe.MOE_ERR_INVALID_ARG
    # T == 0 is a no-op that touches nothing
    assert L.moe_route(None, None, 0, None, None, None) == moe.MOE_OK
    assert L.moe_expert_ffn(None, None, None, None, 0, None, None, None) == moe.MOE_OK
    assert L.moe_combine(None, None, None, 0, None, None, None) == moe.MOE_OK
    assert L.moe_layer(None, None, None, None, 0, None, None, None, None, None, 0, None) == moe.MOE_OK
    # null and misaligned pointers
    assert L.moe_route(None, None, 4, _p(256), _p(256), None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_route(_p(260), None, 4, _p(256), _p(256), None) == moe.MOE_ERR_INVALID_ARG
    assert "aligned" in moe.last_error()
    assert L.moe_expert_ffn(_p(64), _p(128), _p(16), _p(16), 4, _p(128), _p(16), None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_pack_weights(None, _p(128), _p(128), _p(128), None) == moe.MOE_ERR_INVALID_ARG
    # workspace too small / missing
    assert L.moe_permute(_p(256), 2048, _p(256), _p(256), _p(256), _p(256), None, 0, None) \
        == moe.MOE_ERR_WORKSPACE
    ws = moe.layer_workspace_bytes(16)
    assert L.moe_layer(_p(1024), _p(1024), None, _p(1024), 16, None, _p(1024), None, None,
                       _p(1024), ws - 1, None) == moe.MOE_ERR_WORKSPACE
    assert L.moe_layer(_p(1024), _p(1024), None, _p(1024), 16, None, _p(1024), None, None,
                       _p(1040), ws, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_set_wait_timeout_ns(10) == moe.MOE_ERR_INVALID_ARG


def test_binding_raises_with_message():
    with pytest.raises(moe.MoeError) as ei:
        moe._check("moe_route", moe.MOE_ERR_INVALID_ARG)
    assert "status 1" in str(ei.value)


def test_fp8_sizes_and_host_validation():
    L = moe.lib
    gu, d = 128 * 1024 * 1536, 128 * 1536 * 512
    assert moe.packed_fp8_bytes() == gu + d + 128 * (96 + 48) * 4
    # up to 256 tokens the FP8 layer streams codes; above, it expands the layer
    # into the workspace first
    for T in (1, 16, 256):
        assert moe.layer_fp8_workspace_bytes(T) == moe.layer_workspace_bytes(T)
    for T in (257, 2048):
        assert moe.layer_fp8_workspace_bytes(T) == moe.layer_workspace_bytes(T) + moe.packed_weight_bytes()
    assert L.moe_layer_fp8(None, None, None, None, 0, None, None, None, None, None, 0, None) == moe.MOE_OK
    assert L.moe_layer_fp8(_p(1024), _p(1024), None, None, 16, None, _p(1024), None, None,
                           _p(1024), 1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    ws = moe.layer_fp8_workspace_bytes(300)
    assert L.moe_layer_fp8(_p(1024), _p(1024), None, _p(1024), 300, None, _p(1024), None, None,
                           _p(1024), ws - 1, None) == moe.MOE_ERR_WORKSPACE
    assert L.moe_pack_weights_fp8(_p(128), _p(128), None, _p(128), _p(128), _p(128), _p(128),
                                  None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_dequant_fp8(_p(136), _p(128), None) == moe.MOE_ERR_INVALID_ARG


def test_nvfp4_sizes_and_host_validation():
    L = moe.lib
    codes = 128 * 1024 * 768 + 128 * 1536 * 256        # two codes per byte
    mult = (128 * 1024 * 96 + 128 * 1536 * 32) * 2      # one 16-bit multiplier per 16 weights
    assert moe.packed_nvfp4_bytes() == codes + mult
    for T in (1, 256, 257, 2048):
        assert moe.layer_nvfp4_workspace_bytes(T) == moe.layer_fp8_workspace_bytes(T)
        assert L.moe_expert_ffn_nvfp4_workspace_bytes(T) == L.moe_expert_ffn_fp8_workspace_bytes(T)
    assert L.moe_layer_nvfp4(None, None, None, None, 0, None, None, None, None, None, 0,
                             None) == moe.MOE_OK
    assert L.moe_layer_nvfp4(_p(1024), _p(1024), None, None, 16, None, _p(1024), None, None,
                             _p(1024), 1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    ws = moe.layer_nvfp4_workspace_bytes(300)
    assert L.moe_layer_nvfp4(_p(1024), _p(1024), None, _p(1024), 300, None, _p(1024), None,
                             None, _p(1024), ws - 1, None) == moe.MOE_ERR_WORKSPACE
    args = [_p(128)] * 9
    for i in range(9):  # every input pointer is required
        a = list(args)
        a[i] = None
        assert L.moe_pack_weights_nvfp4(*a, _p(128), None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_pack_weights_nvfp4(*args, _p(136), None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_dequant_nvfp4(_p(136), _p(128), None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_expert_ffn_nvfp4(_p(128), _p(128), _p(128), _p(128), 300, _p(128), _p(128),
                                  None, 0, None) == moe.MOE_ERR_WORKSPACE
    assert L.moe_layer_shared_nvfp4(None, None, None, None, None, 0, 0, None, None, None, None,
                                    None, 0, None) == moe.MOE_OK
    assert L.moe_layer_shared_nvfp4(_p(1024), _p(1024), None, None, _p(1024), 1, 16, None,
                                    _p(1024), None, None, _p(1024), 1 << 30,
                                    None) == moe.MOE_ERR_INVALID_ARG
    ws = moe.layer_shared_workspace_bytes(300, 2, True)
    assert L.moe_layer_shared_nvfp4(_p(1024), _p(1024), None, _p(1024), _p(1024), 2, 300, None,
                                    _p(1024), None, None, _p(1024), ws - 1,
                                    None) == moe.MOE_ERR_WORKSPACE


def test_shared_sizes_and_host_validation():
    L = moe.lib
    per = (1024 * 1536 + 1536 * 512) * 2
    assert [moe.packed_shared_bytes(n) for n in (0, 1, 2, 8)] == [0, per, 2 * per, 8 * per]
    assert moe.packed_shared_bytes(9) == 0
    base = moe.layer_workspace_bytes(300)
    assert moe.layer_shared_workspace_bytes(300, 0, False) == base
    assert moe.layer_shared_workspace_bytes(300, 2, False) >= base + 2 * 300 * (4 + (512 + 1536) * 2)
    assert moe.layer_shared_workspace_bytes(300, 2, True) >= moe.layer_fp8_workspace_bytes(300)
    assert L.moe_pack_shared(_p(128), _p(128), _p(128), 0, _p(128), None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_pack_shared(_p(128), _p(128), _p(128), 9, _p(128), None) == moe.MOE_ERR_INVALID_ARG
    ws = moe.layer_shared_workspace_bytes(16, 1, False)
    # exactly one of the bf16 and FP8 routed packs
    assert L.moe_layer_shared(_p(1024), _p(1024), None, _p(1024), _p(1024), _p(1024), 1, 16, None,
                              _p(1024), None, None, _p(1024), ws, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_layer_shared(_p(1024), _p(1024), None, None, None, _p(1024), 1, 16, None,
                              _p(1024), None, None, _p(1024), ws, None) == moe.MOE_ERR_INVALID_ARG
    # shared pack required when n_shared > 0; n_shared bounded
    assert L.moe_layer_shared(_p(1024), _p(1024), None, _p(1024), None, None, 1, 16, None,
                              _p(1024), None, None, _p(1024), ws, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_layer_shared(_p(1024), _p(1024), None, _p(1024), None, _p(1024), 9, 16, None,
                              _p(1024), None, None, _p(1024), ws, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_layer_shared(_p(1024), _p(1024), None, _p(1024), None, _p(1024), 1, 16, None,
                              _p(1024), None, None, _p(1024), ws - 1, None) == moe.MOE_ERR_WORKSPACE


def test_e256_sizes_and_host_validation():
    L = moe.lib
    assert moe.layer_e256_workspace_bytes(16, 2) > moe.layer_e256_workspace_bytes(16, 0) > 0
    assert moe.layer_e256_workspace_bytes(16, 9) == 0
    ws = moe.layer_e256_workspace_bytes(16, 2)
    assert L.moe_route_e256(None, None, 0, None, None, None) == moe.MOE_OK
    assert L.moe_route_e256(_p(260), None, 4, _p(256), _p(256), None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_layer_e256(_p(1024), _p(1024), None, _p(1024), None, _p(1024), 2, 16, None,
                            _p(1024), None, None, _p(1024), ws, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_layer_e256(_p(1024), _p(1024), None, _p(1024), _p(1024), None, 2, 16, None,
                            _p(1024), None, None, _p(1024), ws, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_layer_e256(_p(1024), _p(1024), None, _p(1024), _p(1024), _p(1024), 2, 16, None,
                            _p(1024), None, None, _p(1024), ws - 1, None) == moe.MOE_ERR_WORKSPACE
