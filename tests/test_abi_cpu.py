"""Host-side checks of the C-ABI library that need no GPU: it loads, it exports
every function include/bitnet.h declares, and its argument validation rejects bad
calls before any CUDA work is attempted."""
import ctypes
import re

import pytest

from ternary_weight_bit_b200 import _native


@pytest.fixture(scope="module")
def L():
    return _native.load()


def test_header_declares_the_boundary():
    names = _native.declared_symbols()
    for required in ("bitnet_pack_ternary", "bitnet_act_quant", "bitnet_ternary_gemm",
                     "bitnet_hbitlinear_forward"):
        assert required in names
    assert len(names) >= 10


def test_library_exports_every_declared_symbol(L):
    for name in _native.declared_symbols():
        assert hasattr(L, name), f"{name} declared in bitnet.h but not exported"


def test_abi_version_and_status_strings(L):
    assert L.bitnet_abi_version() == 8
    for s in range(7):
        assert L.bitnet_status_string(s)
    assert L.bitnet_status_string(5).decode().startswith("a kernel gave up")


def test_gemm_token_tile_host_logic(L):
    # decode-sized and rejected problems are answered on the host, without touching a GPU
    assert L.bitnet_gemm_token_tile(16, 4096, 4096) == 0
    assert L.bitnet_gemm_token_tile(1, 2560, 6912) == 0
    assert L.bitnet_gemm_token_tile(-1, 256, 256) == -1
    assert L.bitnet_gemm_token_tile(64, 0, 256) == -1
    assert L.bitnet_gemm_token_tile(64, 256, 100) == -1
    sp = ctypes.c_int(-5)
    assert L.bitnet_forward_gemm_plan(8, 2560, 6912, ctypes.byref(sp)) == 0 and sp.value == 0
    assert L.bitnet_forward_gemm_plan(64, 0, 256, ctypes.byref(sp)) == -1
    for bad in (1, 32, 96, 160, 255, 257, 512, -64):
        assert L.bitnet_gemm_force_token_tile(bad) == _native.ERR_INVALID_ARG
    try:
        for good in (256, 224, 192, 128, 64):
            assert L.bitnet_gemm_force_token_tile(good) == _native.OK
            assert L.bitnet_gemm_token_tile(4096, 4096, 4096) == good  # a forced tile wins
    finally:
        assert L.bitnet_gemm_force_token_tile(0) == _native.OK


def test_forward_split_plans(L):
    # the forward's (token tile, k-split) plans for the sweep shapes on a 148-SM B200
    # (the host answers without a GPU): two halves at 128-256 tokens of long K, four
    # atomic splits at 64 tokens, no split at 512 (measured faster unsplit)
    def plan(M, N, K):
        sp = ctypes.c_int(-1)
        bt = L.bitnet_forward_gemm_plan(M, N, K, ctypes.byref(sp))
        return bt, sp.value
    assert plan(256, 4096, 16384) == (128, 2)
    assert plan(128, 2048, 8192) == (64, 2)
    assert plan(64, 4096, 16384) == (64, 4)
    assert plan(512, 4096, 16384) == (128, 1)
    assert plan(4096, 4096, 4096) == (224, 1)
    for bad in (3, 5, 16, -1):
        assert L.bitnet_gemm_force_k_splits(bad) == _native.ERR_INVALID_ARG
    try:
        for forced in (1, 2, 4, 8):
            assert L.bitnet_gemm_force_k_splits(forced) == _native.OK
            assert plan(512, 4096, 16384)[1] == forced
        assert L.bitnet_gemm_force_k_splits(8) == _native.OK
        # 8 k-blocks: a split needs at least 4 per part, so the automatic plan stands
        assert plan(64, 4096, 1024) == (64, 1)
    finally:
        assert L.bitnet_gemm_force_k_splits(0) == _native.OK
    assert L.bitnet_gemm_token_tile(512, 4096, 16384) == 128  # the standalone GEMM never splits


def test_kv_quant_validation(L):
    s = P(0)
    ok = _native.OK
    assert L.bitnet_kv_quant(FAKE, 0, 2, 3, 128, 5, 1e-5, FAKE, FAKE, None, s) == _native.ERR_INVALID_ARG   # bits
    assert L.bitnet_kv_quant(FAKE, 2, 2, 3, 128, 4, 1e-5, FAKE, FAKE, None, s) == _native.ERR_INVALID_ARG   # dtype
    assert L.bitnet_kv_quant(FAKE, 0, 2, 3, 130, 4, 1e-5, FAKE, FAKE, None, s) == _native.ERR_UNSUPPORTED_SHAPE
    assert L.bitnet_kv_quant(FAKE, 0, 2, 3, 2048, 4, 1e-5, FAKE, FAKE, None, s) == _native.ERR_UNSUPPORTED_SHAPE
    assert L.bitnet_kv_quant(FAKE, 0, -1, 3, 128, 4, 1e-5, FAKE, FAKE, None, s) == _native.ERR_INVALID_ARG
    assert L.bitnet_kv_quant(None, 0, 0, 3, 128, 3, 1e-5, None, None, None, s) == ok   # empty: nothing to do
    assert L.bitnet_kv_quant(None, 0, 2, 3, 128, 3, 1e-5, FAKE, FAKE, None, s) == _native.ERR_INVALID_ARG
    assert L.bitnet_kv_quant(P(4100), 0, 2, 3, 128, 3, 1e-5, FAKE, FAKE, None, s) == _native.ERR_INVALID_ARG


def test_out_dtype_validation(L):
    s = P(0)
    # an output dtype other than fp32 / bf16 is refused before anything else is looked at
    assert L.bitnet_ternary_gemm_ex(FAKE, FAKE, 0, FAKE, FAKE, 4, 256, 256, FAKE, 2, None, s) == _native.ERR_INVALID_ARG
    assert L.bitnet_hbitlinear_forward_ex(FAKE, 0, 4, 256, None, 1e-5, 0, 0, FAKE, FAKE, 256, FAKE, 7, FAKE, 1 << 20,
                                          s) == _native.ERR_INVALID_ARG
    # the shape checks still apply with a valid output dtype
    assert L.bitnet_ternary_gemm_ex(FAKE, FAKE, 0, FAKE, FAKE, 4, 256, 100, FAKE, 1, None, s) == \
        _native.ERR_UNSUPPORTED_SHAPE
    assert L.bitnet_hbitlinear_forward_ex(FAKE, 0, 4, 256, None, 1e-5, 0, 0, FAKE, FAKE, 256, P(4100), 1, FAKE,
                                          1 << 20, s) == _native.ERR_INVALID_ARG  # misaligned out
    assert L.bitnet_ternary_gemm_ex(None, None, 0, None, None, 0, 256, 256, None, 1, None, s) == _native.OK  # M = 0


# The boundary's calls with their parameter lists, as include/bitnet.h declares them.
BOUNDARY = {
    "bitnet_pack_ternary": ["const float *W", "int64_t N", "int64_t K", "float eps", "uint8_t *packed",
                            "float *alpha", "void *ws", "size_t ws_bytes", "void *stream"],
    "bitnet_act_quant": ["const void *X", "bitnet_dtype_t xdt", "int64_t M", "int64_t K", "const float *gain",
                         "float eps", "int fwht", "bitnet_act_mode_t mode", "int8_t *codes", "float *scale_x",
                         "void *stream"],
    "bitnet_ternary_gemm": ["const int8_t *codes", "const float *scale_x", "bitnet_act_mode_t mode",
                            "const uint8_t *packed", "const float *alpha", "int64_t M", "int64_t N", "int64_t K",
                            "float *out", "int32_t *acc_out", "void *ws", "size_t ws_bytes", "void *stream"],
    "bitnet_hbitlinear_forward": ["const void *X", "bitnet_dtype_t xdt", "int64_t M", "int64_t K",
                                  "const float *gain", "float eps", "int fwht", "bitnet_act_mode_t mode",
                                  "const uint8_t *packed", "const float *alpha", "int64_t N", "float *out",
                                  "void *ws", "size_t ws_bytes", "void *stream"],
    "bitnet_workspace_bytes": ["int64_t M", "int64_t N", "int64_t K"],
    "bitnet_status_string": ["bitnet_status_t status"],
    "bitnet_get_last_device_status": ["void *stream"],
}


def _declared_params(name):
    src = open(_native.HEADER).read()
    m = re.search(r"BITNET_API[^;]*?\b" + name + r"\s*\(([^)]*)\)\s*;", src, re.S)
    assert m, f"{name} is not declared in bitnet.h"
    return [" ".join(p.split()) for p in m.group(1).split(",")]


def test_boundary_calls_have_their_listed_signatures(L):
    for name, params in BOUNDARY.items():
        assert _declared_params(name) == params, name
        assert hasattr(L, name)


def test_workspace_sizes(L):
    cnt = 4096  # split-K tile counters
    assert L.bitnet_forward_workspace_bytes(0, 256) == 0
    assert L.bitnet_forward_workspace_bytes(1, 256) == 256 + 256 + cnt
    assert L.bitnet_forward_workspace_bytes(3, 2560) == 7680 + 256 + cnt
    assert L.bitnet_forward_workspace_bytes(100, 128) == 12800 + 512 + cnt
    assert L.bitnet_pack_workspace_bytes(6912, 2560) >= 8 * 1184
    assert L.bitnet_gemm_workspace_bytes(64, 4096, 16384) == cnt
    for M, N, K in ((1, 6912, 2560), (64, 4096, 16384), (8192, 4096, 4096)):
        assert L.bitnet_workspace_bytes(M, N, K) == max(L.bitnet_pack_workspace_bytes(N, K),
                                                        L.bitnet_forward_workspace_bytes(M, K),
                                                        L.bitnet_gemm_workspace_bytes(M, N, K))


def test_forward_kernel_count(L):
    # the activation kernel, then the decode kernel or the tcgen05 GEMM; answered on the host
    assert L.bitnet_forward_kernel_count(1, 6912, 2560, 0, 0) == 2
    assert L.bitnet_forward_kernel_count(4096, 4096, 4096, 1, 1) == 2
    assert L.bitnet_forward_kernel_count(0, 4096, 4096, 0, 0) == 0
    assert L.bitnet_forward_kernel_count(4, 4096, 2560, 1, 0) == -1     # FWHT needs a power of two
    assert L.bitnet_forward_kernel_count(4, 0, 4096, 0, 0) == -1


def test_tl2_host_logic(L):
    # 20 bytes per 96 weights of a row; decode sizes only; the usual argument checks
    assert L.bitnet_tl2_bytes(1, 96) == 20 and L.bitnet_tl2_bytes(3, 2560) == 3 * 20 * 27
    assert L.bitnet_tl2_bytes(1, 6912) * 8 / 6912 == pytest.approx(5 / 3)
    s = P(0)
    assert L.bitnet_ternary_gemm_tl2(FAKE, FAKE, 0, FAKE, FAKE, 17, 256, 256, FAKE, None, s) == \
        _native.ERR_UNSUPPORTED_SHAPE
    assert L.bitnet_ternary_gemm_tl2(FAKE, FAKE, 0, FAKE, FAKE, 4, 256, 100, FAKE, None, s) == \
        _native.ERR_UNSUPPORTED_SHAPE
    assert L.bitnet_hbitlinear_forward_tl2(FAKE, 0, 32, 256, None, 1e-5, 0, 0, FAKE, FAKE, 64, FAKE, FAKE, 1 << 20,
                                           s) == _native.ERR_UNSUPPORTED_SHAPE
    assert L.bitnet_pack_tl2(FAKE, 16, 256, P(4100), s) == _native.ERR_INVALID_ARG
    assert L.bitnet_ternary_gemm_tl2(None, None, 0, None, None, 0, 16, 256, None, None, s) == _native.OK


def test_gemm_workspace_validation(L):
    s = P(0)
    # a workspace is optional; one that is given must be large enough and 256-byte aligned
    assert L.bitnet_ternary_gemm(FAKE, FAKE, 0, FAKE, FAKE, 64, 256, 256, FAKE, None, FAKE, 16, s) == \
        _native.ERR_WORKSPACE
    assert L.bitnet_ternary_gemm(FAKE, FAKE, 0, FAKE, FAKE, 64, 256, 256, FAKE, None, P(4096 + 16), 1 << 20, s) == \
        _native.ERR_WORKSPACE


P = ctypes.c_void_p
FAKE = P(4096)  # never dereferenced: validation fails first


def test_validation_rejects_bad_shapes(L):
    s = P(0)
    # K not a multiple of 128
    assert L.bitnet_act_quant(FAKE, 0, 4, 100, None, 1e-5, 0, 0, FAKE, FAKE, s) == _native.ERR_UNSUPPORTED_SHAPE
    # K too large
    assert L.bitnet_act_quant(FAKE, 0, 4, 65536, None, 1e-5, 0, 0, FAKE, FAKE, s) == _native.ERR_UNSUPPORTED_SHAPE
    # FWHT with K not a power of two (the page's ValueError)
    assert L.bitnet_act_quant(FAKE, 0, 4, 2560, None, 1e-5, 1, 0, FAKE, FAKE, s) == _native.ERR_NOT_POW2
    assert L.bitnet_hbitlinear_forward(FAKE, 0, 4, 6912, None, 1e-5, 1, 0, FAKE, FAKE, 16, FAKE, FAKE, 1 << 20,
                                       s) == _native.ERR_NOT_POW2
    # bad enums
    assert L.bitnet_act_quant(FAKE, 7, 4, 256, None, 1e-5, 0, 0, FAKE, FAKE, s) == _native.ERR_INVALID_ARG
    assert L.bitnet_act_quant(FAKE, 0, 4, 256, None, 1e-5, 0, 9, FAKE, FAKE, s) == _native.ERR_INVALID_ARG
    assert L.bitnet_ternary_gemm(FAKE, FAKE, 3, FAKE, FAKE, 4, 16, 256, FAKE, None, None, 0, s) == _native.ERR_INVALID_ARG
    # negative sizes, N = 0
    assert L.bitnet_ternary_gemm(FAKE, FAKE, 0, FAKE, FAKE, -1, 16, 256, FAKE, None, None, 0, s) == _native.ERR_INVALID_ARG
    assert L.bitnet_ternary_gemm(FAKE, FAKE, 0, FAKE, FAKE, 4, 0, 256, FAKE, None, None, 0, s) == _native.ERR_INVALID_ARG


def test_validation_rejects_bad_pointers(L):
    s = P(0)
    assert L.bitnet_act_quant(None, 0, 4, 256, None, 1e-5, 0, 0, FAKE, FAKE, s) == _native.ERR_INVALID_ARG
    assert L.bitnet_act_quant(P(4100), 0, 4, 256, None, 1e-5, 0, 0, FAKE, FAKE, s) == _native.ERR_INVALID_ARG
    assert L.bitnet_ternary_gemm(FAKE, FAKE, 0, None, FAKE, 4, 16, 256, FAKE, None, None, 0, s) == _native.ERR_INVALID_ARG
    assert L.bitnet_ternary_gemm(FAKE, FAKE, 0, FAKE, FAKE, 4, 16, 256, P(4104), None, None, 0, s) == _native.ERR_INVALID_ARG
    assert L.bitnet_pack_ternary(FAKE, 16, 256, 1e-5, FAKE, FAKE, None, 0, s) == _native.ERR_WORKSPACE
    assert L.bitnet_pack_ternary(FAKE, 16, 256, 1e-5, FAKE, P(4108), FAKE, 1 << 20, s) == _native.ERR_INVALID_ARG
    # forward workspace too small, or misaligned
    assert L.bitnet_hbitlinear_forward(FAKE, 0, 4, 256, None, 1e-5, 1, 0, FAKE, FAKE, 16, FAKE, FAKE, 16,
                                       s) == _native.ERR_WORKSPACE
    assert L.bitnet_hbitlinear_forward(FAKE, 0, 4, 256, None, 1e-5, 1, 0, FAKE, FAKE, 16, FAKE, P(4096 + 16),
                                       1 << 20, s) == _native.ERR_WORKSPACE
    assert L.bitnet_selftest_wait_timeout(0, s) == _native.ERR_INVALID_ARG
    assert L.bitnet_selftest_wait_timeout(2000000, s) == _native.ERR_INVALID_ARG


def test_empty_batch_is_a_noop(L):
    s = P(0)
    assert L.bitnet_act_quant(None, 0, 0, 256, None, 1e-5, 1, 0, None, None, s) == _native.OK
    assert L.bitnet_ternary_gemm(None, None, 0, None, None, 0, 16, 256, None, None, None, 0, s) == _native.OK
    assert L.bitnet_hbitlinear_forward(None, 0, 0, 256, None, 1e-5, 1, 0, FAKE, FAKE, 16, FAKE, None, 0,
                                       s) == _native.OK


def test_no_cpu_fallback():
    # the product path refuses host tensors instead of computing anything on the CPU
    import pytest
    import torch
    import ternary_weight_bit_b200 as tb
    X = torch.randn(4, 256)
    W = torch.randn(64, 256)
    with pytest.raises(ValueError, match="CUDA"):
        tb.bitnet_pack_ternary(W)
    with pytest.raises(ValueError, match="CUDA"):
        tb.bitnet_act_quant(X)
    with pytest.raises(ValueError, match="CUDA"):
        tb.bitnet_hbitlinear_forward(X, torch.zeros(64, 64, dtype=torch.uint8), torch.ones(1), 64)
    with pytest.raises(ValueError, match="CUDA"):
        tb.bitnet_kv_quant(torch.randn(1, 2, 3, 64))
    with pytest.raises(RuntimeError, match="not built"):
        _native.load("/nonexistent/libbitnet.so")
