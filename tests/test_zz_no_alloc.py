"""The allocation-free forward entry point, through the C ABI.

bitnet_hbitlinear_forward_noalloc serves callers that cannot allocate device
memory (plugin interfaces that pass only inputs and outputs, runtimes that own
all device memory, paths that must never reach cudaMalloc): its scratch is a
fixed array inside the library.  These checks compare it with the
workspace-taking bitnet_hbitlinear_forward on two calls in a row -- different
shapes, so a stale scratch from the first call would show in the second -- and
check that oversized calls are refused.

The file is named to be collected last, so a run that stops at the first
failure has already run every other test; it also passes on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

import parity
import ternary_weight_bit_b200 as tb
from ternary_weight_bit_b200 import _native, synthetic

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _vp(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _noalloc(L, X, packed, alpha, N, fwht, mode, out):
    M, K = X.shape
    xdt = _native.BF16 if X.dtype == torch.bfloat16 else _native.F32
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.bitnet_hbitlinear_forward_noalloc(_vp(X), xdt, M, K, None, 1e-5, int(fwht), tb.mode_id(mode),
                                               _vp(packed), _vp(alpha), N, _vp(out), stream)


def test_noalloc_forward_matches_forward_on_two_calls():
    L = _native.load()
    cases = [
        synthetic.msweep_int4(8, 4096, N=1024, seed=21),                      # decode kernel, int4 + FWHT
        synthetic.make_case("noalloc_prefill", 200, 2048, 640, x_dtype="bf16", fwht=False, mode="int8",
                            seed=22),                                           # tcgen05 kernel, int8
    ]
    for case in cases:
        X = case.X.to(DEV)
        packed, alpha = tb.bitnet_pack_ternary(case.W.to(DEV))
        want = tb.bitnet_hbitlinear_forward(X, packed, alpha, case.N, fwht=case.fwht, mode=case.mode)
        got = torch.full((case.M, case.N), float("nan"), device=DEV)
        assert _noalloc(L, X, packed, alpha, case.N, case.fwht, case.mode, got) == _native.OK
        torch.cuda.synchronize()
        parity.check_out_same_codes(got.cpu().numpy(), want.cpu().numpy().astype(np.float64), case.name)
    assert tb.bitnet_get_last_device_status() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    L = _native.load()
    K = 16384
    M = 512  # 512 x 16384 codes = 8 MiB > 4 MiB of scratch
    assert tb.bitnet_forward_workspace_bytes(M, K) > 4 << 20
    X = torch.ones((M, K), device=DEV)
    packed = torch.zeros((64, K // 4), dtype=torch.uint8, device=DEV)
    alpha = torch.ones((1,), device=DEV)
    out = torch.zeros((M, 64), device=DEV)
    assert _noalloc(L, X, packed, alpha, 64, True, "int8", out) == _native.ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0  # nothing was launched
