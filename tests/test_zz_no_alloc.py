"""The allocation-free forward entry point, through the C ABI.

bitnet_hbitlinear_forward_noalloc serves callers that cannot allocate device
memory (plugin interfaces that pass only inputs and outputs, runtimes that own
all device memory, paths that must never reach cudaMalloc): its scratch is a
fixed array inside the library.  These checks compare it with the
workspace-taking bitnet_hbitlinear_forward on calls in a row -- different
shapes, so a stale scratch from one call would show in the next -- including
GEMMs that split K, whose tile counters and pair flags live in that array too;
check the workspace forward itself against the oracle on the split shape; and
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
from oracle import ref
from ternary_weight_bit_b200 import _native, synthetic

pytestmark = pytest.mark.gpu

DEV = "cuda"
MODES = {"int8": ref.ACT_INT8, "int4": ref.ACT_INT4}


def _vp(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _noalloc(L, X, packed, alpha, N, fwht, mode, out):
    M, K = X.shape
    xdt = _native.BF16 if X.dtype == torch.bfloat16 else _native.F32
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.bitnet_hbitlinear_forward_noalloc(_vp(X), xdt, M, K, None, 1e-5, int(fwht), tb.mode_id(mode),
                                               _vp(packed), _vp(alpha), N, _vp(out), stream)


def _prepared(case):
    X = case.X.to(DEV)
    packed, alpha = tb.bitnet_pack_ternary(case.W.to(DEV))
    want = tb.bitnet_hbitlinear_forward(X, packed, alpha, case.N, fwht=case.fwht, mode=case.mode)
    return X, packed, alpha, want


def _check_same(L, case, X, packed, alpha, want, calls=1):
    for i in range(calls):
        got = torch.full((case.M, case.N), float("nan"), device=DEV)
        assert _noalloc(L, X, packed, alpha, case.N, case.fwht, case.mode, got) == _native.OK
        torch.cuda.synchronize()
        parity.check_out_same_codes(got.cpu().numpy(), want.cpu().numpy().astype(np.float64),
                                    f"{case.name} call {i}")
    assert tb.bitnet_get_last_device_status() == 0


def test_noalloc_forward_matches_forward_on_two_calls():
    L = _native.load()
    cases = [
        synthetic.msweep_int4(8, 4096, N=1024, seed=21),                      # decode kernel, int4 + FWHT
        synthetic.make_case("noalloc_prefill", 200, 2048, 640, x_dtype="bf16", fwht=False, mode="int8",
                            seed=22),                                           # tcgen05 kernel, int8
        synthetic.decode(4, N=2560, K=6912, seed=23),                          # decode kernel, int8, no FWHT
    ]
    for case in cases:
        _check_same(L, case, *_prepared(case))


def test_noalloc_split_k_back_to_back():
    # GEMMs that split K keep their tile counters and pair flags in the fixed array;
    # the calls must leave them ready for the next call, so three calls in a row each
    # give the workspace forward's result.  Two halves and four atomic splits forced on
    # a 200-token shape, then the automatic four-way split of a 64-token, K = 16384
    # shape (1 MiB of codes).
    L = _native.load()
    case = synthetic.make_case("noalloc_split", 200, 4096, 1000, x_kind="student_t3", outliers=40,
                               outlier_gain=50.0, fwht=True, mode="int4", seed=24)
    try:
        for splits in (2, 4):
            tb.bitnet_gemm_force_k_splits(splits)
            assert tb.bitnet_forward_gemm_plan(case.M, case.N, case.K)[1] == splits
            _check_same(L, case, *_prepared(case), calls=3)
    finally:
        tb.bitnet_gemm_force_k_splits(0)
    big = synthetic.msweep_int4(64, 16384, N=4096, seed=25)
    assert tb.bitnet_forward_gemm_plan(big.M, big.N, big.K)[1] == 4
    _check_same(L, big, *_prepared(big), calls=3)


def test_noalloc_split_shape_against_the_oracle():
    # the 64-token split shape end to end: the noalloc output is bit-identical to the
    # workspace forward's, whose codes and scales are checked against the oracle
    L = _native.load()
    case = synthetic.msweep_int4(64, 16384, N=4096, seed=26)
    X = case.X.to(DEV)
    packed, alpha = tb.bitnet_pack_ternary(case.W.to(DEV))
    ws = torch.empty((tb.bitnet_forward_workspace_bytes(case.M, case.K),), dtype=torch.uint8, device=DEV)
    want = tb.bitnet_hbitlinear_forward(X, packed, alpha, case.N, fwht=True, mode="int4", ws=ws)
    got = torch.full((case.M, case.N), float("nan"), device=DEV)
    assert _noalloc(L, X, packed, alpha, case.N, True, "int4", got) == _native.OK
    torch.cuda.synchronize()
    assert torch.equal(got, want)
    M, K = case.M, case.K
    codes = ws[:M * K].view(torch.int8).view(M, K).cpu().numpy()
    off = (M * K + 255) // 256 * 256
    scales = ws[off:off + 4 * M].view(torch.float32).cpu().numpy()
    X32 = case.X.numpy()
    p_ref, a_ref, _ = ref.pack_weights(case.W.numpy())
    r = ref.hbitlinear_forward(X32, p_ref, a_ref, case.N, fwht_on=True, mode=ref.ACT_INT4)
    parity.check_codes(codes, r.codes, ref.shadow(X32, None, 1e-5, True, ref.ACT_INT4), case.name)
    parity.check_scale_bound(scales, r.scale_x, K, ref.ACT_INT4, case.name)
    gout = got.cpu().numpy()
    parity.check_out_same_codes(gout, ref.dequant(ref.gemm_packed(codes, p_ref, case.N), scales, a_ref,
                                                  ref.ACT_INT4), case.name)
    parity.check_out_end_to_end(gout, r.out, codes, r.codes, r.scale_x, a_ref, ref.ACT_INT4, case.name)
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
