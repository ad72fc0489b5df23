"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Every comparison follows tests/parity.py: packed bytes, alpha and int32
accumulators bit-exact; activation codes equal except for one-step flips at
rounding near-ties; fp32 outputs within the stated relative bounds.  Shapes span
several tiles plus ragged tails (M, N not multiples of any tile; K with a
128-wide tail), the degenerate inputs (zero tokens, one token) and the full
benchmark sizes on sampled tokens.
"""
import math

import numpy as np
import pytest
import torch

import parity
import ternary_weight_bit_b200 as tb
from oracle import ref
from ternary_weight_bit_b200 import synthetic

pytestmark = pytest.mark.gpu

DEV = "cuda"
MODES = {"int8": ref.ACT_INT8, "int4": ref.ACT_INT4}


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def host(t):
    return t.detach().cpu().numpy()


@pytest.fixture(autouse=True)
def _clean_status():
    yield
    assert tb.bitnet_get_last_device_status() == 0, "a kernel recorded a timeout"


def _heavy_x(M, K, seed, outliers=True):
    g = synthetic.generator(seed)
    X = synthetic.student_t3((M, K), g)
    if outliers:
        X[:, synthetic.outlier_channels(K, max(1, K // 100), g)] *= 50.0
    return X


# ----------------------------------------------------------------------------- pack
@pytest.mark.parametrize("N,K", [(256, 256), (300, 384), (6912, 2560), (2560, 6912)])
def test_pack_matches_oracle(N, K):
    W = synthetic.gaussian((N, K), 0.02, synthetic.generator(N + K))
    packed, alpha = tb.bitnet_pack_ternary(W.to(DEV), eps=1e-5)
    p_ref, a_ref, _ = ref.pack_weights(W.numpy(), eps=1e-5)
    assert host(alpha)[0] == a_ref
    np.testing.assert_array_equal(host(packed), p_ref)


def test_pack_is_deterministic():
    W = synthetic.gaussian((1024, 1024), 0.02, synthetic.generator(5)).to(DEV)
    p1, a1 = tb.bitnet_pack_ternary(W)
    p2, a2 = tb.bitnet_pack_ternary(W)
    assert torch.equal(p1, p2) and torch.equal(a1, a2)


# ----------------------------------------------------------------------------- act_quant
FWHT_K = [128, 256, 512, 1024, 2048, 4096, 8192, 16384, 32768]
PLAIN_K = [128, 384, 2560, 6912, 16384]


def _act_case(M, K, fwht, mode, xdtype, use_gain, seed=0):
    X = _heavy_x(M, K, seed + K)
    if xdtype == "bf16":
        X = X.to(torch.bfloat16)
    gain = None
    if use_gain:
        gain = torch.rand(K, generator=synthetic.generator(seed + 1)) + 0.5
    Xd = X.to(DEV)
    gd = None if gain is None else gain.to(DEV)
    codes, scale = tb.bitnet_act_quant(Xd, gain=gd, eps=1e-5, fwht=fwht, mode=mode)
    X32 = X.float().numpy()
    g32 = None if gain is None else gain.numpy()
    q_ref, s_ref = ref.act_quant(X32, g32, 1e-5, fwht, MODES[mode])
    sh = ref.shadow(X32, g32, 1e-5, fwht, MODES[mode])
    label = f"M={M} K={K} fwht={fwht} {mode} {xdtype} gain={use_gain}"
    parity.check_codes(host(codes), q_ref, sh, label)
    parity.check_scale_bound(host(scale), s_ref, K, MODES[mode], label)


@pytest.mark.parametrize("K", FWHT_K)
@pytest.mark.parametrize("mode", ["int8", "int4"])
def test_act_quant_fwht(K, mode):
    _act_case(7, K, True, mode, "f32", False)


@pytest.mark.parametrize("K", PLAIN_K)
@pytest.mark.parametrize("mode", ["int8", "int4"])
def test_act_quant_plain(K, mode):
    _act_case(5, K, False, mode, "f32", False)


@pytest.mark.parametrize("fwht", [True, False])
def test_act_quant_bf16_and_gain(fwht):
    _act_case(9, 4096, fwht, "int8", "bf16", True)
    _act_case(3, 1024, fwht, "int4", "f32", True)


@pytest.mark.parametrize("K,mode,xdt,gain,M", [
    (2048, "int8", "f32", False, 300), (4096, "int4", "f32", False, 333), (8192, "int8", "bf16", False, 300),
    (16384, "int4", "f32", False, 301), (4096, "int8", "bf16", True, 500), (16384, "int8", "f32", True, 297),
    (2048, "int4", "bf16", True, 400), (8192, "int4", "f32", True, 1000),
])
def test_act_quant_fwht_streaming(K, mode, xdt, gain, M):
    # many tokens (M >= 2 x SMs): the persistent FWHT kernel (two register phases around one
    # swizzled shared-memory transpose, several tokens per CTA); every token checked against
    # the oracle
    gen = synthetic.generator(K + M)
    X = synthetic.student_t3((M, K), gen)
    X[:, synthetic.outlier_channels(K, K // 100, gen)] *= 50.0
    g = (1.0 + 0.5 * torch.rand(K, generator=gen)) if gain else None
    if xdt == "bf16":
        X = X.to(torch.bfloat16)
    codes, scale = tb.bitnet_act_quant(X.to(DEV), gain=None if g is None else g.to(DEV), fwht=True, mode=mode)
    X32 = X.float().numpy()
    gn = None if g is None else g.numpy()
    q_ref, s_ref = ref.act_quant(X32, gn, 1e-5, True, MODES[mode])
    sh = ref.shadow(X32, gn, 1e-5, True, MODES[mode])
    parity.check_codes(host(codes), q_ref, sh, f"stream K={K} {mode} {xdt} gain={gain}")
    parity.check_scale_bound(host(scale), s_ref, K, MODES[mode], f"stream K={K}")


def test_act_quant_many_tokens_flip_rate():
    # 512 tokens x 8192: the flip-rate bound is statistical, so test it on a large sample
    _act_case(512, 8192, True, "int4", "f32", False, seed=11)
    _act_case(512, 8192, True, "int8", "f32", False, seed=12)


def test_act_quant_plain_many_tokens():
    # more tokens than resident CTAs: each CTA walks several tokens, loading the next
    # one while it quantises the current one
    _act_case(3000, 2048, False, "int4", "f32", True, seed=21)
    _act_case(2500, 4096, False, "int8", "bf16", False, seed=22)
    _act_case(1300, 6912, False, "int4", "bf16", False, seed=23)


def test_act_quant_zero_and_constant_tokens():
    X = torch.zeros((4, 1024))
    X[1] = 3.0
    X[2, 5] = -7.0
    for fwht in (True, False):
        for mode in ("int8", "int4"):
            codes, scale = tb.bitnet_act_quant(X.to(DEV), fwht=fwht, mode=mode)
            q_ref, s_ref = ref.act_quant(X.numpy(), None, 1e-5, fwht, MODES[mode])
            sh = ref.shadow(X.numpy(), None, 1e-5, fwht, MODES[mode])
            parity.check_codes(host(codes), q_ref, sh, f"special rows fwht={fwht} {mode}")
            assert np.all(host(codes)[0] == 0) and host(scale)[0] == 0


# ----------------------------------------------------------------------------- GEMM on given codes
GEMM_SHAPES = [
    # decode kernel (M <= 16)
    (1, 64, 128), (2, 100, 384), (5, 700, 2560), (8, 6912, 2560), (8, 2560, 6912), (9, 130, 640),
    (16, 512, 1024),
    # tcgen05 kernel with its automatic token tile (few tiles: small tiles spread over the SMs)
    (17, 256, 128), (64, 200, 640), (128, 256, 256), (130, 300, 384), (256, 520, 1024), (300, 1000, 2048),
    (1200, 2560, 128), (2048, 2560, 256), (2000, 2600, 384), (1051, 4096, 256), (64, 40000, 128),
]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
@pytest.mark.parametrize("mode", ["int8", "int4"])
def test_gemm_exact_accumulators(M, N, K, mode):
    rng = np.random.default_rng(M * 1000003 + N * 7 + K)
    lo, hi = (-128, 128) if mode == "int8" else (-8, 8)
    q = rng.integers(lo, hi, size=(M, K)).astype(np.int8)
    t = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    packed = ref.pack(t)
    scale = rng.uniform(0.1, 10.0, size=M).astype(np.float32)
    alpha = np.array([0.0173], dtype=np.float32)
    acc = torch.empty((M, N), dtype=torch.int32, device=DEV)
    out = tb.bitnet_ternary_gemm(dev(q), dev(scale), mode, dev(packed), dev(alpha), N, acc_out=acc)
    acc_ref = ref.gemm_packed(q, packed, N)
    np.testing.assert_array_equal(host(acc), acc_ref)
    out_ref = ref.dequant(acc_ref, scale, alpha[0], MODES[mode])
    np.testing.assert_array_equal(host(out), out_ref)


def _gemm_case(M, N, K, mode, seed):
    rng = np.random.default_rng(seed)
    lo, hi = (-128, 128) if mode == "int8" else (-8, 8)
    q = rng.integers(lo, hi, size=(M, K)).astype(np.int8)
    t = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    return q, ref.pack(t), rng.uniform(0.1, 10.0, size=M).astype(np.float32), np.array([0.0173], np.float32)


@pytest.mark.parametrize("tile", [256, 224, 192, 128, 64])
def test_gemm_forced_token_tiles(tile):
    # Every token-tile configuration of the tcgen05 kernel, forced, on: several rounds of
    # tiles per SM with ragged tokens and weight rows (bulk-store epilogue); N % 4 != 0 and
    # M < 32 (direct-store epilogue).  Accumulators and outputs must be exact.
    cases = [(10 * tile + 37, 1988, 128), (77, 130, 384), (20, 256, 256)]
    try:
        tb.bitnet_gemm_force_token_tile(tile)
        for i, (M, N, K) in enumerate(cases):
            assert tb.bitnet_gemm_token_tile(M, N, K) == tile
            mode = ("int8", "int4")[i % 2]
            q, packed, scale, alpha = _gemm_case(M, N, K, mode, seed=tile * 10 + i)
            acc = torch.empty((M, N), dtype=torch.int32, device=DEV)
            out = tb.bitnet_ternary_gemm(dev(q), dev(scale), mode, dev(packed), dev(alpha), N, acc_out=acc)
            out2 = tb.bitnet_ternary_gemm(dev(q), dev(scale), mode, dev(packed), dev(alpha), N)
            acc_ref = ref.gemm_packed(q, packed, N)
            np.testing.assert_array_equal(host(acc), acc_ref, err_msg=f"tile {tile} {M}x{N}x{K}")
            out_ref = ref.dequant(acc_ref, scale, alpha[0], MODES[mode])
            np.testing.assert_array_equal(host(out), out_ref)
            np.testing.assert_array_equal(host(out2), out_ref)
        assert tb.bitnet_get_last_device_status() == 0
    finally:
        tb.bitnet_gemm_force_token_tile(0)


DECODE_SHAPES = [
    (1, 11008, 4096),    # many weight rows
    (3, 4096, 16384),    # a long row: many chunks per warp
    (5, 700, 2944),      # K % 256 == 128: a half chunk at the end; ragged rows
    (16, 2000, 384),     # two token groups of 8
    (9, 37, 128),        # fewer weight rows than one CTA's, the last block ragged
    (2, 6912, 2560), (8, 2560, 6912),
]


@pytest.mark.parametrize("M,N,K", DECODE_SHAPES)
def test_gemv_decode_kernel_shapes(M, N, K):
    # the decode kernel on long and short rows, many weight rows, a half chunk at the
    # end of K and ragged tails; exact accumulators, fp32 and bf16 outputs
    mode = ("int8", "int4")[M % 2]
    q, packed, scale, alpha = _gemm_case(M, N, K, mode, seed=M * 7 + N + K)
    acc = torch.empty((M, N), dtype=torch.int32, device=DEV)
    out = tb.bitnet_ternary_gemm(dev(q), dev(scale), mode, dev(packed), dev(alpha), N, acc_out=acc)
    outh = tb.bitnet_ternary_gemm_ex(dev(q), dev(scale), mode, dev(packed), dev(alpha), N, out_dtype=torch.bfloat16)
    acc_ref = ref.gemm_packed(q, packed, N)
    np.testing.assert_array_equal(host(acc), acc_ref, err_msg=f"{M}x{N}x{K}")
    out_ref = ref.dequant(acc_ref, scale, alpha[0], MODES[mode])
    np.testing.assert_array_equal(host(out), out_ref)
    np.testing.assert_array_equal(parity.bf16_bits(outh), ref.round_bf16(out_ref))


# ----------------------------------------------------------------------------- TL2 format
@pytest.mark.parametrize("N,K", [(256, 256), (300, 384), (6912, 2560), (2560, 6912), (37, 128)])
def test_pack_tl2_matches_oracle(N, K):
    # the 2-bit -> TL2 conversion gives the oracle's bytes for the same ternary codes
    W = synthetic.gaussian((N, K), 0.02, synthetic.generator(N + K))
    packed, alpha = tb.bitnet_pack_ternary(W.to(DEV))
    tl2 = tb.bitnet_pack_tl2(packed, K)
    p_ref, a_ref, t_ref = ref.pack_weights(W.numpy())
    np.testing.assert_array_equal(host(packed), p_ref)
    np.testing.assert_array_equal(host(tl2), ref.pack_tl2(t_ref))
    assert tl2.numel() * 8 / (N * K) == pytest.approx(20 * 8 * math.ceil(K / 96) / K)


TL2_SHAPES = [(1, 64, 128), (3, 100, 384), (8, 6912, 2560), (8, 2560, 6912), (16, 512, 1024), (13, 37, 2944),
              (5, 4096, 16384)]


@pytest.mark.parametrize("M,N,K", TL2_SHAPES)
@pytest.mark.parametrize("mode", ["int8", "int4"])
def test_gemm_tl2_exact_accumulators(M, N, K, mode):
    # the TL2 decode kernel: exact int32 sums (oracle reading the TL2 bytes, and the same
    # sums as the 2-bit format), outputs from the same epilogue
    q, packed, scale, alpha = _gemm_case(M, N, K, mode, seed=M * 7 + N + K + 5)
    tl2 = tb.bitnet_pack_tl2(dev(packed), K)
    acc = torch.empty((M, N), dtype=torch.int32, device=DEV)
    out = tb.bitnet_ternary_gemm_tl2(dev(q), dev(scale), mode, tl2, dev(alpha), N, acc_out=acc)
    acc_ref = ref.gemm_tl2(q, host(tl2), N)
    np.testing.assert_array_equal(acc_ref, ref.gemm_packed(q, packed, N))
    np.testing.assert_array_equal(host(acc), acc_ref, err_msg=f"{M}x{N}x{K}")
    np.testing.assert_array_equal(host(out), ref.dequant(acc_ref, scale, alpha[0], MODES[mode]))


@pytest.mark.parametrize("M,NK,fwht,mode", [(1, (6912, 2560), False, "int8"), (8, (2560, 6912), False, "int8"),
                                            (4, (4096, 4096), True, "int4"), (16, (1000, 1024), True, "int8")])
def test_forward_tl2_equals_the_2bit_forward(M, NK, fwht, mode):
    # the same weights in either format give bit-identical forwards, and the forward
    # matches the oracle end to end
    N, K = NK
    case = synthetic.make_case("tl2_fwd", M, K, N, x_kind="student_t3", outliers=max(1, K // 100), outlier_gain=50.0,
                               fwht=fwht, mode=mode, seed=M + N)
    Xd = case.X.to(DEV)
    packed, alpha = tb.bitnet_pack_ternary(case.W.to(DEV))
    tl2 = tb.bitnet_pack_tl2(packed, K)
    ws = torch.empty((tb.bitnet_forward_workspace_bytes(M, K),), dtype=torch.uint8, device=DEV)
    out_tl2 = tb.bitnet_hbitlinear_forward_tl2(Xd, tl2, alpha, N, fwht=fwht, mode=mode, ws=ws)
    gcodes, gs = (host(a) for a in ws_codes_scales(ws, M, K))
    out_2bit = tb.bitnet_hbitlinear_forward(Xd, packed, alpha, N, fwht=fwht, mode=mode)
    torch.cuda.synchronize()
    assert torch.equal(out_tl2, out_2bit)
    X32 = case.X.numpy()
    p_ref, a_ref, _ = ref.pack_weights(case.W.numpy())
    m = MODES[mode]
    r = ref.hbitlinear_forward(X32, p_ref, a_ref, N, fwht_on=fwht, mode=m)
    parity.check_codes(gcodes, r.codes, ref.shadow(X32, None, 1e-5, fwht, m), "tl2 forward")
    parity.check_out_same_codes(host(out_tl2), ref.dequant(ref.gemm_tl2(gcodes, ref.pack_tl2(ref.unpack(p_ref, N, K)),
                                                                        N), gs, a_ref, m), "tl2 forward")
    parity.check_out_end_to_end(host(out_tl2), r.out, gcodes, r.codes, r.scale_x, a_ref, m, "tl2 forward")


def test_gemm_extreme_codes():
    # every code at the int8 extremes, every weight +1/-1: |acc| = 128 K is the largest possible
    for M, N, K in [(4, 64, 16384), (32, 256, 16384)]:
        q = np.full((M, K), -128, np.int8)
        q[::2] = 127
        t = np.ones((N, K), np.int8)
        t[1::3] = -1
        packed = ref.pack(t)
        scale = np.ones(M, np.float32)
        alpha = np.ones(1, np.float32)
        acc = torch.empty((M, N), dtype=torch.int32, device=DEV)
        tb.bitnet_ternary_gemm(dev(q), dev(scale), "int8", dev(packed), dev(alpha), N, acc_out=acc)
        np.testing.assert_array_equal(host(acc), ref.gemm_packed(q, packed, N))


# ----------------------------------------------------------------------------- bf16 output
BF16_GEMM_SHAPES = [
    (1, 64, 128), (5, 700, 2560), (8, 6912, 2560), (16, 512, 1024),           # decode kernel
    (17, 256, 128), (130, 300, 384), (300, 1000, 2048), (2048, 2560, 256),    # tcgen05, bulk-store epilogue
    (77, 130, 384), (64, 1990, 256), (1051, 4100, 256),                      # N % 8 != 0: direct stores
]


@pytest.mark.parametrize("M,N,K", BF16_GEMM_SHAPES)
@pytest.mark.parametrize("mode", ["int8", "int4"])
def test_gemm_bf16_output_exact(M, N, K, mode):
    # the bf16 output is the oracle's fp32 epilogue value rounded once, bit for bit
    q, packed, scale, alpha = _gemm_case(M, N, K, mode, seed=M * 31 + N + K)
    acc = torch.empty((M, N), dtype=torch.int32, device=DEV)
    out = tb.bitnet_ternary_gemm_ex(dev(q), dev(scale), mode, dev(packed), dev(alpha), N, out_dtype=torch.bfloat16,
                                    acc_out=acc)
    assert out.dtype == torch.bfloat16
    acc_ref = ref.gemm_packed(q, packed, N)
    np.testing.assert_array_equal(host(acc), acc_ref)
    want = ref.round_bf16(ref.dequant(acc_ref, scale, alpha[0], MODES[mode]))
    np.testing.assert_array_equal(parity.bf16_bits(out), want, err_msg=f"{M}x{N}x{K} {mode}")
    # the fp32 choice of the same entry point is the plain GEMM
    out32 = tb.bitnet_ternary_gemm_ex(dev(q), dev(scale), mode, dev(packed), dev(alpha), N, out_dtype=torch.float32)
    np.testing.assert_array_equal(host(out32), ref.dequant(acc_ref, scale, alpha[0], MODES[mode]))


@pytest.mark.parametrize("tile", [256, 224, 192, 128, 64])
def test_gemm_bf16_output_forced_tiles(tile):
    try:
        tb.bitnet_gemm_force_token_tile(tile)
        for i, (M, N, K) in enumerate([(6 * tile + 45, 1032, 256), (40, 136, 128)]):
            mode = ("int4", "int8")[i]
            q, packed, scale, alpha = _gemm_case(M, N, K, mode, seed=tile + i)
            out = tb.bitnet_ternary_gemm_ex(dev(q), dev(scale), mode, dev(packed), dev(alpha), N)
            want = ref.round_bf16(ref.dequant(ref.gemm_packed(q, packed, N), scale, alpha[0], MODES[mode]))
            np.testing.assert_array_equal(parity.bf16_bits(out), want, err_msg=f"tile {tile} {M}x{N}x{K}")
    finally:
        tb.bitnet_gemm_force_token_tile(0)


def _forward_case_bf16(case, sample_rows=None):
    Xd = case.X.to(DEV)
    packed, alpha = tb.bitnet_pack_ternary(case.W.to(DEV), eps=case.eps)
    out = tb.bitnet_hbitlinear_forward_ex(Xd, packed, alpha, case.N, eps=case.eps, fwht=case.fwht, mode=case.mode,
                                          out_dtype=torch.bfloat16)
    codes, gscale = tb.bitnet_act_quant(Xd, eps=case.eps, fwht=case.fwht, mode=case.mode)
    torch.cuda.synchronize()
    rows = np.arange(case.M) if sample_rows is None else sample_rows
    X32 = case.X.float().numpy()[rows]
    p_ref, a_ref, _ = ref.pack_weights(case.W.numpy(), eps=case.eps)
    np.testing.assert_array_equal(host(packed), p_ref)
    mode = MODES[case.mode]
    r = ref.hbitlinear_forward(X32, p_ref, a_ref, case.N, eps=case.eps, fwht_on=case.fwht, mode=mode)
    sh = ref.shadow(X32, None, case.eps, case.fwht, mode)
    gcodes = host(codes)[rows]
    parity.check_codes(gcodes, r.codes, sh, case.name)
    gs = host(gscale)[rows]
    parity.check_scale_bound(gs, r.scale_x, case.K, mode, case.name)
    gbits = parity.bf16_bits(out)[rows]
    # same codes and scales -> the same fp32 value, rounded once to the same bf16
    want = ref.round_bf16(ref.dequant(ref.gemm_packed(gcodes, p_ref, case.N), gs, a_ref, mode))
    np.testing.assert_array_equal(gbits, want, err_msg=case.name)
    parity.check_out_end_to_end_bf16(gbits, r.out, gcodes, r.codes, r.scale_x, a_ref, mode, case.name)


@pytest.mark.parametrize("M,K,N,mode,fwht,xdt", [
    (1, 2560, 6912, "int8", False, "f32"),    # decode kernel
    (8, 6912, 2560, "int8", False, "f32"),
    (100, 1024, 300, "int4", True, "f32"),    # tcgen05, N % 8 != 0
    (257, 2048, 520, "int8", False, "bf16"),  # bulk-store epilogue
    (64, 16384, 4096, "int4", True, "f32"),   # a shape the fp32 forward splits over K; bf16 never splits
])
def test_forward_bf16_output(M, K, N, mode, fwht, xdt):
    case = synthetic.make_case("bf16out", M, K, N, x_kind="student_t3", outliers=max(1, K // 100),
                               outlier_gain=50.0, x_dtype=xdt, fwht=fwht, mode=mode, seed=M + K + N)
    _forward_case_bf16(case, None if M <= 300 else _sample(M, 24))


def test_forward_bf16_output_prefill_sampled():
    case = synthetic.prefill_int8(M=4096, K=4096, N=4096, fwht=True)
    _forward_case_bf16(case, _sample(case.M, 16))


# ----------------------------------------------------------------------------- whole forward
def _align256(v):
    return (v + 255) // 256 * 256


def ws_codes_scales(ws, M, K):
    """The codes [M, K] and per-token scales [M] a forward left in its workspace."""
    codes = ws[:M * K].view(torch.int8).view(M, K)
    off = _align256(M * K)
    scales = ws[off:off + 4 * M].view(torch.float32)
    return codes, scales


def _forward_case(case, sample_rows=None):
    Xd = case.X.to(DEV)
    W = case.W.to(DEV)
    packed, alpha = tb.bitnet_pack_ternary(W, eps=case.eps)
    ws = torch.empty((tb.bitnet_forward_workspace_bytes(case.M, case.K),), dtype=torch.uint8, device=DEV)
    out = tb.bitnet_hbitlinear_forward(Xd, packed, alpha, case.N, eps=case.eps, fwht=case.fwht, mode=case.mode,
                                       ws=ws)
    fcodes, fscale = ws_codes_scales(ws, case.M, case.K)  # what the forward used
    codes, gscale = tb.bitnet_act_quant(Xd, eps=case.eps, fwht=case.fwht, mode=case.mode)
    torch.cuda.synchronize()
    rows = np.arange(case.M) if sample_rows is None else sample_rows
    X32 = case.X.float().numpy()[rows]
    p_ref, a_ref, _ = ref.pack_weights(case.W.numpy(), eps=case.eps)
    assert host(alpha)[0] == a_ref
    np.testing.assert_array_equal(host(packed), p_ref)
    mode = MODES[case.mode]
    r = ref.hbitlinear_forward(X32, p_ref, a_ref, case.N, eps=case.eps, fwht_on=case.fwht, mode=mode)
    sh = ref.shadow(X32, None, case.eps, case.fwht, mode)
    gout = host(out)[rows]
    # the standalone activation step and the forward's own codes and scales (the decode
    # kernel may quantise inside itself), each against the oracle
    for label, cc, ss in (("act_quant", codes, gscale), ("forward", fcodes, fscale)):
        gcodes = host(cc)[rows]
        gs = host(ss)[rows]
        parity.check_codes(gcodes, r.codes, sh, f"{case.name} {label}")
        parity.check_scale_bound(gs, r.scale_x, case.K, mode, f"{case.name} {label}")
    gcodes, gs = host(fcodes)[rows], host(fscale)[rows]
    # same codes and scales -> identical output (exact accumulators, same IEEE steps)
    out_same = ref.dequant(ref.gemm_packed(gcodes, p_ref, case.N), gs, a_ref, mode)
    parity.check_out_same_codes(gout, out_same, case.name)
    parity.check_out_end_to_end(gout, r.out, gcodes, r.codes, r.scale_x, a_ref, mode, case.name)


def test_forward_tiny_int8_fwht():
    _forward_case(synthetic.tiny_hbitlinear())


@pytest.mark.parametrize("M", [1, 4, 8])
@pytest.mark.parametrize("NK", [(6912, 2560), (2560, 6912)])
def test_forward_decode_full_size(M, NK):
    _forward_case(synthetic.decode(M, N=NK[0], K=NK[1]))


@pytest.mark.parametrize("M,K,N,mode,fwht,xdt", [
    (3, 1024, 200, "int4", True, "f32"),
    (13, 512, 520, "int8", True, "bf16"),
    (100, 1024, 300, "int4", True, "f32"),
    (257, 2048, 520, "int8", False, "bf16"),
    (384, 4096, 768, "int4", True, "f32"),
])
def test_forward_ragged(M, K, N, mode, fwht, xdt):
    case = synthetic.make_case("ragged", M, K, N, x_kind="student_t3", outliers=max(1, K // 100),
                               outlier_gain=50.0, x_dtype=xdt, fwht=fwht, mode=mode, seed=M + K)
    _forward_case(case)


def _split_k_case(M, K, N, mode, fwht, seed):
    case = synthetic.make_case("splitk", M, K, N, x_kind="student_t3", outliers=max(1, K // 100), outlier_gain=50.0,
                               x_dtype="f32", fwht=fwht, mode=mode, seed=seed)
    _forward_case(case, None if M < 200 else _sample(M, 24))  # against the oracle
    # bit-identical to the unsplit GEMM on the same codes
    Xd = case.X.to(DEV)
    packed, alpha = tb.bitnet_pack_ternary(case.W.to(DEV), eps=case.eps)
    out = tb.bitnet_hbitlinear_forward(Xd, packed, alpha, N, eps=case.eps, fwht=fwht, mode=mode)
    codes, scale = tb.bitnet_act_quant(Xd, eps=case.eps, fwht=fwht, mode=mode)
    out_unsplit = tb.bitnet_ternary_gemm(codes, scale, mode, packed, alpha, N)
    assert torch.equal(out, out_unsplit)
    # the standalone GEMM given a workspace splits K the same way, to the same result
    gws = torch.empty((tb.bitnet_gemm_workspace_bytes(M, N, K),), dtype=torch.uint8, device=DEV)
    out_split = tb.bitnet_ternary_gemm(codes, scale, mode, packed, alpha, N, ws=gws)
    out_split2 = tb.bitnet_ternary_gemm(codes, scale, mode, packed, alpha, N, ws=gws)  # counters left clean
    assert torch.equal(out_split, out_unsplit) and torch.equal(out_split2, out_unsplit)
    assert tb.bitnet_get_last_device_status() == 0


@pytest.mark.parametrize("M,K,N,mode,fwht,splits", [
    (40, 16384, 1000, "int8", False, 8),  # ragged tokens and weight rows
    (33, 8192, 4096, "int4", True, 2),
    (64, 16384, 2048, "int8", False, 8),
    (128, 8192, 2048, "int4", True, 2),
    (200, 8192, 1000, "int8", False, 2),   # pair split: ragged tokens and weight rows
    (300, 8192, 998, "int4", True, 2),     # pair split, N % 4 != 0 (direct stores)
    (260, 16384, 2000, "int4", True, 2),   # pair split, 128-token tiles
])
def test_forward_split_k(M, K, N, mode, fwht, splits):
    # few output tiles for the SMs: the forward splits K.  Two halves: the first parks
    # its int32 sums in the tile's output rows and the second adds them; more splits
    # add int32 partial sums into a zeroed output with atomics.
    assert tb.bitnet_forward_gemm_plan(M, N, K)[1] == splits
    _split_k_case(M, K, N, mode, fwht, seed=M * 7 + K)


@pytest.mark.parametrize("splits", [2, 4, 8])
def test_forward_forced_k_splits(splits):
    # every split protocol on the M = 512 sweep shape, whose automatic plan does not
    # split (whole 256-token chunks for the pair split), bit-identical to the unsplit GEMM
    try:
        tb.bitnet_gemm_force_k_splits(splits)
        assert tb.bitnet_forward_gemm_plan(512, 4096, 16384)[1] == splits
        _split_k_case(512, 16384, 4096, "int4", True, seed=splits)
    finally:
        tb.bitnet_gemm_force_k_splits(0)


@pytest.mark.parametrize("tile", [256, 224, 192, 128, 64])
def test_forward_split_k_forced_tiles(tile):
    try:
        tb.bitnet_gemm_force_token_tile(tile)
        M, K, N = 40, 16384, 1024
        t, sp = tb.bitnet_forward_gemm_plan(M, N, K)
        assert t == tile and sp > 1
        _split_k_case(M, K, N, ("int8", "int4")[tile % 3 == 0], tile % 2 == 0, seed=tile)
    finally:
        tb.bitnet_gemm_force_token_tile(0)


def _swiglu_case(M, K, N, mode, fwht, xdt, seed, sample_rows=None):
    gen = torch.Generator().manual_seed(seed)
    gate = torch.randn(M, K, generator=gen) * 2.0
    up = torch.randn(M, K, generator=gen)
    W = torch.randn(N, K, generator=gen) * 0.02
    if xdt == "bf16":
        gate, up = gate.to(torch.bfloat16), up.to(torch.bfloat16)
    gd, ud = gate.to(DEV), up.to(DEV)
    packed, alpha = tb.bitnet_pack_ternary(W.to(DEV))
    ws = torch.empty((tb.bitnet_forward_workspace_bytes(M, K),), dtype=torch.uint8, device=DEV)
    out = tb.bitnet_hbitlinear_forward_swiglu(gd, ud, packed, alpha, N, fwht=fwht, mode=mode, ws=ws)
    fcodes, fscale = ws_codes_scales(ws, M, K)  # what the forward used
    codes, gscale = tb.bitnet_act_quant_swiglu(gd, ud, fwht=fwht, mode=mode)
    torch.cuda.synchronize()
    rows = np.arange(M) if sample_rows is None else sample_rows
    g32, u32 = gate.float().numpy()[rows], up.float().numpy()[rows]
    p_ref, a_ref, _ = ref.pack_weights(W.numpy())
    m = MODES[mode]
    r = ref.hbitlinear_forward(ref.swiglu(g32, u32), p_ref, a_ref, N, fwht_on=fwht, mode=m)
    sh = ref.shadow_swiglu(g32, u32, eps=1e-5, fwht_on=fwht, mode=m)
    label = f"swiglu M={M} K={K} N={N} {mode} fwht={fwht} {xdt}"
    parity.check_codes(host(codes)[rows], r.codes, sh, label + " act_quant")
    parity.check_scale_bound(host(gscale)[rows], r.scale_x, K, m, label + " act_quant")
    gcodes, gs, gout = host(fcodes)[rows], host(fscale)[rows], host(out)[rows]
    parity.check_codes(gcodes, r.codes, sh, label)
    parity.check_scale_bound(gs, r.scale_x, K, m, label)
    parity.check_out_same_codes(gout, ref.dequant(ref.gemm_packed(gcodes, p_ref, N), gs, a_ref, m), label)
    parity.check_out_end_to_end(gout, r.out, gcodes, r.codes, r.scale_x, a_ref, m, label)
    assert tb.bitnet_get_last_device_status() == 0


@pytest.mark.parametrize("M,K,N,mode,fwht,xdt", [
    (1, 2048, 512, "int4", True, "f32"),     # decode kernel
    (8, 8192, 2048, "int4", True, "f32"),    # decode kernel, Wdown-like
    (13, 1024, 700, "int8", False, "bf16"),  # decode kernel, ragged N, plain quantiser
    (300, 4096, 1000, "int4", True, "f32"),  # tcgen05 kernel, ragged
    (129, 2048, 640, "int8", True, "bf16"),
    (400, 2048, 512, "int8", True, "bf16"),  # many tokens: the per-token FWHT kernel on the SwiGLU product
    (300, 16384, 256, "int4", True, "f32"),
])
def test_forward_swiglu(M, K, N, mode, fwht, xdt):
    # silu(gate) * up formed inside the activation kernel (BitNetV2FFN.forward's down projection)
    _swiglu_case(M, K, N, mode, fwht, xdt, seed=M * 31 + K)


def test_forward_swiglu_wdown_full_size_sampled():
    # the Wdown-style shape: intermediate 8192 -> 2048, int4 + FWHT, 2048 tokens
    _swiglu_case(2048, 8192, 2048, "int4", True, "f32", seed=3, sample_rows=_sample(2048, 24))


# ----------------------------------------------------------------------------- low-bit KV cache
@pytest.mark.parametrize("B,H,S,D,bits,xdt", [
    (1, 2, 9, 128, 4, "f32"),
    (2, 3, 17, 64, 3, "f32"),
    (1, 4, 33, 256, 8, "bf16"),
    (1, 1, 1, 128, 4, "f32"),     # the BOS token alone
    (2, 2, 5, 100, 4, "f32"),     # D not a multiple of 32
    (1, 1, 7, 1024, 3, "bf16"),
    (1, 2, 3, 4, 4, "f32"),       # D = 4
    (2, 3, 3, 32, 4, "bf16"),     # eight lanes per row, BOS rows beside absmean rows in one warp
    (3, 5, 70, 192, 3, "f32"),    # sixteen lanes per row, ragged last warp
])
def test_kv_quant(B, H, S, D, bits, xdt):
    gen = torch.Generator().manual_seed(B * 100 + S * 7 + D)
    kv = synthetic.student_t3((B, H, S, D), gen)
    kv[..., :: max(1, D // 8)] *= 6.0  # a few large channels, as post-RoPE keys have
    if xdt == "bf16":
        kv = kv.to(torch.bfloat16)
    codes, step, deq = tb.bitnet_kv_quant(kv.to(DEV), bits=bits, dequant=True)
    codes2, step2, none = tb.bitnet_kv_quant(kv.to(DEV), bits=bits)
    torch.cuda.synchronize()
    assert none is None
    gc, gs, gd = host(codes), host(step), host(deq)
    np.testing.assert_array_equal(host(codes2), gc)
    np.testing.assert_array_equal(host(step2), gs)
    x32 = kv.float().numpy()
    oc, os_, _ = ref.kv_quant(x32, bits)
    sh = ref.shadow_kv(x32, bits)
    label = f"kv B={B} H={H} S={S} D={D} bits={bits} {xdt}"
    # the 8- and 3-bit rows (and every BOS row) use an exact max: identical codes and steps
    exact_rows = np.ones(x32.shape[:-1], bool) if bits != 4 else (np.arange(S) == 0)[None, None, :].repeat(B, 0).repeat(H, 1)
    np.testing.assert_array_equal(gc[exact_rows], oc[exact_rows], err_msg=label)
    np.testing.assert_array_equal(gs[exact_rows], os_[exact_rows], err_msg=label)
    if bits == 4 and S > 1:
        parity.check_codes(gc[:, :, 1:], oc[:, :, 1:], sh[:, :, 1:], label)
        rel = np.abs(gs[:, :, 1:].astype(np.float64) - os_[:, :, 1:]) / os_[:, :, 1:]
        assert rel.max() <= (D + 32 + 8) * 2.0 ** -24 + 4 * 2.0 ** -24, label  # sum order only
    # the dequantised values are step * code, one rounding
    np.testing.assert_array_equal(gd, gs[..., None] * gc.astype(np.float32))
    assert tb.bitnet_get_last_device_status() == 0


def _sample(M, n=32, seed=0):
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, n - 2, replace=False)]))
    return rows


def test_forward_wdown_int4_full_size_sampled():
    case = synthetic.wdown_int4()  # M=2048, K=8192, N=2048, Student-t + 1% outliers x50
    _forward_case(case, _sample(case.M))


@pytest.mark.parametrize("N,fwht", [(4096, True), (11008, False)])
def test_forward_prefill_bf16_full_size_sampled(N, fwht):
    case = synthetic.prefill_int8(M=4096, K=4096, N=N, fwht=fwht)
    _forward_case(case, _sample(case.M, 24))


@pytest.mark.parametrize("M,K", [(1, 16384), (8, 4096), (64, 16384), (512, 4096), (8192, 16384)])
def test_forward_msweep_int4_sampled(M, K):
    case = synthetic.msweep_int4(M, K)
    _forward_case(case, None if M <= 64 else _sample(M, 16))


# ----------------------------------------------------------------------------- properties
def test_forward_deterministic_and_graph_capturable():
    case = synthetic.msweep_int4(64, 4096, N=1024, seed=3)
    Xd = case.X.to(DEV)
    layer = tb.HBitLinear(case.W.to(DEV), mode="int4", fwht=True)
    o1 = layer(Xd).clone()
    o2 = layer(Xd).clone()
    assert torch.equal(o1, o2)
    out = torch.empty_like(o1)
    layer.workspace(Xd.shape[0], Xd.device)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        layer(Xd, out=out)  # warm (attribute caches) outside capture
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer(Xd, out=out)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, o1)


@pytest.mark.parametrize("M,fwht,mode", [(4, False, "int8"), (300, True, "int4"), (1, True, "int8")])
def test_forward_chain_reads_the_previous_layers_output(M, fwht, mode):
    # Three layers back to back on one stream, each reading the output the kernel just
    # before it wrote (the GEMV/GEMM of the previous layer): the activation kernel may
    # launch early and prefetch its input into L2, but reads it only after the
    # dependency wait.  Each layer is checked against the oracle on the GPU's own input.
    K = 1024
    gen = synthetic.generator(M + 7)
    X = synthetic.student_t3((M, K), gen)
    Ws = [synthetic.gaussian((K, K), 0.02, gen) for _ in range(3)]
    layers = [tb.HBitLinear(W.to(DEV), mode=mode, fwht=fwht) for W in Ws]
    xs = [X.to(DEV)]
    for layer in layers:
        xs.append(layer(xs[-1]))
    torch.cuda.synchronize()
    for i, W in enumerate(Ws):
        xin = host(xs[i]).astype(np.float32)
        p_ref, a_ref, _ = ref.pack_weights(W.numpy(), eps=1e-5)
        r = ref.hbitlinear_forward(xin, p_ref, a_ref, K, eps=1e-5, fwht_on=fwht, mode=MODES[mode])
        # the codes and scales this layer's forward used, left in its workspace
        codes, gs = ws_codes_scales(layers[i].workspace(M, xs[i].device), M, K)
        gcodes = host(codes)
        sh = ref.shadow(xin, None, 1e-5, fwht, MODES[mode])
        label = f"chain layer {i} M={M}"
        parity.check_codes(gcodes, r.codes, sh, label)
        same = ref.dequant(ref.gemm_packed(gcodes, p_ref, K), host(gs), a_ref, MODES[mode])
        parity.check_out_same_codes(host(xs[i + 1]), same, label)


def _guarded(n, dtype, poison, pad):
    """A flat buffer of pad + n + pad elements filled with `poison`; returns it and the
    middle n elements (16-byte aligned when pad is a multiple of 16 bytes)."""
    big = torch.full((pad + n + pad,), poison, dtype=dtype, device=DEV)
    return big, big[pad:pad + n]


@pytest.mark.parametrize("M,K,N,mode,fwht,out_dt", [
    (5, 2560, 700, "int8", False, torch.float32),    # decode kernel, ragged N
    (77, 384, 130, "int4", False, torch.float32),    # GEMM, direct stores (M < 32 tokens per box)
    (300, 8192, 998, "int4", True, torch.float32),   # pair split, N % 4 != 0
    (200, 8192, 1000, "int8", False, torch.float32), # pair split, ragged tiles
    (40, 16384, 1000, "int8", False, torch.float32), # atomic split, ragged
    (2000, 384, 2600, "int8", False, torch.float32), # GEMM, bulk-store epilogue
    (64, 256, 1990, "int4", False, torch.bfloat16),  # bf16 output, N % 8 != 0
    (130, 1024, 2048, "int8", True, torch.bfloat16), # bf16 output, bulk-store epilogue
])
def test_writes_stay_inside_the_output_and_workspace(M, K, N, mode, fwht, out_dt):
    # guard bands around the output and the workspace: every byte outside them must
    # keep its poison after the forward
    gen = synthetic.generator(M + N)
    X = synthetic.student_t3((M, K), gen).to(DEV)
    W = synthetic.gaussian((N, K), 0.02, gen).to(DEV)
    packed, alpha = tb.bitnet_pack_ternary(W)
    pad = 4096  # elements of the output: 8 or 16 KB, 16-byte aligned either way
    poison = -7777.0
    obig, out_flat = _guarded(M * N, out_dt, poison, pad)
    out = out_flat.view(M, N)
    nbytes = tb.bitnet_forward_workspace_bytes(M, K)
    wpad = 4096  # bytes, a multiple of 256
    wbig, ws = _guarded(nbytes, torch.uint8, 0xA5, wpad)
    if out_dt == torch.float32:
        tb.bitnet_hbitlinear_forward(X, packed, alpha, N, fwht=fwht, mode=mode, out=out, ws=ws)
    else:
        tb.bitnet_hbitlinear_forward_ex(X, packed, alpha, N, fwht=fwht, mode=mode, out_dtype=out_dt, out=out, ws=ws)
    torch.cuda.synchronize()
    assert tb.bitnet_get_last_device_status() == 0
    ob = obig.float().cpu()
    stored = torch.full((1,), poison, dtype=out_dt).float().item()  # the poison as the dtype holds it
    assert bool((ob[:pad] == stored).all()) and bool((ob[pad + M * N:] == stored).all()), "write outside the output"
    assert bool(torch.isfinite(ob[pad:pad + M * N]).all())
    wb = wbig.cpu()
    assert bool((wb[:wpad] == 0xA5).all()) and bool((wb[wpad + nbytes:] == 0xA5).all()), "write outside the workspace"
    # and the result is the unguarded forward's
    ref_out = (tb.bitnet_hbitlinear_forward(X, packed, alpha, N, fwht=fwht, mode=mode) if out_dt == torch.float32 else
               tb.bitnet_hbitlinear_forward_ex(X, packed, alpha, N, fwht=fwht, mode=mode, out_dtype=out_dt))
    assert torch.equal(out, ref_out)


def test_empty_batch_and_errors():
    W = synthetic.gaussian((64, 256), 0.02, synthetic.generator(1)).to(DEV)
    packed, alpha = tb.bitnet_pack_ternary(W)
    X = torch.empty((0, 256), device=DEV)
    out = tb.bitnet_hbitlinear_forward(X, packed, alpha, 64)
    assert out.shape == (0, 64)
    with pytest.raises(tb.BitnetError) as e:
        tb.bitnet_act_quant(torch.ones((2, 2560), device=DEV), fwht=True)
    assert e.value.status == 3
    with pytest.raises(tb.BitnetError):
        tb.bitnet_act_quant(torch.ones((2, 200), device=DEV), fwht=False)


def test_timeout_path_reports_and_recovers():
    tb.bitnet_selftest_wait_timeout(2000)
    assert tb.bitnet_get_last_device_status() == 5
    assert tb.bitnet_get_last_device_status() == 0
    # the context is still usable afterwards
    x = torch.ones((2, 256), device=DEV)
    codes, scale = tb.bitnet_act_quant(x, fwht=True)
    torch.cuda.synchronize()
    assert host(codes)[0, 0] == 127
