"""Pins for the CPU oracle: checks against what the pages and the mathematics fix,
never against a retyped copy of the oracle's own formulas.

  * FWHT: the closed-form Sylvester entries (-1)^popcount(i&j)/sqrt(n), scipy's
    Sylvester Hadamard matrix, H = H^T, H.H = I, H e0 and H 1, Parseval.
  * RMSNorm: constant rows (closed form), gain linearity, scale invariance.
  * Activation quantisation: round-half-even/clip tie tables with exact
    multipliers, the int8 max-code invariant, the int4 code histogram of a
    normal row against its closed-form probabilities.
  * Weights: codes in {-1,0,1}; alpha against numpy's float64 mean; the zero
    fraction of Gaussian weights against 2*Phi(sqrt(2/pi)/2) - 1.
  * Packing: hand-worked byte layouts, round trip.
  * TL2 format: the page's 14 base triplets and their mirrors, hand-worked bytes,
    every triplet round trip, 5/3 bits per weight, GEMM against numpy.
  * GEMM: numpy int64 matmul.
  * Whole path: the hand-worked tiny cases.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg
import torch

from oracle import ref

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _popcount(v):
    return bin(v).count("1")


# ----------------------------------------------------------------------------- FWHT
@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 32, 64])
def test_fwht_matches_closed_form_sylvester(n):
    H = ref.fwht(np.eye(n, dtype=np.float32))  # row j = H e_j = column j of H
    closed = np.array([[(-1.0) ** _popcount(i & j) for j in range(n)] for i in range(n)]) / math.sqrt(n)
    np.testing.assert_allclose(H, closed, rtol=0, atol=4e-7 * max(1, math.log2(n)))
    sy = scipy.linalg.hadamard(n).astype(np.float64) / math.sqrt(n)
    np.testing.assert_allclose(H, sy, rtol=0, atol=4e-7 * max(1, math.log2(n)))


@pytest.mark.parametrize("n", [2, 8, 64])
def test_fwht_symmetric_and_involutive(n):
    H = ref.fwht(np.eye(n, dtype=np.float32)).astype(np.float64)
    np.testing.assert_allclose(H, H.T, atol=1e-7)
    HH = ref.fwht(ref.fwht(np.eye(n, dtype=np.float32))).astype(np.float64)
    np.testing.assert_allclose(HH, np.eye(n), atol=2e-6)
    np.testing.assert_allclose(H @ H, np.eye(n), atol=2e-6)


@pytest.mark.parametrize("n", [256, 4096, 16384])
def test_fwht_basis_and_parseval(n):
    e0 = np.zeros((1, n), np.float32)
    e0[0, 0] = 1
    np.testing.assert_allclose(ref.fwht(e0)[0], np.full(n, 1 / math.sqrt(n)), rtol=2e-6)
    ones = np.ones((1, n), np.float32)
    out = ref.fwht(ones)[0]
    assert abs(out[0] - math.sqrt(n)) < 1e-5 * math.sqrt(n)
    assert np.all(out[1:] == 0)
    rng = np.random.default_rng(1)
    x = rng.standard_normal((3, n)).astype(np.float32)
    y = ref.fwht(x)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-5)


def test_fwht_against_scipy_matrix_large():
    n = 2048
    rng = np.random.default_rng(2)
    x = rng.standard_normal((4, n)).astype(np.float32)
    H = scipy.linalg.hadamard(n).astype(np.float64) / math.sqrt(n)
    exact = x.astype(np.float64) @ H.T
    got = ref.fwht(x).astype(np.float64)
    np.testing.assert_allclose(got, exact, rtol=0, atol=2e-5)


def test_fwht_rejects_non_power_of_two():
    with pytest.raises(ref.OracleError) as e:
        ref.fwht(np.ones((1, 6), np.float32))
    assert e.value.rc == 3
    with pytest.raises(ref.OracleError):
        ref.fwht(np.ones((1, 2560), np.float32))


# ----------------------------------------------------------------------------- RMSNorm
def test_rmsnorm_constant_row_closed_form():
    for c in (1.0, 3.0, 0.001, 250.0):
        x = np.full((1, 64), c, np.float32)
        y = ref.rmsnorm(x, eps=1e-5)[0].astype(np.float64)
        want = c / math.sqrt(c * c + 1e-5)
        np.testing.assert_allclose(y, want, rtol=3e-7)


def test_rmsnorm_zero_row_is_zero():
    y = ref.rmsnorm(np.zeros((2, 128), np.float32), eps=1e-5)
    assert np.all(y == 0)


def test_rmsnorm_unit_mean_square_and_scale_invariance():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((4, 2560)) * 7).astype(np.float32)
    y = ref.rmsnorm(x, eps=0.0).astype(np.float64)
    np.testing.assert_allclose((y * y).mean(axis=1), 1.0, rtol=2e-5)
    y2 = ref.rmsnorm(x * np.float32(4.0), eps=0.0)
    np.testing.assert_array_equal(y2, ref.rmsnorm(x, eps=0.0))  # power-of-two scale is exact


def test_rmsnorm_gain_is_elementwise():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((3, 256)).astype(np.float32)
    g = rng.uniform(0.5, 2.0, 256).astype(np.float32)
    np.testing.assert_array_equal(ref.rmsnorm(x, g), ref.rmsnorm(x) * g)


# ----------------------------------------------------------------------------- activation quant
def test_roundclip_tie_table_int8():
    d = _gold("roundclip_ties.json")["int8"]
    y = np.array([d["y"]], np.float32)
    q, s = ref.act_quant_codes(y, ref.ACT_INT8, eps=d["eps"])
    assert q[0].tolist() == d["codes"]
    assert s[0] == np.float32(d["scale"])


def test_roundclip_tie_table_int4():
    d = _gold("roundclip_ties.json")["int4"]
    y = np.array([d["y"]], np.float32)
    assert hex(int(y[0, 9].view(np.uint32))) == d["y9_bits"]
    q, s = ref.act_quant_codes(y, ref.ACT_INT4, eps=d["eps"])
    assert q[0].tolist() == d["codes"]
    assert s[0] == np.float32(np.sqrt(7.0)) / np.float32(2.0)


def test_int8_max_code_invariant():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((64, 1024)).astype(np.float32)
    for fw in (False, True):
        q, s = ref.act_quant(x, fwht_on=fw, mode=ref.ACT_INT8)
        assert np.all(np.abs(q.astype(np.int32)).max(axis=1) == 127)
        assert q.min() >= -127  # |y*s| <= 127*gamma/(gamma+eps) < 127.5, so -128 never appears


def test_zero_token_gives_zero_codes_and_scale():
    x = np.zeros((2, 256), np.float32)
    for mode in (ref.ACT_INT8, ref.ACT_INT4):
        q, s = ref.act_quant(x, fwht_on=True, mode=mode)
        assert np.all(q == 0) and np.all(s == 0)


def _phi(z):
    return 0.5 * (1 + math.erf(z / math.sqrt(2)))


def test_int4_histogram_matches_normal_closed_form():
    # RMSNorm'd N(0,1) rows: beta -> E|y| = sqrt(2/pi), step delta = beta/sqrt7; code k has mass
    # Phi((k+1/2) delta) - Phi((k-1/2) delta), with the tails folded into 7 and -8.
    rng = np.random.default_rng(6)
    x = rng.standard_normal((64, 16384)).astype(np.float32)
    q, _ = ref.act_quant(x, mode=ref.ACT_INT4)
    n = q.size
    delta = math.sqrt(2 / math.pi) / math.sqrt(7)
    for k in range(-8, 8):
        lo = -math.inf if k == -8 else (k - 0.5) * delta
        hi = math.inf if k == 7 else (k + 0.5) * delta
        p = (_phi(hi) if hi != math.inf else 1.0) - (_phi(lo) if lo != -math.inf else 0.0)
        got = np.count_nonzero(q == k) / n
        sd = math.sqrt(p * (1 - p) / n)
        assert abs(got - p) < 5 * sd + 1.5e-3 * p, (k, got, p)
    assert abs(np.count_nonzero(q == 0) / n - 0.1199) < 2e-3


def test_shadow_agrees_with_fp32_codes_away_from_ties():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((8, 4096)).astype(np.float32)
    for mode in (ref.ACT_INT8, ref.ACT_INT4):
        q, _ = ref.act_quant(x, fwht_on=True, mode=mode)
        v = ref.shadow(x, fwht_on=True, mode=mode)
        lo, hi = (-128, 127) if mode == ref.ACT_INT8 else (-8, 7)
        want = np.clip(np.rint(v), lo, hi)
        frac = np.abs(v - np.floor(v) - 0.5)
        far = frac > 1e-3
        np.testing.assert_array_equal(q[far], want[far])


# ----------------------------------------------------------------------------- weights
def test_ternary_codes_and_alpha():
    rng = np.random.default_rng(8)
    W = (rng.standard_normal((300, 512)) * 0.02).astype(np.float32)
    a = ref.weight_alpha(W)
    assert a == np.float32(np.mean(np.abs(W.astype(np.float64))))
    t = ref.ternarize(W, a)
    assert set(np.unique(t).tolist()) <= {-1, 0, 1}


@pytest.mark.slow
def test_gaussian_weight_zero_fraction_closed_form():
    # P(t = 0) = P(|w| < (alpha+eps)/2) -> 2*Phi(sqrt(2/pi)/2) - 1 = 0.3101 for Gaussian W.
    from ternary_weight_bit_b200 import synthetic
    W = synthetic.decode(1).W.numpy()  # 6912 x 2560 = 17.7 M weights, N(0, 0.02^2)
    _, _, t = ref.pack_weights(W)
    p0 = 2 * _phi(0.5 * math.sqrt(2 / math.pi)) - 1
    assert abs(p0 - 0.3101) < 1e-4
    f0 = np.count_nonzero(t == 0) / t.size
    assert abs(f0 - p0) < 1e-3
    fp = np.count_nonzero(t == 1) / t.size
    assert abs(fp - (1 - p0) / 2) < 1e-3


# ----------------------------------------------------------------------------- packing
def test_pack_layout_golden():
    for case in _gold("pack_layout.json")["cases"]:
        t = np.array([case["t"]], np.int8)
        p = ref.pack(t)
        assert p[0].tolist() == case["bytes"], case["derivation"]
        np.testing.assert_array_equal(ref.unpack(p, 1, t.shape[1]), t)


def test_pack_roundtrip_random():
    rng = np.random.default_rng(9)
    t = rng.integers(-1, 2, size=(37, 256)).astype(np.int8)
    p = ref.pack(t)
    assert p.shape == (37, 64)
    np.testing.assert_array_equal(ref.unpack(p, 37, 256), t)


def test_unpack_flags_invalid_code():
    p = np.full((1, 4), 0xFF, np.uint8)
    with pytest.raises(ref.OracleError):
        ref.unpack(p, 1, 16)


# ----------------------------------------------------------------------------- GEMM
def test_integer_gemm_matches_numpy():
    rng = np.random.default_rng(10)
    q = rng.integers(-128, 128, size=(9, 384)).astype(np.int8)
    t = rng.integers(-1, 2, size=(13, 384)).astype(np.int8)
    want = q.astype(np.int64) @ t.astype(np.int64).T
    np.testing.assert_array_equal(ref.gemm_int(q, t), want)
    np.testing.assert_array_equal(ref.gemm_packed(q, ref.pack(t), 13), want)


def test_integer_gemm_extreme_values():
    K = 16384
    q = np.full((2, K), -128, np.int8)
    q[1] = 127
    t = np.ones((3, K), np.int8)
    t[1] = -1
    t[2, ::2] = 0
    want = q.astype(np.int64) @ t.astype(np.int64).T
    np.testing.assert_array_equal(ref.gemm_packed(q, ref.pack(t), 3), want)


# ----------------------------------------------------------------------------- whole path
@pytest.mark.parametrize("mode_name", ["int8", "int4"])
def test_hand_cases(mode_name):
    g = _gold("hand_cases.json")
    mode = ref.ACT_INT8 if mode_name == "int8" else ref.ACT_INT4
    W = np.array(g["W"], np.float32)
    alpha = ref.weight_alpha(W)
    assert alpha == np.float32(g["alpha"])
    t = ref.ternarize(W, alpha, eps=g["eps"])
    assert t.tolist() == g["t"]
    for case in g["cases"]:
        x = np.array([case["x"]], np.float32)
        y = ref.fwht(ref.rmsnorm(x, eps=g["eps"]))
        np.testing.assert_allclose(y[0], case["Hy"], rtol=2e-6, atol=1e-6)
        q, s = ref.act_quant(x, eps=g["eps"], fwht_on=True, mode=mode)
        acc = ref.gemm_int(q, t)  # K = 4 is below the 16-wide packing granule
        out = ref.dequant(acc, s, alpha, mode)
        exp = case[mode_name]
        assert q[0].tolist() == exp["codes"]
        np.testing.assert_allclose(s[0], exp["scale"], rtol=2e-6)
        assert acc[0].tolist() == exp["acc"]
        np.testing.assert_allclose(out[0], exp["out"], rtol=2e-6, atol=1e-9)


# ----------------------------------------------------------------------------- SwiGLU input
# (bitnet_v2_engine.py page, BitNetV2FFN.forward: silu(gate_proj(x)) * up_proj(x))
def _ulp_rel(a, b):
    return abs(float(a) - float(b)) / max(abs(float(b)), 1e-30)


def test_swiglu_closed_form_values():
    gate = np.array([[0.0, 1.0, -1.0, 2.0, 50.0, -100.0, 20.0]], np.float32)
    up = np.array([[3.0, 1.0, 2.0, 0.5, 2.0, 5.0, 1.0]], np.float32)
    got = ref.swiglu(gate, up)[0]
    assert got[0] == 0.0                                       # silu(0) = 0
    assert _ulp_rel(got[1], 1.0 / (1.0 + math.exp(-1.0))) < 3e-7  # sigmoid(1)
    assert _ulp_rel(got[2], -2.0 / (1.0 + math.e)) < 3e-7      # 2 * silu(-1) = -2 / (1 + e)
    assert _ulp_rel(got[3], 1.0 / (1.0 + math.exp(-2.0))) < 3e-7  # 0.5 * silu(2) = sigmoid(2)
    assert got[4] == 100.0                                     # e^-50 vanishes against 1
    assert got[5] == 0.0 and math.copysign(1.0, got[5]) < 0   # -100 / inf = -0
    assert got[6] == 20.0                                      # sigmoid(20) rounds to 1 in fp32


def test_swiglu_odd_part_is_the_identity():
    # silu(x) - silu(-x) = x (sigmoid(x) + sigmoid(-x) = 1)
    x = np.random.default_rng(5).uniform(-12, 12, size=4000).astype(np.float32)
    ones = np.ones_like(x)
    d = ref.swiglu(x[None], ones[None])[0].astype(np.float64) - ref.swiglu(-x[None], ones[None])[0]
    np.testing.assert_allclose(d, x.astype(np.float64), rtol=2e-6, atol=1e-6)


def test_swiglu_minimum_is_minus_lambert_w_of_inverse_e():
    # min_x x*sigmoid(x) = -W(1/e) at x = -1 - W(1/e) (W: Lambert W, principal branch)
    w = 0.27846454276107380  # W(e^-1), the solution of w e^w = e^-1
    x = np.arange(-3.0, 0.0, 1e-3, dtype=np.float64).astype(np.float32)
    f = ref.swiglu(x[None], np.ones_like(x)[None])[0]
    assert abs(float(f.min()) + w) < 2e-6
    assert abs(float(x[np.argmin(f)]) + 1.0 + w) < 2e-3


def test_swiglu_scales_exactly_with_up():
    g = np.random.default_rng(6).normal(0, 3, size=(4, 64)).astype(np.float32)
    one = ref.swiglu(g, np.ones_like(g))
    for p2 in (0.25, 4.0, -8.0):
        np.testing.assert_array_equal(ref.swiglu(g, np.full_like(g, p2)), one * np.float32(p2))


def test_shadow_swiglu_agrees_with_fp32_codes_away_from_ties():
    rng = np.random.default_rng(7)
    gate = rng.normal(0, 2, size=(6, 512)).astype(np.float32)
    up = rng.normal(0, 1, size=(6, 512)).astype(np.float32)
    for mode in (ref.ACT_INT8, ref.ACT_INT4):
        q, _ = ref.act_quant(ref.swiglu(gate, up), eps=1e-5, fwht_on=True, mode=mode)
        v = ref.shadow_swiglu(gate, up, eps=1e-5, fwht_on=True, mode=mode)
        lo, hi = (-128, 127) if mode == ref.ACT_INT8 else (-8, 7)
        want = np.clip(np.rint(v), lo, hi)
        far = np.abs(v - np.floor(v) - 0.5) > 1e-3
        np.testing.assert_array_equal(q[far], want[far])


# ----------------------------------------------------------------------------- low-bit KV cache
# (bitnet_v2_engine.py page, BitNetV2Attention._quantize_kv_head)
def test_kv_hand_case():
    # one head, two tokens of D = 4: x = [1, -2, 0.5, 3]; computed by hand from the page's formulas
    x = np.array([[[1.0, -2.0, 0.5, 3.0], [1.0, -2.0, 0.5, 3.0]]], np.float32)
    c3, s3, d3 = ref.kv_quant(x, 3)
    c4, s4, _ = ref.kv_quant(x, 4)
    # BOS token: int8 absmax, 127 / (3 + 1e-5) * x -> [42.33, -84.67, 21.17, 127.0]
    assert c3[0, 0].tolist() == [42, -85, 21, 127] == c4[0, 0].tolist()
    assert _ulp_rel(s3[0, 0], (3.0 + 1e-5) / 127.0) < 3e-7
    # 3-bit: 3 / (3 + 1e-5) * x -> [0.99999, -1.99999, 0.499998, 2.99999]
    assert c3[0, 1].tolist() == [1, -2, 0, 3]
    assert _ulp_rel(s3[0, 1], (3.0 + 1e-5) / 3.0) < 3e-7
    np.testing.assert_allclose(d3[0, 1], np.array([1, -2, 0, 3]) * (3.0 + 1e-5) / 3.0, rtol=3e-7)
    # 4-bit absmean: beta = 6.5 / 4 = 1.625, sqrt7 / (1.625 + 1e-5) * x -> [1.63, -3.26, 0.81, 4.88]
    assert c4[0, 1].tolist() == [2, -3, 1, 5]
    assert _ulp_rel(s4[0, 1], (1.625 + 1e-5) / math.sqrt(7.0)) < 3e-7


def test_kv_3bit_tie_table():
    # eps = 0 and gamma = 6: the multiplier 3 / 6 = 0.5 is exact, so 0.5 * x lands on half-integers
    x = np.array([[[6.0, 1.0, 3.0, 5.0, -1.0, -3.0, -5.0, -6.0]] * 2], np.float32)
    codes, step, deq = ref.kv_quant(x, 3, eps=0.0)
    assert codes[0, 1].tolist() == [3, 0, 2, 2, 0, -2, -2, -3]  # round half to even
    assert step[0, 1] == 2.0
    np.testing.assert_array_equal(deq[0, 1], 2.0 * codes[0, 1])


def test_kv_absmax_codes_stay_inside_the_symmetric_range():
    # |x| <= gamma makes |3x / (gamma + eps)| < 3.5 and |127x / (gamma + eps)| < 127.5: -4 and -128 never occur
    kv = np.random.default_rng(11).standard_t(3, size=(4, 2, 64, 128)).astype(np.float32)
    for bits, lim in ((3, 3), (8, 127)):
        codes, _, _ = ref.kv_quant(kv, bits)
        rest = codes[..., 1:, :]  # token 0 is always int8
        assert rest.min() >= -lim and rest.max() <= lim
        assert (np.abs(rest).max(axis=-1) == lim).all()  # the max element reaches the top code
        assert np.abs(codes[..., 0, :]).max() <= 127


def test_kv_reconstruction_within_half_a_step():
    kv = np.random.default_rng(12).normal(size=(2, 3, 17, 64)).astype(np.float32)
    for bits in (3, 8):
        _, step, deq = ref.kv_quant(kv, bits)
        err = np.abs(deq.astype(np.float64) - kv)
        assert (err <= 0.5 * step[..., None] * (1 + 1e-5) + 1e-7).all()


def test_kv_bos_token_is_always_int8():
    kv = np.random.default_rng(13).normal(size=(3, 5, 9, 32)).astype(np.float32)
    c8, s8, _ = ref.kv_quant(kv, 8)
    for bits in (3, 4):
        c, s, _ = ref.kv_quant(kv, bits)
        np.testing.assert_array_equal(c[:, :, 0], c8[:, :, 0])
        np.testing.assert_array_equal(s[:, :, 0], s8[:, :, 0])
        assert np.abs(c[:, :, 1:]).max() <= (3 if bits == 3 else 8)


def test_kv_shadow_agrees_away_from_ties():
    kv = np.random.default_rng(14).normal(size=(2, 4, 33, 64)).astype(np.float32)
    for bits, lo, hi in ((3, -4, 3), (4, -8, 7), (8, -128, 127)):
        codes, _, _ = ref.kv_quant(kv, bits)
        v = ref.shadow_kv(kv, bits)
        lo_b = np.where(np.arange(33)[None, None, :, None] == 0, -128, lo)
        hi_b = np.where(np.arange(33)[None, None, :, None] == 0, 127, hi)
        want = np.clip(np.rint(v), lo_b, hi_b)
        far = np.abs(v - np.floor(v) - 0.5) > 1e-3
        np.testing.assert_array_equal(codes[far], want[far])


# ----------------------------------------------------------------------------- bf16 output
# (the fp32 output rounded once to bf16, to nearest, ties to even)
def _bits(x):
    return np.array([x], np.float32).view(np.uint32)[0]


def _from_bits32(u):
    return np.array([u], np.uint32).view(np.float32)[0]


def _bf16_value(b):
    return np.asarray(b, np.uint32) << 16


def test_bf16_hand_table():
    e = 2.0 ** -8
    cases = [
        (1.0 + e, 0x3F80),               # midpoint between 1 and 1 + 2^-7: the even one, 1
        (1.0 + 3 * e, 0x3F82),           # midpoint between 1 + 2^-7 and 1 + 2^-6: the even one
        (1.0 + e + 2.0 ** -23, 0x3F81),  # just past the midpoint: up
        (1.0 + e - 2.0 ** -23, 0x3F80),  # just short of it: down
        (-(1.0 + 3 * e), 0xBF82),        # the sign is kept, the magnitude rounds alike
        (3.5, 0x4060),                   # representable: unchanged
        (0.0, 0x0000),
        (-0.0, 0x8000),
        (65280.0 + 128.0, 0x4780),       # 2^16 - 2^8 + 2^7: midpoint, odd neighbour 0x477F, even 0x4780
    ]
    got = ref.round_bf16(np.array([c[0] for c in cases], np.float32))
    for (x, want), g in zip(cases, got):
        assert int(g) == want, (x, hex(int(g)), hex(want))


def test_bf16_special_bit_patterns():
    pats = np.array([0x7F7FFFFF,   # largest fp32: past the largest bf16 -> infinity
                     0x7F7F7FFF,   # just below that midpoint -> largest finite bf16
                     0x7F800000,   # infinity stays
                     0xFF800000,   # -infinity stays
                     0x00000001,   # smallest subnormal -> +0
                     0x00008000,   # subnormal midpoint, even neighbour 0
                     0x00018000,   # subnormal midpoint, odd neighbour 1 -> 2
                     0x7FC00000,   # quiet NaN
                     0x7F800001],  # signalling NaN: must not become infinity
                    np.uint32)
    got = ref.round_bf16(pats.view(np.float32)).astype(np.uint32)
    assert list(got[:7]) == [0x7F80, 0x7F7F, 0x7F80, 0xFF80, 0x0000, 0x0000, 0x0002]
    for g in got[7:]:
        assert (g & 0x7F80) == 0x7F80 and (g & 0x7F) != 0  # NaN


def test_bf16_is_the_nearest_lattice_point_by_brute_force():
    # every result is a bf16 value (a 16-bit pattern), no adjacent bf16 value is nearer,
    # and a result at exactly half a bf16 step has an even last bit
    rng = np.random.default_rng(21)
    x = (rng.standard_normal(20000) * np.exp2(rng.integers(-60, 60, 20000))).astype(np.float32)
    x[:2000] = (np.float32(1.0) + rng.integers(0, 2 ** 16, 2000).astype(np.float32) * np.float32(2.0 ** -23)) \
        * np.where(rng.random(2000) < 0.5, -1, 1).astype(np.float32)  # dense near the midpoints of [1, 2)
    b = ref.round_bf16(x).astype(np.uint32)
    r = _bf16_value(b).view(np.float32).astype(np.float64)
    x64 = x.astype(np.float64)
    d = np.abs(x64 - r)
    for nb in (b + 1, b - 1):
        ok = (nb & 0x7F80) != 0x7F80  # skip neighbours that are not finite
        rn = _bf16_value(nb).view(np.float32).astype(np.float64)
        dn = np.abs(x64 - rn)
        assert (d[ok] <= dn[ok]).all()
        tie = ok & (d == dn)
        assert ((b[tie] & 1) == 0).all()
    assert (d <= np.abs(x64) * 2.0 ** -8 + 1e-300).all()  # half a step of 2^-7 relative at most


def test_bf16_agrees_with_torch_cpu_conversion():
    rng = np.random.default_rng(22)
    x = (rng.standard_normal(50000) * np.exp2(rng.integers(-30, 30, 50000))).astype(np.float32)
    t = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ref.round_bf16(x), t)


def test_bf16_is_odd_and_monotone():
    rng = np.random.default_rng(23)
    x = np.sort((rng.standard_normal(10000) * 100).astype(np.float32))
    b = ref.round_bf16(x)
    np.testing.assert_array_equal(ref.round_bf16(-x), b ^ np.uint16(0x8000))
    v = _bf16_value(b.astype(np.uint32)).view(np.float32)
    assert (np.diff(v) >= 0).all()


# ----------------------------------------------------------------------------- the rotation's purpose
# (bitnet_v2_engine.py page: the Hadamard step spreads outlier channels so that the
# activation distribution becomes closer to Gaussian before the low-bit quantiser)
def test_fwht_gaussianises_heavy_tailed_tokens():
    from ternary_weight_bit_b200 import synthetic
    gen = synthetic.generator(31)
    K = 8192
    X = synthetic.student_t3((6, K), gen)
    X[:, synthetic.outlier_channels(K, 82, gen)] *= 50.0  # the wdown input: 1 % channels x50
    x = ref.rmsnorm(X.numpy())
    y = ref.fwht(x)

    def excess_kurtosis(a):
        a = a.astype(np.float64)
        m = a.mean(axis=1, keepdims=True)
        v = ((a - m) ** 2).mean(axis=1)
        return ((a - m) ** 4).mean(axis=1) / v ** 2 - 3.0

    def peak_to_rms(a):
        a = a.astype(np.float64)
        return np.abs(a).max(axis=1) / np.sqrt((a * a).mean(axis=1))

    kx, ky = excess_kurtosis(x), excess_kurtosis(y)
    px, py = peak_to_rms(x), peak_to_rms(y)
    assert (kx > 20).all() and (np.abs(ky) < 0.5).all()  # heavy-tailed in, close to Gaussian out
    assert (px > 5 * py).all() and (py < 6).all()       # the outliers are spread over all channels
    # the transform is orthogonal: the mean square (RMSNorm made it 1) is kept
    np.testing.assert_allclose((y.astype(np.float64) ** 2).mean(axis=1), 1.0, rtol=1e-4)


# ----------------------------------------------------------------------------- TL2 format
def _tl2_fields(tl2_row, j):
    """(index, sign) of triplet j of one TL2 row, read by the documented layout."""
    grp = tl2_row[(j // 32) * 20:(j // 32) * 20 + 20]
    jj = j % 32
    word = int.from_bytes(bytes(grp[4 * (jj // 8):4 * (jj // 8) + 4]), "little")
    sign = int.from_bytes(bytes(grp[16:20]), "little")
    return (word >> (4 * (jj % 8))) & 15, (sign >> jj) & 1


def test_tl2_base_table_and_mirrors_match_the_page():
    for idx, trip in _gold("tl2_base_triplets.json")["base"]:
        for sgn, t in ((0, trip), (1, [-v for v in trip])):
            row = np.array([t], np.int8)
            packed = ref.pack_tl2(row)
            want_sign = sgn if any(trip) else 0
            assert _tl2_fields(packed[0], 0) == (idx, want_sign), (trip, sgn)
            np.testing.assert_array_equal(ref.unpack_tl2(packed, 1, 3), row)


def test_tl2_layout_golden():
    for case in _gold("tl2_layout.json")["cases"]:
        K = case["K"]
        t = np.zeros((1, K), np.int8)
        for j, trip in case["triplets"].items():
            for e, v in enumerate(trip):
                if 3 * int(j) + e < K:
                    t[0, 3 * int(j) + e] = v
        packed = ref.pack_tl2(t)
        assert packed.tolist() == [case["bytes"]], case["derivation"]


def test_tl2_every_triplet_round_trips_and_mirrors():
    trips = np.array([[a, b, c] for a in (-1, 0, 1) for b in (-1, 0, 1) for c in (-1, 0, 1)], np.int8)  # 27
    row = trips.reshape(1, -1)
    packed = ref.pack_tl2(row)
    np.testing.assert_array_equal(ref.unpack_tl2(packed, 1, row.shape[1]), row)
    neg = ref.pack_tl2(-row)
    seen = set()
    for j in range(27):
        i1, s1 = _tl2_fields(packed[0], j)
        i2, s2 = _tl2_fields(neg[0], j)
        assert i1 == i2 and i1 <= 13
        assert (s1 ^ s2) == (1 if trips[j].any() else 0)
        seen.add((i1, s1))
    assert len(seen) == 27  # the 27 triplets have 27 distinct encodings (14 indices x sign)


@pytest.mark.parametrize("N,K", [(5, 96), (7, 100), (3, 4096), (2, 2560), (1, 3)])
def test_tl2_random_round_trip_and_gemm(N, K):
    rng = np.random.default_rng(N * 1000 + K)
    t = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    packed = ref.pack_tl2(t)
    assert packed.shape == (N, 20 * math.ceil(K / 96))
    np.testing.assert_array_equal(ref.unpack_tl2(packed, N, K), t)
    q = rng.integers(-128, 128, size=(4, K)).astype(np.int8)
    want = q.astype(np.int64) @ t.astype(np.int64).T
    np.testing.assert_array_equal(ref.gemm_tl2(q, packed, N), want)


def test_tl2_is_five_bits_per_three_weights():
    # the page's 1.67 bits per weight: 4-bit index + 1 sign bit per triplet
    for K in (96, 960, 6912):
        assert ref.tl2_row_bytes(K) * 8 / K == pytest.approx(5 / 3)
    assert ref.tl2_row_bytes(2560) * 8 / 2560 == pytest.approx(20 * 27 * 8 / 2560)  # padded to 2592
