"""ctypes front end of the C oracle (test infrastructure only).

Every arithmetic step happens in ``bitnet_oracle.c``; this module only marshals
numpy arrays and sequences the C calls in the order the forward path runs them:
RMSNorm -> optional FWHT -> activation quantisation -> integer GEMM on the packed
ternary weights -> dequant epilogue.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

from . import build as _build

ACT_INT8 = 0
ACT_INT4 = 1

_LIB = None


def lib(path: str | None = None) -> ctypes.CDLL:
    """Load (building first if needed) the oracle shared library."""
    global _LIB
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _LIB is None:
        # ORACLE_LIB lets the mutation tests point the pins at a deliberately broken build.
        override = os.environ.get("ORACLE_LIB")
        _LIB = _bind(ctypes.CDLL(override if override else _build.build()))
    return _LIB


def _bind(L: ctypes.CDLL) -> ctypes.CDLL:
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    F = ctypes.c_float
    D = ctypes.c_double
    I = ctypes.c_int
    L.oracle_rmsnorm.argtypes = [P, I64, I64, P, F, P]
    L.oracle_fwht.argtypes = [P, I64, I64]
    L.oracle_act_quant.argtypes = [P, I64, I64, I, F, P, P]
    L.oracle_shadow_prerounding.argtypes = [P, I64, I64, P, D, I, I, P]
    L.oracle_weight_alpha.argtypes = [P, I64]
    L.oracle_weight_alpha.restype = F
    L.oracle_ternarize.argtypes = [P, I64, F, F, P]
    L.oracle_pack.argtypes = [P, I64, I64, P]
    L.oracle_unpack.argtypes = [P, I64, I64, P]
    L.oracle_gemm_int.argtypes = [P, P, I64, I64, I64, P]
    L.oracle_gemm_packed.argtypes = [P, P, I64, I64, I64, P]
    L.oracle_dequant.argtypes = [P, P, F, I, I64, I64, P]
    L.oracle_swiglu.argtypes = [P, P, I64, P]
    L.oracle_kv_quant.argtypes = [P, I64, I64, I64, I, F, P, P, P]
    L.oracle_shadow_kv.argtypes = [P, I64, I64, I64, I, D, P]
    L.oracle_shadow_swiglu.argtypes = [P, P, I64, I64, P, D, I, I, P]
    L.oracle_round_bf16.argtypes = [P, I64, P]
    L.oracle_tl2_row_bytes.argtypes = [I64]
    L.oracle_tl2_row_bytes.restype = I64
    L.oracle_pack_tl2.argtypes = [P, I64, I64, P]
    L.oracle_unpack_tl2.argtypes = [P, I64, I64, P]
    L.oracle_gemm_tl2.argtypes = [P, P, I64, I64, I64, P]
    for name in ("oracle_rmsnorm", "oracle_fwht", "oracle_act_quant", "oracle_shadow_prerounding",
                 "oracle_ternarize", "oracle_pack", "oracle_unpack", "oracle_gemm_int",
                 "oracle_gemm_packed", "oracle_dequant", "oracle_swiglu", "oracle_shadow_swiglu",
                 "oracle_kv_quant", "oracle_shadow_kv", "oracle_pack_tl2", "oracle_unpack_tl2",
                 "oracle_gemm_tl2"):
        getattr(L, name).restype = ctypes.c_int
    return L


class OracleError(RuntimeError):
    def __init__(self, fn: str, rc: int):
        super().__init__(f"{fn} returned {rc}")
        self.rc = rc


def _p(a: np.ndarray) -> int:
    return a.ctypes.data


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


def _check(fn: str, rc: int) -> None:
    if rc != 0:
        raise OracleError(fn, rc)


# --------------------------------------------------------------------------- steps
def rmsnorm(x, g=None, eps: float = 1e-5, L=None) -> np.ndarray:
    L = L or lib()
    x = _f32(x)
    M, K = x.shape
    y = np.empty_like(x)
    gp = None if g is None else _f32(g)
    _check("rmsnorm", L.oracle_rmsnorm(_p(x), M, K, None if gp is None else _p(gp), eps, _p(y)))
    return y


def fwht(y, L=None) -> np.ndarray:
    L = L or lib()
    y = _f32(y).copy()
    M, K = y.shape
    _check("fwht", L.oracle_fwht(_p(y), M, K))
    return y


def act_quant_codes(y, mode: int, eps: float = 1e-5, L=None):
    """Step 3 on an already normalised (and possibly rotated) fp32 [M, K] array."""
    L = L or lib()
    y = _f32(y)
    M, K = y.shape
    q = np.empty((M, K), dtype=np.int8)
    s = np.empty((M,), dtype=np.float32)
    _check("act_quant", L.oracle_act_quant(_p(y), M, K, mode, eps, _p(q), _p(s)))
    return q, s


def act_quant(x, g=None, eps: float = 1e-5, fwht_on: bool = False, mode: int = ACT_INT8, L=None):
    """Steps 1-3: RMSNorm -> optional FWHT -> quantisation. Returns (codes int8 [M,K], scale fp32 [M])."""
    L = L or lib()
    y = rmsnorm(x, g, eps, L=L)
    if fwht_on:
        y = fwht(y, L=L)
    return act_quant_codes(y, mode, eps, L=L)


def shadow(x, g=None, eps: float = 1e-5, fwht_on: bool = False, mode: int = ACT_INT8, L=None) -> np.ndarray:
    """fp64 pre-rounding value of every activation code."""
    L = L or lib()
    x = _f32(x)
    M, K = x.shape
    v = np.empty((M, K), dtype=np.float64)
    gp = None if g is None else _f32(g)
    _check("shadow", L.oracle_shadow_prerounding(_p(x), M, K, None if gp is None else _p(gp),
                                                 float(np.float32(eps)), int(fwht_on), mode, _p(v)))
    return v


def swiglu(gate, up, L=None) -> np.ndarray:
    """SwiGLU input of the FFN down projection: silu(gate) * up, fp32 (same shape)."""
    L = L or lib()
    g = _f32(gate)
    u = _f32(up)
    assert g.shape == u.shape
    out = np.empty_like(g)
    _check("swiglu", L.oracle_swiglu(_p(g), _p(u), g.size, _p(out)))
    return out


def shadow_swiglu(gate, up, g=None, eps: float = 1e-5, fwht_on: bool = False, mode: int = ACT_INT8,
                  L=None) -> np.ndarray:
    """fp64 pre-rounding value of every activation code of the SwiGLU input."""
    L = L or lib()
    ga = _f32(gate)
    u = _f32(up)
    M, K = ga.shape
    v = np.empty((M, K), dtype=np.float64)
    gp = None if g is None else _f32(g)
    _check("shadow_swiglu", L.oracle_shadow_swiglu(_p(ga), _p(u), M, K, None if gp is None else _p(gp),
                                                   float(np.float32(eps)), int(fwht_on), mode, _p(v)))
    return v


def kv_quant(kv, bits: int, eps: float = 1e-5, L=None):
    """Low-bit KV cache of a [B, H, S, D] (or [BH, S, D]) tensor: (codes int8, step fp32 [.., S], deq fp32)."""
    L = L or lib()
    x = _f32(kv)
    S, D = x.shape[-2], x.shape[-1]
    BH = x.size // (S * D) if S * D else 0
    codes = np.empty(x.shape, dtype=np.int8)
    step = np.empty(x.shape[:-1], dtype=np.float32)
    deq = np.empty(x.shape, dtype=np.float32)
    _check("kv_quant", L.oracle_kv_quant(_p(x), BH, S, D, bits, eps, _p(codes), _p(step), _p(deq)))
    return codes, step, deq


def shadow_kv(kv, bits: int, eps: float = 1e-5, L=None) -> np.ndarray:
    L = L or lib()
    x = _f32(kv)
    S, D = x.shape[-2], x.shape[-1]
    BH = x.size // (S * D) if S * D else 0
    v = np.empty(x.shape, dtype=np.float64)
    _check("shadow_kv", L.oracle_shadow_kv(_p(x), BH, S, D, bits, float(np.float32(eps)), _p(v)))
    return v


def weight_alpha(W, L=None) -> np.float32:
    L = L or lib()
    W = _f32(W)
    return np.float32(L.oracle_weight_alpha(_p(W), W.size))


def ternarize(W, alpha, eps: float = 1e-5, L=None) -> np.ndarray:
    L = L or lib()
    W = _f32(W)
    t = np.empty(W.shape, dtype=np.int8)
    _check("ternarize", L.oracle_ternarize(_p(W), W.size, float(alpha), eps, _p(t)))
    return t


def pack(t, L=None) -> np.ndarray:
    L = L or lib()
    t = np.ascontiguousarray(t, dtype=np.int8)
    N, K = t.shape
    out = np.empty((N, K // 4), dtype=np.uint8)
    _check("pack", L.oracle_pack(_p(t), N, K, _p(out)))
    return out


def unpack(packed, N: int, K: int, L=None) -> np.ndarray:
    L = L or lib()
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    t = np.empty((N, K), dtype=np.int8)
    _check("unpack", L.oracle_unpack(_p(packed), N, K, _p(t)))
    return t


def tl2_row_bytes(K: int, L=None) -> int:
    """Bytes of one row in the TL2 format (20 per 32 triplets)."""
    return int((L or lib()).oracle_tl2_row_bytes(K))


def pack_tl2(t, L=None) -> np.ndarray:
    """Ternary codes [N, K] -> TL2 bytes [N, 20 * ceil(K / 96)] (index and sign planes)."""
    L = L or lib()
    t = np.ascontiguousarray(t, dtype=np.int8)
    N, K = t.shape
    out = np.empty((N, tl2_row_bytes(K, L)), dtype=np.uint8)
    _check("pack_tl2", L.oracle_pack_tl2(_p(t), N, K, _p(out)))
    return out


def unpack_tl2(tl2, N: int, K: int, L=None) -> np.ndarray:
    L = L or lib()
    tl2 = np.ascontiguousarray(tl2, dtype=np.uint8)
    t = np.empty((N, K), dtype=np.int8)
    _check("unpack_tl2", L.oracle_unpack_tl2(_p(tl2), N, K, _p(t)))
    return t


def gemm_tl2(q, tl2, N: int, L=None) -> np.ndarray:
    L = L or lib()
    q = np.ascontiguousarray(q, dtype=np.int8)
    tl2 = np.ascontiguousarray(tl2, dtype=np.uint8)
    M, K = q.shape
    acc = np.empty((M, N), dtype=np.int32)
    _check("gemm_tl2", L.oracle_gemm_tl2(_p(q), _p(tl2), M, N, K, _p(acc)))
    return acc


def pack_weights(W, eps: float = 1e-5, L=None):
    """Step 4: (packed uint8 [N, K/4], alpha float32, t int8 [N, K])."""
    alpha = weight_alpha(W, L=L)
    t = ternarize(W, alpha, eps, L=L)
    return pack(t, L=L), alpha, t


def gemm_int(q, t, L=None) -> np.ndarray:
    L = L or lib()
    q = np.ascontiguousarray(q, dtype=np.int8)
    t = np.ascontiguousarray(t, dtype=np.int8)
    M, K = q.shape
    N = t.shape[0]
    acc = np.empty((M, N), dtype=np.int32)
    _check("gemm_int", L.oracle_gemm_int(_p(q), _p(t), M, N, K, _p(acc)))
    return acc


def gemm_packed(q, packed, N: int, L=None) -> np.ndarray:
    L = L or lib()
    q = np.ascontiguousarray(q, dtype=np.int8)
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    M, K = q.shape
    acc = np.empty((M, N), dtype=np.int32)
    _check("gemm_packed", L.oracle_gemm_packed(_p(q), _p(packed), M, N, K, _p(acc)))
    return acc


def dequant(acc, scale_x, alpha, mode: int, L=None) -> np.ndarray:
    L = L or lib()
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    s = _f32(scale_x)
    M, N = acc.shape
    out = np.empty((M, N), dtype=np.float32)
    _check("dequant", L.oracle_dequant(_p(acc), _p(s), float(alpha), mode, M, N, _p(out)))
    return out


def round_bf16(x, L=None) -> np.ndarray:
    """bf16 bit patterns (uint16) of x rounded to nearest, ties to even."""
    L = L or lib()
    x = _f32(x)
    out = np.empty(x.shape, dtype=np.uint16)
    _check("round_bf16", L.oracle_round_bf16(_p(x), x.size, _p(out)))
    return out


@dataclass
class ForwardResult:
    codes: np.ndarray
    scale_x: np.ndarray
    acc: np.ndarray
    out: np.ndarray


def hbitlinear_forward(x, packed, alpha, N: int, g=None, eps: float = 1e-5, fwht_on: bool = True,
                       mode: int = ACT_INT8, L=None) -> ForwardResult:
    """The whole forward: codes, per-token scale, int32 accumulators and fp32 output."""
    q, s = act_quant(x, g, eps, fwht_on, mode, L=L)
    acc = gemm_packed(q, packed, N, L=L)
    out = dequant(acc, s, alpha, mode, L=L)
    return ForwardResult(q, s, acc, out)
