"""ternary_weight_bit_b200 -- the BitNet H-BitLinear forward path on B200 (sm_100a).

Python front end of libbitnet.so.  The functions carry the names of the C ABI
(include/bitnet.h) and only marshal arguments: torch tensors supply device
memory and the current CUDA stream, the kernels of libbitnet.so do every step.
There is no CPU or PyTorch fallback; a missing library or a non-CUDA tensor
raises.

    packed, alpha = bitnet_pack_ternary(W)                        # once per weight
    out = bitnet_hbitlinear_forward(X, packed, alpha, N, fwht=True, mode="int4")

The step-by-step entry points bitnet_act_quant and bitnet_ternary_gemm expose the
intermediate int8 codes, per-token scales and (optionally) the int32 accumulators.
"""
from __future__ import annotations

import ctypes

import torch

from . import _native
from ._native import BitnetError

__all__ = [
    "BitnetError", "HBitLinear", "bitnet_pack_ternary", "bitnet_act_quant", "bitnet_ternary_gemm",
    "bitnet_hbitlinear_forward", "bitnet_hbitlinear_forward_noalloc", "bitnet_forward_workspace_bytes", "bitnet_pack_workspace_bytes",
    "bitnet_get_last_device_status", "bitnet_selftest_wait_timeout", "bitnet_abi_version", "mode_id",
    "bitnet_gemm_token_tile", "bitnet_gemm_force_token_tile", "bitnet_gemm_force_k_splits",
    "bitnet_forward_gemm_plan", "bitnet_workspace_bytes", "bitnet_gemm_workspace_bytes",
    "bitnet_forward_kernel_count", "bitnet_tl2_bytes", "bitnet_pack_tl2", "bitnet_ternary_gemm_tl2",
    "bitnet_hbitlinear_forward_tl2",
    "bitnet_act_quant_swiglu", "bitnet_hbitlinear_forward_swiglu", "bitnet_kv_quant",
    "bitnet_ternary_gemm_ex", "bitnet_hbitlinear_forward_ex",
]

_MODES = {"int8": _native.ACT_INT8_ABSMAX, "int4": _native.ACT_INT4_ABSMEAN}


def mode_id(mode) -> int:
    if isinstance(mode, int):
        return mode
    try:
        return _MODES[mode]
    except KeyError:
        raise ValueError(f"mode must be 'int8' or 'int4', got {mode!r}") from None


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype=None, shape=None) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (libbitnet has no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def bitnet_abi_version() -> int:
    return _native.load().bitnet_abi_version()


def bitnet_gemm_token_tile(M: int, N: int, K: int) -> int:
    """Token-tile size of the tcgen05 GEMM for this shape (0: decode kernel, -1: rejected)."""
    return _native.load().bitnet_gemm_token_tile(M, N, K)


def bitnet_forward_gemm_plan(M: int, N: int, K: int) -> tuple:
    """(token tile, k-splits) of the GEMM inside the forward; (0, 0) for the decode kernel."""
    sp = ctypes.c_int(0)
    tile = _native.load().bitnet_forward_gemm_plan(M, N, K, ctypes.byref(sp))
    return tile, sp.value


def bitnet_gemm_force_token_tile(token_tile: int) -> None:
    """Force the GEMM token tile (256/224/192/128/64) process-wide; 0 restores the automatic choice."""
    _native.check("bitnet_gemm_force_token_tile", _native.load().bitnet_gemm_force_token_tile(token_tile))


def bitnet_gemm_force_k_splits(k_splits: int) -> None:
    """Force the forward's k-split count (0 = automatic; 1, 2, 4, 8 where the shape allows it)."""
    _native.check("bitnet_gemm_force_k_splits", _native.load().bitnet_gemm_force_k_splits(k_splits))


def bitnet_pack_workspace_bytes(N: int, K: int) -> int:
    return _native.load().bitnet_pack_workspace_bytes(N, K)


def bitnet_workspace_bytes(M: int, N: int, K: int) -> int:
    """One workspace size that serves pack, forward and GEMM on an M x N x K problem."""
    return _native.load().bitnet_workspace_bytes(M, N, K)


def bitnet_gemm_workspace_bytes(M: int, N: int, K: int) -> int:
    return _native.load().bitnet_gemm_workspace_bytes(M, N, K)


def bitnet_forward_kernel_count(M: int, N: int, K: int, fwht: bool = True, gain: bool = False) -> int:
    """Kernels the forward launches for this problem (1 when the decode kernel runs the
    activation step itself, else 2; 0 for M == 0; -1 for rejected sizes)."""
    return _native.load().bitnet_forward_kernel_count(M, N, K, int(bool(fwht)), int(bool(gain)))


def bitnet_forward_workspace_bytes(M: int, K: int) -> int:
    return _native.load().bitnet_forward_workspace_bytes(M, K)


def bitnet_pack_ternary(W: torch.Tensor, eps: float = 1e-5, packed=None, alpha=None, ws=None, stream=None):
    """Ternarise W [N, K] (fp32, CUDA) with its absmean and pack it at 2 bits per weight.

    Returns (packed uint8 [N, K/4], alpha float32 [1]), both on W's device."""
    L = _native.load()
    _need(W, "W", torch.float32)
    N, K = W.shape
    dev = W.device
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device=dev) if packed is None else packed
    alpha = torch.empty((1,), dtype=torch.float32, device=dev) if alpha is None else alpha
    _need(packed, "packed", torch.uint8, (N, K // 4))
    _need(alpha, "alpha", torch.float32)
    nbytes = L.bitnet_pack_workspace_bytes(N, K)
    ws = torch.empty((nbytes,), dtype=torch.uint8, device=dev) if ws is None else ws
    _native.check("bitnet_pack_ternary",
                  L.bitnet_pack_ternary(_ptr(W), N, K, eps, _ptr(packed), _ptr(alpha), _ptr(ws), ws.numel(),
                                        _stream(stream)))
    return packed, alpha


def _xdt(X: torch.Tensor) -> int:
    if X.dtype == torch.float32:
        return _native.F32
    if X.dtype == torch.bfloat16:
        return _native.BF16
    raise ValueError(f"X must be float32 or bfloat16, got {X.dtype}")


def bitnet_act_quant(X: torch.Tensor, gain=None, eps: float = 1e-5, fwht: bool = True, mode="int8",
                     codes=None, scale_x=None, stream=None):
    """RMSNorm -> optional FWHT -> per-token int8/int4 codes.  Returns (codes int8 [M,K], scale fp32 [M])."""
    L = _native.load()
    _need(X, "X")
    M, K = X.shape
    codes = torch.empty((M, K), dtype=torch.int8, device=X.device) if codes is None else codes
    scale_x = torch.empty((M,), dtype=torch.float32, device=X.device) if scale_x is None else scale_x
    _need(codes, "codes", torch.int8, (M, K))
    _need(scale_x, "scale_x", torch.float32, (M,))
    if gain is not None:
        _need(gain, "gain", torch.float32, (K,))
    _native.check("bitnet_act_quant",
                  L.bitnet_act_quant(_ptr(X), _xdt(X), M, K, _ptr(gain), eps, int(bool(fwht)), mode_id(mode),
                                     _ptr(codes), _ptr(scale_x), _stream(stream)))
    return codes, scale_x


def _need_pair(gate: torch.Tensor, up: torch.Tensor) -> None:
    _need(gate, "gate")
    _need(up, "up", gate.dtype, tuple(gate.shape))


def bitnet_act_quant_swiglu(gate: torch.Tensor, up: torch.Tensor, gain=None, eps: float = 1e-5, fwht: bool = True,
                            mode="int4", codes=None, scale_x=None, stream=None):
    """bitnet_act_quant on the SwiGLU product silu(gate) * up (formed in registers, never stored).
    Returns (codes int8 [M,K], scale fp32 [M])."""
    L = _native.load()
    _need_pair(gate, up)
    M, K = gate.shape
    codes = torch.empty((M, K), dtype=torch.int8, device=gate.device) if codes is None else codes
    scale_x = torch.empty((M,), dtype=torch.float32, device=gate.device) if scale_x is None else scale_x
    _need(codes, "codes", torch.int8, (M, K))
    _need(scale_x, "scale_x", torch.float32, (M,))
    if gain is not None:
        _need(gain, "gain", torch.float32, (K,))
    _native.check("bitnet_act_quant_swiglu",
                  L.bitnet_act_quant_swiglu(_ptr(gate), _ptr(up), _xdt(gate), M, K, _ptr(gain), eps, int(bool(fwht)),
                                            mode_id(mode), _ptr(codes), _ptr(scale_x), _stream(stream)))
    return codes, scale_x


def bitnet_hbitlinear_forward_swiglu(gate: torch.Tensor, up: torch.Tensor, packed: torch.Tensor, alpha: torch.Tensor,
                                     N: int, gain=None, eps: float = 1e-5, fwht: bool = True, mode="int4", out=None,
                                     ws=None, stream=None):
    """The H-BitLinear down projection of a BitNet v2 FFN on silu(gate) * up.  Returns out fp32 [M, N]."""
    L = _native.load()
    _need_pair(gate, up)
    M, K = gate.shape
    _need(packed, "packed", torch.uint8, (N, K // 4))
    _need(alpha, "alpha", torch.float32)
    if gain is not None:
        _need(gain, "gain", torch.float32, (K,))
    out = torch.empty((M, N), dtype=torch.float32, device=gate.device) if out is None else out
    _need(out, "out", torch.float32, (M, N))
    nbytes = L.bitnet_forward_workspace_bytes(M, K)
    ws = torch.empty((max(nbytes, 256),), dtype=torch.uint8, device=gate.device) if ws is None else ws
    _need(ws, "ws", torch.uint8)
    _native.check("bitnet_hbitlinear_forward_swiglu",
                  L.bitnet_hbitlinear_forward_swiglu(_ptr(gate), _ptr(up), _xdt(gate), M, K, _ptr(gain), eps,
                                                     int(bool(fwht)), mode_id(mode), _ptr(packed), _ptr(alpha), N,
                                                     _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def bitnet_kv_quant(kv: torch.Tensor, bits: int = 4, eps: float = 1e-5, dequant: bool = False, codes=None,
                    step=None, deq=None, stream=None):
    """Low-bit KV cache of a [..., S, D] key or value tensor (token 0 kept at int8).
    Returns (codes int8 [..., S, D], step fp32 [..., S], deq fp32 [..., S, D] or None)."""
    L = _native.load()
    _need(kv, "kv")
    S, D = kv.shape[-2], kv.shape[-1]
    BH = kv.numel() // (S * D) if S * D else 0
    codes = torch.empty(kv.shape, dtype=torch.int8, device=kv.device) if codes is None else codes
    step = torch.empty(kv.shape[:-1], dtype=torch.float32, device=kv.device) if step is None else step
    if dequant and deq is None:
        deq = torch.empty(kv.shape, dtype=torch.float32, device=kv.device)
    _need(codes, "codes", torch.int8, tuple(kv.shape))
    _need(step, "step", torch.float32, tuple(kv.shape[:-1]))
    if deq is not None:
        _need(deq, "deq", torch.float32, tuple(kv.shape))
    _native.check("bitnet_kv_quant", L.bitnet_kv_quant(_ptr(kv), _xdt(kv), BH, S, D, bits, eps, _ptr(codes),
                                                       _ptr(step), _ptr(deq), _stream(stream)))
    return codes, step, deq


def bitnet_ternary_gemm(codes: torch.Tensor, scale_x: torch.Tensor, mode, packed: torch.Tensor,
                        alpha: torch.Tensor, N: int, out=None, acc_out=None, ws=None, stream=None):
    """acc = codes @ t^T (exact int32) and out = acc * (alpha * scale_x / Q).  Returns out fp32 [M, N].

    ws (optional, uint8, >= bitnet_gemm_workspace_bytes) lets a problem with few output
    tiles split K; without it K is never split.  The result is the same either way."""
    L = _native.load()
    _need(codes, "codes", torch.int8)
    M, K = codes.shape
    _need(scale_x, "scale_x", torch.float32, (M,))
    _need(packed, "packed", torch.uint8, (N, K // 4))
    _need(alpha, "alpha", torch.float32)
    out = torch.empty((M, N), dtype=torch.float32, device=codes.device) if out is None else out
    _need(out, "out", torch.float32, (M, N))
    if acc_out is not None:
        _need(acc_out, "acc_out", torch.int32, (M, N))
    if ws is not None:
        _need(ws, "ws", torch.uint8)
    _native.check("bitnet_ternary_gemm",
                  L.bitnet_ternary_gemm(_ptr(codes), _ptr(scale_x), mode_id(mode), _ptr(packed), _ptr(alpha), M, N,
                                        K, _ptr(out), _ptr(acc_out), _ptr(ws), 0 if ws is None else ws.numel(),
                                        _stream(stream)))
    return out


def bitnet_hbitlinear_forward(X: torch.Tensor, packed: torch.Tensor, alpha: torch.Tensor, N: int, gain=None,
                              eps: float = 1e-5, fwht: bool = True, mode="int8", out=None, ws=None, stream=None):
    """The whole H-BitLinear forward.  Returns out fp32 [M, N]."""
    L = _native.load()
    _need(X, "X")
    M, K = X.shape
    _need(packed, "packed", torch.uint8, (N, K // 4))
    _need(alpha, "alpha", torch.float32)
    if gain is not None:
        _need(gain, "gain", torch.float32, (K,))
    out = torch.empty((M, N), dtype=torch.float32, device=X.device) if out is None else out
    _need(out, "out", torch.float32, (M, N))
    nbytes = L.bitnet_forward_workspace_bytes(M, K)
    ws = torch.empty((max(nbytes, 256),), dtype=torch.uint8, device=X.device) if ws is None else ws
    _need(ws, "ws", torch.uint8)
    _native.check("bitnet_hbitlinear_forward",
                  L.bitnet_hbitlinear_forward(_ptr(X), _xdt(X), M, K, _ptr(gain), eps, int(bool(fwht)),
                                              mode_id(mode), _ptr(packed), _ptr(alpha), N, _ptr(out), _ptr(ws),
                                              ws.numel(), _stream(stream)))
    return out


def bitnet_hbitlinear_forward_noalloc(X: torch.Tensor, packed: torch.Tensor, alpha: torch.Tensor, N: int,
                                      gain=None, eps: float = 1e-5, fwht: bool = True, mode="int8", out=None,
                                      stream=None):
    """The forward without a caller workspace, for callers that cannot allocate device memory
    (the scratch is a fixed 4 MiB array inside the library; see include/bitnet.h)."""
    L = _native.load()
    _need(X, "X")
    M, K = X.shape
    _need(packed, "packed", torch.uint8, (N, K // 4))
    _need(alpha, "alpha", torch.float32)
    if gain is not None:
        _need(gain, "gain", torch.float32, (K,))
    if out is None:
        raise ValueError("out must be given: this entry point is for callers that cannot allocate")
    _need(out, "out", torch.float32, (M, N))
    _native.check("bitnet_hbitlinear_forward_noalloc",
                  L.bitnet_hbitlinear_forward_noalloc(_ptr(X), _xdt(X), M, K, _ptr(gain), eps, int(bool(fwht)),
                                                      mode_id(mode), _ptr(packed), _ptr(alpha), N, _ptr(out),
                                                      _stream(stream)))
    return out


_OUT_DT = {torch.float32: 0, torch.bfloat16: 1}  # bitnet_dtype_t


def _out_dt(dtype) -> int:
    if dtype not in _OUT_DT:
        raise ValueError(f"output dtype must be torch.float32 or torch.bfloat16, got {dtype}")
    return _OUT_DT[dtype]


def bitnet_ternary_gemm_ex(codes: torch.Tensor, scale_x: torch.Tensor, mode, packed: torch.Tensor,
                           alpha: torch.Tensor, N: int, out_dtype=torch.bfloat16, out=None, acc_out=None,
                           stream=None):
    """bitnet_ternary_gemm with the output stored as out_dtype (fp32, or bf16 rounded to nearest even)."""
    L = _native.load()
    _need(codes, "codes", torch.int8)
    M, K = codes.shape
    _need(scale_x, "scale_x", torch.float32, (M,))
    _need(packed, "packed", torch.uint8, (N, K // 4))
    _need(alpha, "alpha", torch.float32)
    dt = _out_dt(out_dtype)
    out = torch.empty((M, N), dtype=out_dtype, device=codes.device) if out is None else out
    _need(out, "out", out_dtype, (M, N))
    if acc_out is not None:
        _need(acc_out, "acc_out", torch.int32, (M, N))
    _native.check("bitnet_ternary_gemm_ex",
                  L.bitnet_ternary_gemm_ex(_ptr(codes), _ptr(scale_x), mode_id(mode), _ptr(packed), _ptr(alpha), M,
                                           N, K, _ptr(out), dt, _ptr(acc_out), _stream(stream)))
    return out


def bitnet_hbitlinear_forward_ex(X: torch.Tensor, packed: torch.Tensor, alpha: torch.Tensor, N: int, gain=None,
                                 eps: float = 1e-5, fwht: bool = True, mode="int8", out_dtype=torch.bfloat16,
                                 out=None, ws=None, stream=None):
    """bitnet_hbitlinear_forward with the output stored as out_dtype (fp32, or bf16 rounded to nearest even)."""
    L = _native.load()
    _need(X, "X")
    M, K = X.shape
    _need(packed, "packed", torch.uint8, (N, K // 4))
    _need(alpha, "alpha", torch.float32)
    if gain is not None:
        _need(gain, "gain", torch.float32, (K,))
    dt = _out_dt(out_dtype)
    out = torch.empty((M, N), dtype=out_dtype, device=X.device) if out is None else out
    _need(out, "out", out_dtype, (M, N))
    nbytes = L.bitnet_forward_workspace_bytes(M, K)
    ws = torch.empty((max(nbytes, 256),), dtype=torch.uint8, device=X.device) if ws is None else ws
    _need(ws, "ws", torch.uint8)
    _native.check("bitnet_hbitlinear_forward_ex",
                  L.bitnet_hbitlinear_forward_ex(_ptr(X), _xdt(X), M, K, _ptr(gain), eps, int(bool(fwht)),
                                                 mode_id(mode), _ptr(packed), _ptr(alpha), N, _ptr(out), dt,
                                                 _ptr(ws), ws.numel(), _stream(stream)))
    return out


def bitnet_tl2_bytes(N: int, K: int) -> int:
    """Bytes of an N x K weight matrix in the TL2 format (20 per 96 weights of a row)."""
    return _native.load().bitnet_tl2_bytes(N, K)


def bitnet_pack_tl2(packed: torch.Tensor, K: int, tl2=None, stream=None):
    """2-bit packed weights [N, K/4] -> the TL2 format (5 bits per 3 weights), exactly.
    Returns uint8 [N, 20 * ceil(K/96)]."""
    L = _native.load()
    _need(packed, "packed", torch.uint8)
    N = packed.shape[0]
    if packed.shape[1] * 4 != K:
        raise ValueError(f"packed must be [N, K/4] = [N, {K // 4}], got {tuple(packed.shape)}")
    rb = L.bitnet_tl2_bytes(1, K)
    tl2 = torch.empty((N, rb), dtype=torch.uint8, device=packed.device) if tl2 is None else tl2
    _need(tl2, "tl2", torch.uint8, (N, rb))
    _native.check("bitnet_pack_tl2", L.bitnet_pack_tl2(_ptr(packed), N, K, _ptr(tl2), _stream(stream)))
    return tl2


def bitnet_ternary_gemm_tl2(codes: torch.Tensor, scale_x: torch.Tensor, mode, tl2: torch.Tensor,
                            alpha: torch.Tensor, N: int, out=None, acc_out=None, stream=None):
    """bitnet_ternary_gemm with TL2 weights (M <= 16).  Returns out fp32 [M, N]."""
    L = _native.load()
    _need(codes, "codes", torch.int8)
    M, K = codes.shape
    _need(scale_x, "scale_x", torch.float32, (M,))
    _need(tl2, "tl2", torch.uint8, (N, L.bitnet_tl2_bytes(1, K)))
    _need(alpha, "alpha", torch.float32)
    out = torch.empty((M, N), dtype=torch.float32, device=codes.device) if out is None else out
    _need(out, "out", torch.float32, (M, N))
    if acc_out is not None:
        _need(acc_out, "acc_out", torch.int32, (M, N))
    _native.check("bitnet_ternary_gemm_tl2",
                  L.bitnet_ternary_gemm_tl2(_ptr(codes), _ptr(scale_x), mode_id(mode), _ptr(tl2), _ptr(alpha), M, N,
                                            K, _ptr(out), _ptr(acc_out), _stream(stream)))
    return out


def bitnet_hbitlinear_forward_tl2(X: torch.Tensor, tl2: torch.Tensor, alpha: torch.Tensor, N: int, gain=None,
                                  eps: float = 1e-5, fwht: bool = True, mode="int8", out=None, ws=None,
                                  stream=None):
    """The whole H-BitLinear forward with TL2 weights (M <= 16).  Returns out fp32 [M, N]."""
    L = _native.load()
    _need(X, "X")
    M, K = X.shape
    _need(tl2, "tl2", torch.uint8, (N, L.bitnet_tl2_bytes(1, K)))
    _need(alpha, "alpha", torch.float32)
    if gain is not None:
        _need(gain, "gain", torch.float32, (K,))
    out = torch.empty((M, N), dtype=torch.float32, device=X.device) if out is None else out
    _need(out, "out", torch.float32, (M, N))
    nbytes = L.bitnet_forward_workspace_bytes(M, K)
    ws = torch.empty((max(nbytes, 256),), dtype=torch.uint8, device=X.device) if ws is None else ws
    _need(ws, "ws", torch.uint8)
    _native.check("bitnet_hbitlinear_forward_tl2",
                  L.bitnet_hbitlinear_forward_tl2(_ptr(X), _xdt(X), M, K, _ptr(gain), eps, int(bool(fwht)),
                                                  mode_id(mode), _ptr(tl2), _ptr(alpha), N, _ptr(out), _ptr(ws),
                                                  ws.numel(), _stream(stream)))
    return out


def bitnet_get_last_device_status(stream=None) -> int:
    """Synchronise the stream, return and clear the kernels' timeout status word."""
    return _native.load().bitnet_get_last_device_status(_stream(stream))


def bitnet_selftest_wait_timeout(limit_us: int, stream=None) -> None:
    _native.check("bitnet_selftest_wait_timeout",
                  _native.load().bitnet_selftest_wait_timeout(limit_us, _stream(stream)))


class HBitLinear:
    """Pack once, forward many: an H-BitLinear layer over a fixed weight matrix.

    W is [out_features, in_features] fp32 on a CUDA device.  fwht=True gives the
    H-BitLinear of the BitNet v2 page (Wo / Wdown); fwht=False the plain BitLinear.
    The layer keeps one forward workspace and reuses it, so calls of the same layer
    on different streams must be ordered (events, or one stream)."""

    def __init__(self, W: torch.Tensor, mode="int8", fwht: bool = True, eps: float = 1e-5, gain=None):
        self.N, self.K = W.shape
        self.mode = mode_id(mode)
        self.fwht = bool(fwht)
        self.eps = float(eps)
        self.gain = gain
        self.packed, self.alpha = bitnet_pack_ternary(W, eps)
        self._ws = None

    def workspace(self, M: int, device) -> torch.Tensor:
        need = max(bitnet_forward_workspace_bytes(M, self.K), 256)
        if self._ws is None or self._ws.numel() < need or self._ws.device != device:
            self._ws = torch.empty((need,), dtype=torch.uint8, device=device)
        return self._ws

    def __call__(self, X: torch.Tensor, out=None, stream=None) -> torch.Tensor:
        return bitnet_hbitlinear_forward(X, self.packed, self.alpha, self.N, gain=self.gain, eps=self.eps,
                                         fwht=self.fwht, mode=self.mode, out=out,
                                         ws=self.workspace(X.shape[0], X.device), stream=stream)
