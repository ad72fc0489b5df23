"""ctypes binding of libbitnet.so (the C ABI in include/bitnet.h).

Argument marshalling only: every step of the H-BitLinear path runs in the CUDA
kernels of libbitnet.so.  torch supplies device memory and the current stream.
There is no fallback: if the library is missing or the device is not a CUDA
device, the calls raise.
"""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libbitnet.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "bitnet.h")

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED_SHAPE = 2
ERR_NOT_POW2 = 3
ERR_CUDA = 4
ERR_TIMEOUT = 5
ERR_WORKSPACE = 6

ACT_INT8_ABSMAX = 0
ACT_INT4_ABSMEAN = 1
F32 = 0
BF16 = 1

_LIBS: dict = {}  # loaded libraries by path


class BitnetError(RuntimeError):
    def __init__(self, fn: str, status: int, text: str):
        super().__init__(f"{fn}: status {status} ({text})")
        self.status = status


def declared_symbols(header: str = HEADER) -> list[str]:
    """Names of every function the C header declares."""
    with open(header) as f:
        src = f.read()
    return sorted(set(re.findall(r"BITNET_API\s+[\w\s\*]*?\b(bitnet_\w+)\s*\(", src)))


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libbitnet.so and declare its signatures (no CUDA call is made)."""
    if path in _LIBS:
        return _LIBS[path]
    if not os.path.exists(path):
        raise RuntimeError(f"libbitnet.so not built: {path} is missing (run __graft_entry__.build())")
    L = ctypes.CDLL(path)
    P, I64, F, I, SZ, U32 = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_int, ctypes.c_size_t,
                             ctypes.c_uint32)
    sigs = {
        "bitnet_pack_workspace_bytes": (SZ, [I64, I64]),
        "bitnet_pack_ternary": (I, [P, I64, I64, F, P, P, P, SZ, P]),
        "bitnet_act_quant": (I, [P, I, I64, I64, P, F, I, I, P, P, P]),
        "bitnet_ternary_gemm": (I, [P, P, I, P, P, I64, I64, I64, P, P, P, SZ, P]),
        "bitnet_gemm_workspace_bytes": (SZ, [I64, I64, I64]),
        "bitnet_workspace_bytes": (SZ, [I64, I64, I64]),
        "bitnet_forward_kernel_count": (I, [I64, I64, I64, I, I]),
        "bitnet_tl2_bytes": (SZ, [I64, I64]),
        "bitnet_pack_tl2": (I, [P, I64, I64, P, P]),
        "bitnet_ternary_gemm_tl2": (I, [P, P, I, P, P, I64, I64, I64, P, P, P]),
        "bitnet_hbitlinear_forward_tl2": (I, [P, I, I64, I64, P, F, I, I, P, P, I64, P, P, SZ, P]),
        "bitnet_forward_workspace_bytes": (SZ, [I64, I64]),
        "bitnet_hbitlinear_forward": (I, [P, I, I64, I64, P, F, I, I, P, P, I64, P, P, SZ, P]),
        "bitnet_hbitlinear_forward_noalloc": (I, [P, I, I64, I64, P, F, I, I, P, P, I64, P, P]),
        "bitnet_act_quant_swiglu": (I, [P, P, I, I64, I64, P, F, I, I, P, P, P]),
        "bitnet_kv_quant": (I, [P, I, I64, I64, I64, I, F, P, P, P, P]),
        "bitnet_ternary_gemm_ex": (I, [P, P, I, P, P, I64, I64, I64, P, I, P, P]),
        "bitnet_hbitlinear_forward_ex": (I, [P, I, I64, I64, P, F, I, I, P, P, I64, P, I, P, SZ, P]),
        "bitnet_hbitlinear_forward_swiglu": (I, [P, P, I, I64, I64, P, F, I, I, P, P, I64, P, P, SZ, P]),
        "bitnet_status_string": (ctypes.c_char_p, [I]),
        "bitnet_get_last_device_status": (I, [P]),
        "bitnet_selftest_wait_timeout": (I, [U32, P]),
        "bitnet_abi_version": (I, []),
        "bitnet_gemm_token_tile": (I, [I64, I64, I64]),
        "bitnet_gemm_force_token_tile": (I, [I]),
        "bitnet_gemm_force_k_splits": (I, [I]),
        "bitnet_forward_gemm_plan": (I, [I64, I64, I64, ctypes.POINTER(ctypes.c_int)]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _LIBS[path] = L
    return L


def status_string(status: int) -> str:
    return load().bitnet_status_string(status).decode()


def check(fn: str, status: int) -> None:
    if status != OK:
        raise BitnetError(fn, status, status_string(status))
