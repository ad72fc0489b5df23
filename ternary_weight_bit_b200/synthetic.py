"""Seeded synthetic inputs for the H-BitLinear forward path.

This module only draws random numbers; it holds none of the method's arithmetic,
so both the CUDA path and the CPU oracle can be fed from it.  All draws use a
CPU ``torch.Generator`` seeded explicitly, in a fixed order (activations, then
the outlier-channel permutation, then the weights), so every machine sees the
same bytes.

Distributions follow the workloads the BitNet pages discuss:
  * activations N(0, 1), or Student-t with 3 degrees of freedom (heavy tails)
    with a set of outlier channels scaled up (the "outlier channels" of the
    intermediate projections that motivate the Hadamard rotation);
  * weights N(0, 0.02^2) (the initialisation of BitLinear_b158's weight).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


def generator(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def gaussian(shape, std: float, gen: torch.Generator) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, dtype=torch.float32) * std


def student_t3(shape, gen: torch.Generator) -> torch.Tensor:
    """Student-t with 3 degrees of freedom: Z / sqrt(chi2_3 / 3), chi2_3 from three fresh normals."""
    z = torch.randn(*shape, generator=gen, dtype=torch.float32)
    c = torch.zeros(*shape, dtype=torch.float32)
    for _ in range(3):
        n = torch.randn(*shape, generator=gen, dtype=torch.float32)
        c += n * n
    return z / torch.sqrt(c / 3.0)


def outlier_channels(K: int, count: int, gen: torch.Generator) -> torch.Tensor:
    """The first ``count`` entries of a seeded permutation of the K channels."""
    return torch.randperm(K, generator=gen)[:count]


@dataclass
class Case:
    """One H-BitLinear problem: activations X [M, K] and latent weights W [N, K].
    With `up` set, X is the SwiGLU gate and the layer's input is silu(X) * up."""
    name: str
    X: torch.Tensor          # float32 (or bfloat16 when x_dtype == "bf16")
    W: torch.Tensor          # float32 [N, K]
    fwht: bool
    mode: str                # "int8" or "int4"
    eps: float = 1e-5
    up: torch.Tensor | None = None

    @property
    def M(self) -> int:
        return self.X.shape[0]

    @property
    def K(self) -> int:
        return self.X.shape[1]

    @property
    def N(self) -> int:
        return self.W.shape[0]


def make_case(name: str, M: int, K: int, N: int, *, x_kind: str = "normal", outliers: int = 0,
              outlier_gain: float = 20.0, x_dtype: str = "f32", w_std: float = 0.02,
              fwht: bool = True, mode: str = "int8", seed: int = 0) -> Case:
    """Draw X (for x_kind "swiglu": the gate, then up), the outlier permutation, then W,
    from one generator seeded ``seed``."""
    gen = generator(seed)
    up = None
    if x_kind == "normal":
        X = gaussian((M, K), 1.0, gen)
    elif x_kind == "student_t3":
        X = student_t3((M, K), gen)
    elif x_kind == "swiglu":
        X = gaussian((M, K), 2.0, gen)   # gate pre-activations
        up = gaussian((M, K), 1.0, gen)
    else:
        raise ValueError(f"unknown x_kind {x_kind!r}")
    if outliers:
        ch = outlier_channels(K, outliers, gen)
        X[:, ch] *= outlier_gain
    W = gaussian((N, K), w_std, gen)
    if x_dtype == "bf16":
        X = X.to(torch.bfloat16)
        up = None if up is None else up.to(torch.bfloat16)
    elif x_dtype != "f32":
        raise ValueError(f"unknown x_dtype {x_dtype!r}")
    return Case(name, X, W, fwht, mode, up=up)


# --------------------------------------------------------------------------- workloads
def tiny_hbitlinear(seed: int = 0) -> Case:
    """Single H-BitLinear, int8 absmax, FWHT on: X [16, 256] N(0,1) with 2 channels x20; W [256, 256]."""
    return make_case("tiny_int8_fwht", 16, 256, 256, outliers=2, outlier_gain=20.0,
                     fwht=True, mode="int8", seed=seed)


def decode(M: int, N: int = 6912, K: int = 2560, seed: int = 0) -> Case:
    """Decode GEMV, int8 absmax, no FWHT: X [M, K] N(0,1); W [N, K] N(0, 0.02^2)."""
    return make_case(f"decode_M{M}_N{N}_K{K}", M, K, N, fwht=False, mode="int8", seed=seed)


def wdown_int4(M: int = 2048, K: int = 8192, N: int = 2048, seed: int = 0) -> Case:
    """Wdown-style H-BitLinear, int4 absmean + FWHT: Student-t(3) X with 1% channels x50."""
    return make_case(f"wdown_int4_M{M}_N{N}_K{K}", M, K, N, x_kind="student_t3",
                     outliers=round(0.01 * K), outlier_gain=50.0, fwht=True, mode="int4", seed=seed)


def wdown_swiglu(M: int = 2048, K: int = 8192, N: int = 2048, seed: int = 0) -> Case:
    """The FFN down projection on its SwiGLU input: gate N(0, 2^2), up N(0, 1) [M, K]; int4 + FWHT."""
    return make_case(f"wdown_swiglu_M{M}_N{N}_K{K}", M, K, N, x_kind="swiglu", fwht=True, mode="int4", seed=seed)


def prefill_int8(M: int = 4096, K: int = 4096, N: int = 4096, fwht: bool = False, seed: int = 0) -> Case:
    """Prefill int8 projection: X N(0,1) rounded to bf16 and passed as bf16; W [N, K]."""
    return make_case(f"prefill_int8_M{M}_N{N}_K{K}{'_fwht' if fwht else ''}", M, K, N,
                     x_dtype="bf16", fwht=fwht, mode="int8", seed=seed)


def msweep_int4(M: int, K: int, N: int = 4096, seed: int = 0) -> Case:
    """M-sweep of a 4096-hidden block (Wo: K=4096, Wdown: K=16384), int4 + FWHT, Student-t X with outliers."""
    return make_case(f"msweep_int4_M{M}_N{N}_K{K}", M, K, N, x_kind="student_t3",
                     outliers=round(0.01 * K), outlier_gain=50.0, fwht=True, mode="int4", seed=seed)
