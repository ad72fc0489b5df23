"""Comparison rules between the CUDA path and the oracle (shared by the GPU tests,
the smoke check and the benchmark's parity spot checks).

Rules (from the BitNet v2 page's Eq. 5/6 and the exactness of integer arithmetic):
  * Packed weight bytes and alpha: identical.
  * int32 accumulators on the same codes: identical.
  * fp32 output on the same codes and scales: out = (float)acc * f, f computed in
    the same IEEE order on both sides, so identical.  The per-token scales
    themselves differ only by fp32 summation order, within scale_rtol(K, mode).
  * Activation codes: the GPU sums and rotates in another order than the oracle's
    sequential fp32 loops, so a code may differ by exactly one, only where the exact
    (fp64) pre-rounding value lies within TIE_TOL of the half-integer between the
    two codes, and on at most FLIP_RATE of the elements (never fewer than one
    allowed flip for tiny inputs).
  * End-to-end output: per token, max|gpu - oracle| <= 1e-3 * max|oracle| plus
    one weight step (alpha * scale_x / Q) per flipped code of that token.
"""
from __future__ import annotations

import math
import os

import numpy as np

TIE_TOL = 2e-3      # code units; fp32 reordering errors are ~1e-5 of a code
FLIP_RATE = 1e-4    # at most this fraction of codes may differ (by one)
OUT_RTOL = 1e-3     # max relative error of the fp32 output (normwise per token)
SQRT7 = np.float32(math.sqrt(7.0))


def q_of(mode: int) -> np.float32:
    return np.float32(127.0) if mode == 0 else SQRT7


def check_codes(gpu: np.ndarray, ora: np.ndarray, shadow: np.ndarray, label: str = "") -> int:
    """Assert the near-tie rule; return the number of flipped codes."""
    gpu = gpu.astype(np.int32)
    ora = ora.astype(np.int32)
    d = gpu - ora
    flips = np.nonzero(d)
    nflip = len(flips[0])
    worst = 0.0
    if nflip:
        assert np.abs(d).max() == 1, f"{label}: a code differs by {np.abs(d).max()}"
        boundary = (gpu[flips] + ora[flips]) / 2.0
        dist = np.abs(shadow[flips] - boundary)
        worst = float(dist.max())
        assert worst <= TIE_TOL, f"{label}: a flipped code is {worst:.3g} code units from its rounding tie"
    log = os.environ.get("BITNET_PARITY_LOG")  # optional record of every comparison: label, codes, flips, worst
    if log:
        with open(log, "a") as f:
            f.write(f"{label}\t{gpu.size}\t{nflip}\t{worst:.3e}\n")
    allowed = max(1, int(math.floor(FLIP_RATE * gpu.size)))
    assert nflip <= allowed, f"{label}: {nflip} flipped codes of {gpu.size} (allowed {allowed})"
    return nflip


def check_out_same_codes(gpu_out: np.ndarray, ref_out: np.ndarray, label: str = "") -> None:
    """Output computed from identical codes and identical per-token scales: the
    accumulators are exact and f = (alpha * s) / Q, out = (float)acc * f are single
    IEEE roundings in the same order on both sides, so the outputs are identical."""
    bad = np.nonzero(gpu_out != ref_out)
    assert len(bad[0]) == 0, (f"{label}: {len(bad[0])} outputs differ from the oracle's dequant of the exact "
                              f"accumulators, first at {tuple(int(b[0]) for b in bad)}")


def scale_rtol(K: int, mode: int) -> float:
    """Bound on |s_gpu - s_oracle| / s_oracle for the per-token scale (gamma or beta).

    Both sides sum the K positive squares of RMSNorm in fp32: the oracle sequentially
    (relative error <= (K - 1) u), the GPU per thread over at most 128 terms and then
    in a tree (<= (128 + log2 K) u), u = 2^-24.  r = 1/sqrt(mean + eps) halves that
    relative error and adds a few roundings; gamma = max|x r g| inherits it; beta =
    mean|x r g| adds a second K-term sum of positive terms (the plain kernel forms it
    as r times the sum of |x|: the same sum, one rounding moved).  A constant 16 u
    covers the remaining single roundings (divide, add eps, sqrt, reciprocal, two
    products)."""
    u = 2.0 ** -24
    sum_err = (K + 128 + math.log2(K)) * u
    return (0.5 * sum_err if mode == 0 else 1.5 * sum_err) + 16 * u


def check_scale_bound(gpu: np.ndarray, ora: np.ndarray, K: int, mode: int, label: str = "") -> None:
    rel = np.abs(gpu.astype(np.float64) - ora) / np.maximum(np.abs(ora.astype(np.float64)), 1e-30)
    tol = scale_rtol(K, mode)
    assert float(rel.max()) <= tol, f"{label}: per-token scale rel err {float(rel.max()):.3g} > {tol:.3g}"


def check_out_end_to_end(gpu_out, ora_out, gpu_codes, ora_codes, ora_scale, alpha, mode, label=""):
    """Normwise per-token bound, widened by one weight step per flipped code."""
    flips = (gpu_codes != ora_codes).sum(axis=1)
    step = np.float64(alpha) * ora_scale.astype(np.float64) / float(q_of(mode))
    err = np.abs(gpu_out.astype(np.float64) - ora_out).max(axis=1)
    ref = np.abs(ora_out).max(axis=1)
    bound = OUT_RTOL * ref + flips * step * 1.001 + 1e-30
    bad = np.nonzero(err > bound)[0]
    assert len(bad) == 0, (f"{label}: token {bad[0]} err {err[bad[0]]:.3g} > bound {bound[bad[0]]:.3g} "
                           f"(flips {flips[bad[0]]})")
    assert float((err / np.maximum(ref, 1e-30)).max()) <= OUT_RTOL + float((flips * step / np.maximum(ref, 1e-30)).max())


def bf16_bits(t):
    """uint16 bit patterns of a bf16 torch tensor (on any device)."""
    return t.detach().contiguous().view(__import__("torch").int16).cpu().numpy().view(np.uint16)


def bf16_values(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32)


def check_out_end_to_end_bf16(gpu_bits, ora_out, gpu_codes, ora_codes, ora_scale, alpha, mode, label=""):
    """The fp32 bound of check_out_end_to_end plus the bf16 rounding of each element
    (at most half a bf16 step, 2^-9 of the value, taken as 2^-8 of the oracle's)."""
    g = bf16_values(gpu_bits).astype(np.float64)
    flips = (gpu_codes != ora_codes).sum(axis=1)
    step = np.float64(alpha) * ora_scale.astype(np.float64) / float(q_of(mode))
    ref = np.abs(ora_out).max(axis=1)
    bound = (OUT_RTOL * ref + flips * step * 1.001)[:, None] + 2.0 ** -8 * np.abs(ora_out) + 1e-30
    bad = np.argwhere(np.abs(g - ora_out) > bound)
    assert len(bad) == 0, f"{label}: element {tuple(bad[0])} outside the bf16 end-to-end bound"

