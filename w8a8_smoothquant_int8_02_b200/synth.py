"""Seeded synthetic inputs for the SmoothQuant W8A8 linear layer.

This module only draws random numbers; it holds none of the layer's
arithmetic, so both the CUDA path and the CPU oracle can be fed from it.

Recipe (the pages describe transformer activations with a few outlier
channels 10-100x larger than the rest -- "Weight-Activation Quantization" §2
"The Problem: Activation Outliers" -- and roughly Gaussian weights):

* numpy ``Generator(PCG64(SeedSequence(seed)))``; seven independent child
  streams, spawned in this order: outlier-channel set, outlier factors, X,
  X_cal, W, bias, the normalization's gain.
* A layer fed by an RMS normalization (``norm_eps`` > 0): X and X_cal are the
  normalization's input, drawn as above; its gain gamma ~ U(0.5, 2.0) per
  channel in float32.
* X, X_cal ~ N(0, 1) in float32. A fixed set of input channels (the first
  ``round(p*K)`` entries of a seeded permutation of K, or an explicit list) is
  multiplied by one factor per channel drawn from U(lo, hi); the same channels
  and factors apply to X and to the calibration batch X_cal.
* W ~ N(0, w_std) in float32, bias ~ N(0, bias_std).
* bf16 tensors are the float32 draws rounded to nearest-even, returned as raw
  uint16 bit patterns (numpy has no bfloat16).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> raw bf16 bit patterns (uint16), round-to-nearest-even."""
    t = torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


@dataclass
class LinearCase:
    name: str
    M: int
    K: int
    N: int
    x_dtype: str                 # "f32" or "bf16"
    alpha: float
    qtype: str                   # "i8" or "e4m3"; weight-only: "w8" / "w4"
    w_std: float
    outlier_frac: float = 0.01
    outlier_lo: float = 20.0
    outlier_hi: float = 100.0
    outlier_channels: tuple = ()  # explicit list overrides outlier_frac
    outlier_factor: float = 0.0   # fixed factor for an explicit list
    bias_std: float = 0.0         # 0 => no bias
    cal_tokens: int = 512         # 0 => calibrate on X itself
    act_scaling: str = "token"    # "token" (per-token), "tensor" (per-tensor, delayed), "none"
    smooth: bool = True           # False => no smoothing factors (plain FP8 / INT8)
    norm_eps: float = 0.0         # > 0 => X comes from an RMS normalization (this eps)
    seed: int = 0
    note: str = field(default="")

    @property
    def ops(self) -> int:
        return 2 * self.M * self.N * self.K


def generate(case: LinearCase, M: int | None = None) -> dict:
    """Draw X [M,K], X_cal, W [K,N] and the optional bias for ``case``.

    ``M`` overrides the token count (the rows are the first M of the stream
    only when M equals case.M; other M values give a different but equally
    seeded draw)."""
    M = case.M if M is None else M
    K, N = case.K, case.N
    ss = np.random.SeedSequence(case.seed)
    st_set, st_fac, st_x, st_cal, st_w, st_b, st_g = ss.spawn(7)
    if case.outlier_channels:
        ch = np.array(sorted(case.outlier_channels), np.int64)
        fac = np.full(ch.size, case.outlier_factor, np.float32)
    else:
        n_out = int(round(case.outlier_frac * K))
        perm = np.random.Generator(np.random.PCG64(st_set)).permutation(K)
        ch = np.sort(perm[:n_out]).astype(np.int64)
        fac = np.random.Generator(np.random.PCG64(st_fac)).uniform(
            case.outlier_lo, case.outlier_hi, size=ch.size).astype(np.float32)
    gx = np.random.Generator(np.random.PCG64(st_x))
    x = gx.standard_normal((M, K), dtype=np.float32)
    x[:, ch] *= fac
    if case.cal_tokens:
        gc = np.random.Generator(np.random.PCG64(st_cal))
        x_cal = gc.standard_normal((case.cal_tokens, K), dtype=np.float32)
        x_cal[:, ch] *= fac
    else:
        x_cal = x
    gw = np.random.Generator(np.random.PCG64(st_w))
    w = gw.standard_normal((K, N), dtype=np.float32) * np.float32(case.w_std)
    bias = None
    if case.bias_std:
        gb = np.random.Generator(np.random.PCG64(st_b))
        bias = to_bf16_bits(gb.standard_normal(N, dtype=np.float32)
                            * np.float32(case.bias_std))
    if case.x_dtype == "bf16":
        x = to_bf16_bits(x)
        x_cal = to_bf16_bits(x_cal) if case.cal_tokens else x
        w = to_bf16_bits(w)
    gamma = None
    if case.norm_eps:
        gamma = np.random.Generator(np.random.PCG64(st_g)).uniform(
            0.5, 2.0, size=K).astype(np.float32)
    return dict(x=x, x_cal=x_cal, w=w, bias=bias, gamma=gamma, outlier_channels=ch,
                outlier_factors=fac)


def random_matrix(shape, dtype, seed: int, lo: int = -127, hi: int = 127) -> np.ndarray:
    """Seeded integer / code matrix for stage-wise tests (uniform in [lo, hi])."""
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed)))
    return g.integers(lo, hi + 1, size=shape).astype(dtype)


def random_floats(shape, seed: int, std: float = 1.0, lo: float | None = None,
                  hi: float | None = None) -> np.ndarray:
    """Seeded float32 matrix: N(0,std), or U(lo,hi) when both bounds given."""
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed)))
    if lo is not None and hi is not None:
        return g.uniform(lo, hi, size=shape).astype(np.float32)
    return g.standard_normal(shape, dtype=np.float32) * np.float32(std)
