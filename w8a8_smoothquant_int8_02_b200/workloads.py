"""The linear-layer workloads this library is measured on: five per-token
SmoothQuant cases, one per-tensor FP8 case, the two weight-only schemes
(W8A16, W4A16) at the decode shape, and the MLP up-projection fed by an RMS
normalization with the smoothing folded into its gain.

Shapes follow transformer linear layers: Y[M,N] = X[M,K] W[K,N], M tokens,
K input channels, N output channels.  Prefill / MLP shapes are compute-bound
and run on the 8-bit tensor cores; the 16-token decode shape is bound by the
weight read from HBM ("W8A8 vs W4A16": prefill is compute-bound, decode is
memory-bound).
"""
from __future__ import annotations

from .synth import LinearCase

TINY = LinearCase(
    name="tiny_16x64x64", M=16, K=64, N=64, x_dtype="f32", alpha=0.5,
    qtype="i8", w_std=0.02, outlier_channels=(3, 41), outlier_factor=60.0,
    cal_tokens=0,
    note="X fp32 [16,64] N(0,1), channels 3 and 41 x60; W fp32 [64,64] "
         "N(0,0.02); calibrated on X itself")

PREFILL = LinearCase(
    name="prefill_512x4096x4096", M=512, K=4096, N=4096, x_dtype="bf16",
    alpha=0.5, qtype="i8", w_std=0.02, outlier_frac=0.01, outlier_lo=20.0,
    outlier_hi=100.0, cal_tokens=512,
    note="X bf16 [512,4096], 1% outlier channels x U(20,100); W bf16 "
         "[4096,4096] N(0,0.02); 512 calibration tokens")

MLP_UP = LinearCase(
    name="mlp_up_4096x4096x14336", M=4096, K=4096, N=14336, x_dtype="bf16",
    alpha=0.5, qtype="i8", w_std=0.02, outlier_frac=0.01, outlier_lo=20.0,
    outlier_hi=100.0, bias_std=0.01, cal_tokens=512,
    note="X bf16 [4096,4096], 1% outlier channels x U(20,100); W bf16 "
         "[4096,14336] N(0,0.02); bias bf16 N(0,0.01); 512 calibration tokens")

FP8_DOWN = LinearCase(
    name="fp8_down_4096x14336x4096", M=4096, K=14336, N=4096, x_dtype="bf16",
    alpha=0.85, qtype="e4m3", w_std=0.015, outlier_frac=0.005,
    outlier_lo=10.0, outlier_hi=80.0, cal_tokens=512,
    note="X bf16 [4096,14336], 0.5% outlier channels x U(10,80); W bf16 "
         "[14336,4096] N(0,0.015); alpha 0.85; E4M3 with amax/448 scales")

DECODE = LinearCase(
    name="decode_16x8192x28672", M=16, K=8192, N=28672, x_dtype="bf16",
    alpha=0.5, qtype="i8", w_std=0.02, outlier_frac=0.01, outlier_lo=20.0,
    outlier_hi=100.0, cal_tokens=512,
    note="X bf16 [16,8192], 1% outlier channels x U(20,100); W bf16 "
         "[8192,28672] N(0,0.02) quantized offline; HBM-bound")

FP8_TENSOR = LinearCase(
    name="fp8_tensor_4096x4096x14336", M=4096, K=4096, N=14336, x_dtype="bf16",
    alpha=0.5, qtype="e4m3", w_std=0.02, outlier_frac=0.01, outlier_lo=20.0,
    outlier_hi=100.0, bias_std=0.01, cal_tokens=512, act_scaling="tensor", smooth=False,
    note="the MLP-up shape in native FP8: no smoothing, one E4M3 scale for the whole "
         "activation tensor from the previous step's max (delayed scaling; the first "
         "step's from the 512 calibration tokens), per-output-channel E4M3 weights")

# The weight-only schemes the pages set against W8A8 at decode (W8A16, W4A16):
# bf16 activations as they are, per-output-channel INT8 / INT4 weights, the
# decode shape above. Bound by the weight read from HBM.
DECODE_W8A16 = LinearCase(
    name="decode_w8a16_16x8192x28672", M=16, K=8192, N=28672, x_dtype="bf16",
    alpha=0.5, qtype="w8", w_std=0.02, outlier_frac=0.01, outlier_lo=20.0,
    outlier_hi=100.0, cal_tokens=0, act_scaling="none", smooth=False,
    note="weight-only W8A16: X bf16 [16,8192], 1% outlier channels x U(20,100), not "
         "quantized; W bf16 [8192,28672] N(0,0.02) as per-channel INT8 codes; HBM-bound")

DECODE_W4A16 = LinearCase(
    name="decode_w4a16_16x8192x28672", M=16, K=8192, N=28672, x_dtype="bf16",
    alpha=0.5, qtype="w4", w_std=0.02, outlier_frac=0.01, outlier_lo=20.0,
    outlier_hi=100.0, cal_tokens=0, act_scaling="none", smooth=False,
    note="weight-only W4A16: X bf16 [16,8192], 1% outlier channels x U(20,100), not "
         "quantized; W bf16 [8192,28672] N(0,0.02) as per-channel INT4 codes packed two per "
         "byte; HBM-bound")

# The MLP up-projection with its producer: X is the output of the layer's RMS
# normalization, 1/s is folded into the normalization's gain offline, and one
# kernel normalizes and quantizes each token row (the pages' "offline, no
# runtime overhead" smoothing made literal).
MLP_UP_RMSNORM = LinearCase(
    name="mlp_up_rmsnorm_4096x4096x14336", M=4096, K=4096, N=14336, x_dtype="bf16",
    alpha=0.5, qtype="i8", w_std=0.02, outlier_frac=0.01, outlier_lo=20.0,
    outlier_hi=100.0, bias_std=0.01, cal_tokens=512, norm_eps=1e-5,
    note="the MLP-up shape fed by an RMS normalization: its input X bf16 [4096,4096] with 1% "
         "outlier channels x U(20,100), gain U(0.5,2), eps 1e-5; calibration on the "
         "normalization's output of 512 tokens; W bf16 [4096,14336] N(0,0.02); bias bf16 "
         "N(0,0.01)")

ALL = {c.name: c for c in (TINY, PREFILL, MLP_UP, FP8_DOWN, DECODE, FP8_TENSOR, DECODE_W8A16,
                           DECODE_W4A16, MLP_UP_RMSNORM)}
WEIGHT_ONLY_BITS = {"w8": 8, "w4": 4}   # qtype of a weight-only workload -> weight bits
