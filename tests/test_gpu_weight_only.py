"""Weight-only quantized GEMM (W8A16 / W4A16) against the CPU oracle.

The pages' weight-only schemes: "Weight-Activation Quantization"
(infra.bea.ai) §1 table, W4A16 row (INT4 weights dequantized, then a 16-bit
multiply); the zenaique flashcard (weights dequantized on the fly against BF16
activations); the grasp.study lesson §1 / §3 (W8A16). Weight codes and scales
are bit-exact; outputs are within 1e-3 of the binary64 product on the
normalized metric |y - y_ref| / (sw * sum_k |x q| + |bias|), which bounds the
tensor cores' binary32 accumulation of exact products (K * 2^-24 < 1e-3 for
K <= 16384); the bf16 output is the nearest-even rounding of the binary32 one.
"""
import numpy as np
import pytest
import torch

import oracle
from w8a8_smoothquant_int8_02_b200 import ops, synth

from _gpu_util import dev, host, weight_only_error_denominator

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("K,N", [(64, 64), (4096, 256), (96, 8), (256, 1000), (8192, 136)])
def test_quantize_weight_int4(dtype, K, N):
    w = synth.random_floats((K, N), seed=K + 3 * N, std=0.02)
    w[:, 0] = 0.0                         # an all-zero output channel
    w[K // 3, min(1, N - 1)] = 0.3        # a dominant weight
    w = synth.to_bf16_bits(w) if dtype == "bf16" else w
    wq_ref, sw_ref = oracle.quantize_weight_i4(w)
    wq, sw = ops.quantize_weight(dev(w), None, "i4")
    assert ops.device_status() == ops.SQ_OK
    np.testing.assert_array_equal(host(sw), sw_ref)
    np.testing.assert_array_equal(host(wq), wq_ref)


SHAPES = [(1, 8, 32), (5, 136, 1056), (16, 1000, 256), (16, 4096, 8192), (3, 28672, 256),
          (17, 256, 512), (40, 384, 4096), (16, 128, 16384), (16, 2048, 8192),
          (9, 2056, 8256), (16, 28672, 1024)]   # 8256: a partial last stage


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("with_bias", [False, True])
def test_gemm_weight_only(bits, M, N, K, with_bias):
    g = np.random.default_rng(M * 7 + N + K + bits)
    x = (g.standard_normal((M, K)) * 2).astype(np.float32)
    x[:, g.choice(K, size=max(1, K // 100), replace=False)] *= 50.0   # outlier channels
    xb = synth.to_bf16_bits(x)
    w = synth.random_floats((K, N), seed=N + K, std=0.02)
    w[:, -1] = 0.0
    bias = synth.to_bf16_bits(synth.random_floats(N, seed=N, std=0.1)) if with_bias else None
    if bits == 8:
        wq, sw = oracle.quantize_weight(w, None)
        codes = wq
    else:
        wq, sw = oracle.quantize_weight_i4(w)
        codes = oracle.unpack_i4(wq)
    b = None if bias is None else dev(bias)
    yf = ops.gemm_weight_only(dev(xb), dev(wq), dev(sw), b, bits, out_dtype=torch.float32)
    yb = ops.gemm_weight_only(dev(xb), dev(wq), dev(sw), b, bits)
    assert ops.device_status() == ops.SQ_OK
    y_ref = oracle.gemm_weight_only(xb, wq, sw, bias, bits)
    got = host(yf)
    e = np.abs(got.astype(np.float64) - y_ref) / weight_only_error_denominator(xb, codes, sw, bias)
    assert e.max() <= 1e-3, e.max()
    np.testing.assert_array_equal(host(yb), oracle.f32_to_bf16(got))


@pytest.mark.parametrize("bits", [8, 4])
def test_weight_only_extreme_codes_and_one_hot_tokens(bits):
    """Rows of +-max codes and one-hot token rows: each output of a one-hot
    token is one dequantized weight, exact in binary32 (q * sw, one rounding)."""
    K, N = 1024, 256
    qmax = 127 if bits == 8 else 7
    codes = np.full((N, K), qmax, np.int8)
    codes[1::2] = -qmax
    codes[5, :] = 0
    codes[5, 77] = 3
    if bits == 8:
        wq = codes
    else:
        lo = codes[:, 0::2].astype(np.int16) & 0xF
        hi = codes[:, 1::2].astype(np.int16) & 0xF
        wq = (lo | (hi << 4)).astype(np.uint8)
    sw = synth.random_floats(N, seed=9, lo=1e-3, hi=1e-1)
    x = np.zeros((16, K), np.float32)
    x[np.arange(16), np.arange(16) * 61] = 1.0
    x[0, :] = 1.0                                    # a row summing every code
    xb = synth.to_bf16_bits(x)
    y = host(ops.gemm_weight_only(dev(xb), dev(wq), dev(sw), None, bits, out_dtype=torch.float32))
    assert ops.device_status() == ops.SQ_OK
    y_ref = oracle.gemm_weight_only(xb, wq, sw, None, bits)
    np.testing.assert_array_equal(y[1:], y_ref[1:].astype(np.float32))
    np.testing.assert_array_equal(y[0], y_ref[0].astype(np.float32))   # sums of +-q exact
    assert y[0, 0] == np.float32(np.float64(qmax * K) * np.float64(sw[0]))


def test_weight_only_validation():
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    wq = torch.zeros((16, 64), dtype=torch.int8, device="cuda")
    sw = torch.ones(16, dtype=torch.float32, device="cuda")
    x48 = torch.zeros((4, 48), dtype=torch.bfloat16, device="cuda")
    wq48 = torch.zeros((16, 24), dtype=torch.uint8, device="cuda")
    with pytest.raises(ops.SQError):
        ops.gemm_weight_only(x48, wq48, sw, bits=4)                # K not a multiple of 32
    y = ops.gemm_weight_only(x[:0], wq, sw, bits=8)                # empty batch
    assert y.shape == (0, 16)
