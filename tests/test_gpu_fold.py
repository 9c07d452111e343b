"""Offline fold of the activation smoothing into the producer of X on the GPU
against the CPU oracle ("Weight-Activation Quantization" §3: X~ = X diag(1/s)
is part of the offline preparation). The folded parameters bit for bit (both
input types, both axes, 1-D gains, ragged and full-size producer weights,
edge values), then the layer that follows: a gain producer emitting X~
through the folded gain and quantized without s gives the same codes, scales
and output as the unfolded producer quantized with s when s is a power of
two, and the module's fold feeds its own path bit-exactly.
"""
import numpy as np
import pytest
import torch

import oracle
from w8a8_smoothquant_int8_02_b200 import ops, synth

from _gpu_util import dev, host

pytestmark = pytest.mark.gpu


def _p(rows, cols, seed):
    g = np.random.default_rng(seed)
    return (g.standard_normal((rows, cols)) * np.exp(g.uniform(-8, 8, (rows, cols)))).astype(np.float32)


def _bits(a):
    return np.asarray(a, np.float32).view(np.uint32)


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("axis", ["column", "row"])
@pytest.mark.parametrize("rows,cols", [(1, 64), (1, 14336), (37, 208), (300, 1000), (513, 4096)])
def test_fold_parity(bf16, axis, rows, cols):
    p = _p(rows, cols, seed=rows * 7 + cols)
    pin = synth.to_bf16_bits(p) if bf16 else p
    s = synth.random_floats(cols if axis == "column" else rows, seed=rows + cols, lo=0.05, hi=20.0)
    got = ops.fold_smoothing(dev(pin), dev(s), axis)
    want = oracle.fold_smoothing(pin, s, per_column=(axis == "column"))
    np.testing.assert_array_equal(_bits(host(got)), _bits(want))
    assert ops.device_status() == ops.SQ_OK


@pytest.mark.parametrize("axis", ["column", "row"])
def test_fold_one_dimensional_gain(axis):
    K = 4096
    gamma = synth.random_floats(K, seed=71, lo=0.5, hi=2.0)
    s = synth.random_floats(K, seed=72, lo=0.05, hi=20.0)
    got = ops.fold_smoothing(dev(gamma), dev(s), axis)
    assert got.shape == (K,)
    np.testing.assert_array_equal(_bits(host(got)),
                                  _bits(oracle.fold_smoothing(gamma, s, per_column=True)[0]))


@pytest.mark.parametrize("rows,cols,axis", [(4096, 4096, "column"), (4096, 14336, "column"),
                                            (14336, 4096, "row")])
def test_fold_full_size_producer_weights(rows, cols, axis):
    """The producer weights in front of the MLP-up (K = 4096) and MLP-down
    (K = 14336) layers, bf16, in both layouts."""
    g = np.random.default_rng(rows + cols)
    p = synth.to_bf16_bits((g.standard_normal((rows, cols)) * 0.02).astype(np.float32))
    s = synth.random_floats(cols if axis == "column" else rows, seed=73, lo=0.05, hi=20.0)
    got = ops.fold_smoothing(dev(p), dev(s), axis)
    want = oracle.fold_smoothing(p, s, per_column=(axis == "column"))
    np.testing.assert_array_equal(_bits(host(got)), _bits(want))


def test_fold_edge_values():
    """Signed zeros, subnormal quotients, overflow to infinity, power-of-two
    and extreme smoothing factors."""
    K = 64
    p = np.zeros((4, K), np.float32)
    p[0, :8] = [0.0, -0.0, 1e-40, -1e-40, 1e-38, 3e38, -3e38, 1.0]
    p[1] = np.float32(2.0) ** np.arange(-60, 68, 2).astype(np.float32)
    p[2] = -p[1]
    p[3] = np.linspace(-1000, 1000, K).astype(np.float32)
    s = synth.random_floats(K, seed=74, lo=0.05, hi=20.0)
    s[:8] = [1.0, 2.0, 0.5, 3.0, 2.0 ** 30, 2.0 ** -30, 2.0 ** -30, 2.0 ** -126]
    s[8:12] = [2.0 ** 40, 2.0 ** -40, 7.0, 1e-30]
    got = host(ops.fold_smoothing(dev(p), dev(s), "column"))
    want = oracle.fold_smoothing(p, s, per_column=True)
    np.testing.assert_array_equal(_bits(got), _bits(want))
    assert np.isinf(want[0, 5]) and want[0, 2] != 0 and np.signbit(want[0, 1])


def test_fold_empty_is_a_no_op():
    p = torch.empty((0, 64), dtype=torch.float32, device="cuda")
    s = torch.ones(64, dtype=torch.float32, device="cuda")
    assert ops.fold_smoothing(p, s, "column").shape == (0, 64)


@pytest.mark.parametrize("qtype", ["i8", "e4m3"])
def test_folded_gain_producer_matches_unfolded_for_power_of_two_s(qtype):
    """The producer's output x * gamma, in bf16: folded (gamma / s, then the
    layer without s) and unfolded (gamma, then the layer divides by s) are the
    same numbers when s is a power of two, so codes, scales and Y agree bit
    for bit. torch's elementwise product stands in for the producer."""
    M, K, N = 300, 1024, 256
    g = np.random.default_rng(75)
    x = dev(synth.to_bf16_bits(g.standard_normal((M, K)).astype(np.float32)))
    gamma = dev(synth.random_floats(K, seed=76, lo=0.5, hi=2.0))
    s = dev(np.ldexp(np.ones(K), g.integers(-4, 8, K)).astype(np.float32))
    w = dev(synth.to_bf16_bits((g.standard_normal((K, N)) * 0.02).astype(np.float32)))
    wq, sw = ops.quantize_weight(w, s, qtype)
    x_unfolded = (x.float() * gamma).to(torch.bfloat16)
    x_folded = (x.float() * ops.fold_smoothing(gamma, s)).to(torch.bfloat16)
    q1, sx1 = ops.quantize_act(x_unfolded, s, qtype)
    q2, sx2 = ops.quantize_act(x_folded, None, qtype)
    assert torch.equal(q1.view(torch.uint8), q2.view(torch.uint8))
    assert torch.equal(sx1, sx2)
    y1 = ops.linear(x_unfolded, s, wq, sw, None, qtype)
    y2 = ops.linear(x_folded, None, wq, sw, None, qtype)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    assert ops.device_status() == ops.SQ_OK


def test_module_fold_smoothing_into():
    """SmoothQuantLinear folds its 1/s into the producer's gain once, then
    takes X~ without dividing: its output equals the oracle's layer on the
    same X~ with s = NULL, and a second fold is refused."""
    from w8a8_smoothquant_int8_02_b200.ops import SmoothQuantLinear
    M, K, N = 256, 512, 384
    g = np.random.default_rng(77)
    xn = g.standard_normal((M, K)).astype(np.float32)
    xn[:, [3, 100, 400]] *= 40
    x_cal = dev(synth.to_bf16_bits(xn[:128]))
    w = dev(synth.to_bf16_bits((g.standard_normal((K, N)) * 0.02).astype(np.float32)))
    layer = SmoothQuantLinear(w, x_cal, alpha=0.5, qtype="i8")
    s = host(layer.s)
    gamma = synth.random_floats(K, seed=78, lo=0.5, hi=2.0)
    gamma_f = layer.fold_smoothing_into(dev(gamma))
    assert layer.s is None and np.array_equal(host(layer.folded_s), s)
    np.testing.assert_array_equal(_bits(host(gamma_f)), _bits(oracle.fold_smoothing(gamma, s)[0]))
    x_t = (dev(synth.to_bf16_bits(xn)).float() * gamma_f).to(torch.bfloat16)
    y = layer(x_t)
    ref = oracle.linear(host(x_t), None, host(layer.wq), host(layer.sw), None, oracle.INT8)
    np.testing.assert_array_equal(host(y), ref["y_bf16"])
    with pytest.raises(RuntimeError):
        layer.fold_smoothing_into(dev(gamma))
    assert ops.device_status() == ops.SQ_OK
