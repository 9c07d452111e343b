"""The producer of X with the smoothing folded in: RMS normalization fused with
per-token quantization (sq_rmsnorm_quantize_act), against the CPU oracle.

Bar: codes and per-token scales bit for bit ("Weight-Activation Quantization"
§3 "Step 1" and the grasp.study lesson §2: the smoothing moves offline into
the producer; the normalization's sum of squares is exact, so nothing is left
to rounding order).
"""
import numpy as np
import pytest
import torch

import oracle
from w8a8_smoothquant_int8_02_b200 import ops, synth

from _gpu_util import dev, host, ulp_distance

pytestmark = pytest.mark.gpu


def _rows(M, K, seed):
    x = synth.random_floats((M, K), seed=seed, std=1.0)
    g = np.random.default_rng(seed)
    if K > 16:
        x[:, g.choice(K, size=max(1, K // 100), replace=False)] *= 60.0   # outlier channels
    if M > 3:
        x[1] = 0.0                                     # an all-zero row
        x[2] *= 2.0 ** -120                            # bf16 subnormals and tiny normals
        x[3, :] = 2.0 ** -60                           # far below the row's largest ...
        x[3, 0] = 2.0 ** 20                            # ... so those squares drop out
    if M > 5:
        x[4] *= 2.0 ** 100                             # large magnitudes
        x[5, ::7] = -0.0                               # signed zeros
    if M > 6:
        x[6] = g.standard_normal(K) * 2.0 ** -131      # a row of bf16 subnormals only
    if M > 7:
        x[7, 1::2] *= 2.0 ** -20                       # half the row 20 binades down
    return synth.to_bf16_bits(x)


@pytest.mark.parametrize("M,K", [(1, 8), (7, 64), (37, 4096), (300, 1000), (64, 16384),
                                 (2049, 512)])
@pytest.mark.parametrize("qt", ["i8", "e4m3"])
@pytest.mark.parametrize("eps", [1e-6, 1e-2])
def test_rmsnorm_quantize_matches_oracle(M, K, qt, eps):
    xb = _rows(M, K, seed=M + K)
    gamma = synth.random_floats(K, seed=K, lo=0.3, hi=2.5)
    gamma[::5] *= -1.0                                 # negative gains too
    q_ref, s_ref, _, xn_ref = oracle.rmsnorm_quantize_act(
        xb, gamma, eps, oracle.INT8 if qt == "i8" else oracle.E4M3)
    # both forms: the plain one (which also writes xn) and the streaming one
    want_xn = eps == 1e-6
    out = ops.rmsnorm_quantize_act(dev(xb), dev(gamma), eps, qt, want_xn=want_xn)
    assert ops.device_status() == ops.SQ_OK
    np.testing.assert_array_equal(host(out[1]), s_ref)
    np.testing.assert_array_equal(host(out[0]).view(np.uint8), q_ref.view(np.uint8))
    if want_xn:                  # bit patterns: signed zeros included
        np.testing.assert_array_equal(host(out[2]).view(np.uint32), xn_ref.view(np.uint32))


@pytest.mark.parametrize("qt", ["i8", "e4m3"])
def test_folded_producer_feeds_the_layer(qt):
    """Offline, all on the GPU: the normalization's output of the calibration
    tokens, its per-channel max, s, the quantized weights, 1/s folded into the
    gain; at runtime the fused normalization + quantization, then the 8-bit
    GEMM. Every stage equals the oracle's chain bit for bit (the FP8 GEMM
    within its accumulation bound)."""
    M, K, N = 256, 1024, 512
    xb = _rows(M, K, seed=91)
    xcal = _rows(128, K, seed=94)
    gamma = synth.random_floats(K, seed=92, lo=0.5, hi=2.0)
    w = synth.random_floats((K, N), seed=93, std=0.02)
    qcode = oracle.INT8 if qt == "i8" else oracle.E4M3
    eps = 1e-5
    p = ops.prepare_rmsnorm(dev(w), dev(xcal), dev(gamma), eps, 0.5, qt)
    _, _, _, xn_cal = oracle.rmsnorm_quantize_act(xcal, gamma, eps)
    ax_ref = oracle.amax(xn_cal, True)
    np.testing.assert_array_equal(host(p["amax_x"]), ax_ref)
    s_ref = oracle.smooth_factors(ax_ref, oracle.amax(w, False), 0.5)
    assert ulp_distance(host(p["s"]), s_ref).max() <= 2      # pow: libm vs the GPU's
    s = host(p["s"])       # each later stage on the same inputs (no cascade of that ulp)
    g_ref = oracle.fold_smoothing(gamma, s)[0]
    wq_ref, sw_ref = oracle.quantize_weight(w, s, qcode)
    q_ref, sx_ref, _, _ = oracle.rmsnorm_quantize_act(xb, g_ref, eps, qcode)
    np.testing.assert_array_equal(host(p["g"]), g_ref)
    np.testing.assert_array_equal(host(p["wq"]).view(np.uint8), wq_ref.view(np.uint8))
    np.testing.assert_array_equal(host(p["sw"]), sw_ref)
    xq, sx = ops.rmsnorm_quantize_act(dev(xb), p["g"], eps, qt)
    np.testing.assert_array_equal(host(sx), sx_ref)
    np.testing.assert_array_equal(host(xq).view(np.uint8), q_ref.view(np.uint8))
    if qt == "i8":
        y = ops.gemm_w8a8(xq, sx, p["wq"], p["sw"], out_dtype=torch.float32)
        y_ref, _ = oracle.epilogue(oracle.gemm_i8(q_ref, wq_ref), sx_ref, sw_ref, None)
        np.testing.assert_array_equal(host(y), y_ref)
    assert ops.device_status() == ops.SQ_OK


def test_rmsnorm_quantize_validation():
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    g = torch.ones(64, dtype=torch.float32, device="cuda")
    with pytest.raises(ops.SQError):
        ops.rmsnorm_quantize_act(x, g, 0.0)                      # eps must be > 0
    with pytest.raises(ops.SQError):
        ops.rmsnorm_quantize_act(x[:, :60].contiguous(), g[:60].contiguous(), 1e-6)  # K % 8
    big = torch.zeros((1, 16392), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ops.SQError):
        ops.rmsnorm_quantize_act(big, torch.ones(16392, device="cuda"), 1e-6)   # K > 16384
    xq, sx = ops.rmsnorm_quantize_act(x[:0], g, 1e-6)             # empty batch
    assert xq.shape == (0, 64) and sx.shape == (0,)


@pytest.mark.parametrize("force_exact", [False, True])
@pytest.mark.parametrize("qt", ["i8", "e4m3"])
def test_many_rows_sum_paths(force_exact, qt, monkeypatch):
    """Many rows (the one-warp-per-row form): its binary64 sum of squares with
    the interval check, which falls back to the exact integer sum for the
    rows whose r it cannot settle (about one in a few thousand here), and the
    exact sum for every row (SQ_NORM_EXACT_SUM=1); both bit-exact."""
    if force_exact:
        monkeypatch.setenv("SQ_NORM_EXACT_SUM", "1")
    M, K = 20000, 256
    xb = _rows(M, K, seed=4242)
    gamma = synth.random_floats(K, seed=4243, lo=0.3, hi=2.5)
    q_ref, s_ref, _, _ = oracle.rmsnorm_quantize_act(
        xb, gamma, 1e-5, oracle.INT8 if qt == "i8" else oracle.E4M3)
    xq, sx = ops.rmsnorm_quantize_act(dev(xb), dev(gamma), 1e-5, qt)
    assert ops.device_status() == ops.SQ_OK
    np.testing.assert_array_equal(host(sx), s_ref)
    np.testing.assert_array_equal(host(xq).view(np.uint8), q_ref.view(np.uint8))



@pytest.mark.parametrize("M,K", [(37, 4096), (300, 1000), (64, 16384), (511, 8192)])
def test_block_form_exact_sum_path(M, K, monkeypatch):
    """The one-CTA-per-row form (fewer rows, or rows above 8192 elements) with
    the exact integer sum forced for every row (SQ_NORM_EXACT_SUM=1), and
    with its binary64 sum; both bit-exact against the oracle."""
    xb = _rows(M, K, seed=M * 7 + K)
    gamma = synth.random_floats(K, seed=K + 11, lo=0.3, hi=2.5)
    q_ref, s_ref, _, _ = oracle.rmsnorm_quantize_act(xb, gamma, 1e-5)
    for force in ("1", "0"):
        monkeypatch.setenv("SQ_NORM_EXACT_SUM", force)
        xq, sx = ops.rmsnorm_quantize_act(dev(xb), dev(gamma), 1e-5, "i8")
        assert ops.device_status() == ops.SQ_OK
        np.testing.assert_array_equal(host(sx), s_ref)
        np.testing.assert_array_equal(host(xq).view(np.uint8), q_ref.view(np.uint8))


@pytest.mark.parametrize("M,K", [(700, 8192), (1500, 2048), (600, 4096), (900, 24)])
@pytest.mark.parametrize("qt", ["i8", "e4m3"])
def test_warp_form_row_lengths(M, K, qt):
    """The one-warp-per-row form at row lengths with the gains in shared memory
    (up to 4096) and from L1 (above), bit-exact against the oracle."""
    xb = _rows(M, K, seed=M + 3 * K)
    gamma = synth.random_floats(K, seed=K + 17, lo=0.3, hi=2.5)
    gamma[1::3] *= -1.0
    q_ref, s_ref, _, _ = oracle.rmsnorm_quantize_act(
        xb, gamma, 1e-5, oracle.INT8 if qt == "i8" else oracle.E4M3)
    xq, sx = ops.rmsnorm_quantize_act(dev(xb), dev(gamma), 1e-5, qt)
    assert ops.device_status() == ops.SQ_OK
    np.testing.assert_array_equal(host(sx), s_ref)
    np.testing.assert_array_equal(host(xq).view(np.uint8), q_ref.view(np.uint8))


def _sweep_cases(n=24, seed=77):
    g = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        K = int(g.choice([8, 16, 24, 64, 200, 1000, 2048, 4096, 4104, 8192, 12288, 16384]))
        M = int(g.integers(1, max(2, min(5000, 8_000_000 // K))))
        cases.append((i, M, K, bool(g.integers(0, 2)), float(g.choice([1e-6, 1e-5, 0.1]))))
    return cases


@pytest.mark.parametrize("i,M,K,e4m3,eps", _sweep_cases())
def test_seeded_shape_sweep(i, M, K, e4m3, eps):
    """Seeded random shapes across every form (plain when xn is asked for,
    one warp per row, one CTA per row) and both code types."""
    xb = _rows(M, K, seed=1000 + i)
    gamma = synth.random_floats(K, seed=2000 + i, lo=0.2, hi=3.0)
    qt = "e4m3" if e4m3 else "i8"
    q_ref, s_ref, _, xn_ref = oracle.rmsnorm_quantize_act(
        xb, gamma, eps, oracle.E4M3 if e4m3 else oracle.INT8)
    out = ops.rmsnorm_quantize_act(dev(xb), dev(gamma), eps, qt, want_xn=(i % 4 == 0))
    assert ops.device_status() == ops.SQ_OK
    np.testing.assert_array_equal(host(out[1]), s_ref)
    np.testing.assert_array_equal(host(out[0]).view(np.uint8), q_ref.view(np.uint8))
    if i % 4 == 0:
        np.testing.assert_array_equal(host(out[2]).view(np.uint32), xn_ref.view(np.uint32))


@pytest.mark.parametrize("qt", ["i8", "e4m3"])
def test_rmsnorm_layer_api(qt):
    """The layer object: its offline preparation and forward equal the oracle's
    chain (calibration on the normalization's output, s, weight codes, the
    folded gain, the fused normalization + quantization, the GEMM)."""
    M, K, N = 300, 1024, 768
    h = _rows(M, K, seed=501)
    h_cal = _rows(256, K, seed=502)
    gamma = synth.random_floats(K, seed=503, lo=0.5, hi=2.0)
    w = synth.random_floats((K, N), seed=504, std=0.02)
    bias = synth.to_bf16_bits(synth.random_floats(N, seed=505, std=0.01))
    qcode = oracle.INT8 if qt == "i8" else oracle.E4M3
    layer = ops.RMSNormSmoothQuantLinear(dev(w), dev(h_cal), dev(gamma), 1e-5, 0.5, qt,
                                         bias=dev(bias))
    s = host(layer.s)          # stage-wise: the later stages on the layer's own s
    xn_cal = oracle.rmsnorm_quantize_act(h_cal, gamma, 1e-5)[3]
    s_ref = oracle.smooth_factors(oracle.amax(xn_cal, True), oracle.amax(w, False), 0.5)
    assert ulp_distance(s, s_ref).max() <= 2
    g_ref = oracle.fold_smoothing(gamma, s)[0]
    np.testing.assert_array_equal(host(layer.g), g_ref)
    wq_ref, sw_ref = oracle.quantize_weight(w, s, qcode)
    q_ref, sx_ref, _, _ = oracle.rmsnorm_quantize_act(h, g_ref, 1e-5, qcode)
    y = layer(dev(h), out_dtype=torch.float32)
    assert ops.device_status() == ops.SQ_OK
    if qt == "i8":
        y_ref, _ = oracle.epilogue(oracle.gemm_i8(q_ref, wq_ref), sx_ref, sw_ref, bias)
        np.testing.assert_array_equal(host(y), y_ref)
    else:
        y_ref, _ = oracle.epilogue(oracle.gemm_e4m3(q_ref, wq_ref), sx_ref, sw_ref, bias)
        err = np.abs(host(y).astype(np.float64) - y_ref)
        scale = (np.abs(oracle.e4m3_decode(q_ref)).astype(np.float64) @
                 np.abs(oracle.e4m3_decode(wq_ref)).astype(np.float64).T) * sx_ref[:, None] * sw_ref[None, :]
        assert (err <= 1e-3 * (scale + np.abs(oracle.bf16_to_f32_array(bias))[None, :]) + 1e-30).all()
