"""Pins for the CPU oracle: checks against what the pages print and what the
mathematics fixes, never against the oracle's own formulas retyped.

Pages: "Weight-Activation Quantization" (infra.bea.ai) §2 (per-tensor scale
80/127), §3 (worked smoothing example, smoothing-factor formula), §4 (E4M3
range and scaling).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from w8a8_smoothquant_int8_02_b200 import synth, workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _fixture(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split(":", 1)
            out[k.strip()] = v.split()
    return out


def _f32_dot(a, b):
    """Sequential binary32 dot product."""
    acc = np.float32(0.0)
    for x, y in zip(np.asarray(a, np.float32), np.asarray(b, np.float32)):
        acc = np.float32(acc + np.float32(x * y))
    return acc


# ---------------------------------------------------------------------------
# §3 worked example: smoothing preserves the inner product.
# ---------------------------------------------------------------------------

def test_worked_example_smoothing_values():
    fx = _fixture("worked_example.txt")
    x = np.array([fx["x"]], np.float32)
    w = np.array(fx["w"], np.float32).reshape(3, 1)
    s = np.array(fx["s"], np.float32)
    xs = oracle.smooth_act(x, s)[0]
    ws = oracle.smooth_weight(w, s)[:, 0]
    np.testing.assert_array_equal(xs, np.array(fx["x_smoothed"], np.float32))
    np.testing.assert_array_equal(ws, np.array(fx["w_smoothed"], np.float32))


def test_worked_example_inner_product_preserved():
    fx = _fixture("worked_example.txt")
    x = np.array([fx["x"]], np.float32)
    w = np.array(fx["w"], np.float32).reshape(3, 1)
    s = np.array(fx["s"], np.float32)
    xs = oracle.smooth_act(x, s)[0]
    ws = oracle.smooth_weight(w, s)[:, 0]
    target = float(fx["inner_product"][0])
    before = _f32_dot(x[0], w[:, 0])
    after = _f32_dot(xs, ws)
    assert abs(float(before) - target) < 1e-5
    # s is a power of two, so every product is unchanged and the binary32
    # sums agree bit for bit.
    assert before == after


def test_power_of_two_smoothing_is_exact_on_random_rows():
    rng = np.random.default_rng(5)
    K = 97
    x = rng.standard_normal((3, K)).astype(np.float32)
    w = rng.standard_normal((K, 4)).astype(np.float32)
    s = (2.0 ** rng.integers(-6, 7, size=K)).astype(np.float32)
    xs = oracle.smooth_act(x, s)
    ws = oracle.smooth_weight(w, s)
    for m in range(3):
        for n in range(4):
            assert _f32_dot(x[m], w[:, n]) == _f32_dot(xs[m], ws[:, n])


def test_general_smoothing_preserves_product_within_rounding():
    rng = np.random.default_rng(6)
    K = 256
    x = rng.standard_normal((4, K)).astype(np.float32)
    w = rng.standard_normal((K, 5)).astype(np.float32)
    s = rng.uniform(0.05, 20.0, size=K).astype(np.float32)
    xs = oracle.smooth_act(x, s).astype(np.float64)
    ws = oracle.smooth_weight(w, s).astype(np.float64)
    exact = x.astype(np.float64) @ w.astype(np.float64)
    smoothed = xs @ ws
    # each smoothed product carries two binary32 roundings
    bound = 2.5 * 2.0 ** -24 * (np.abs(x.astype(np.float64)) @ np.abs(w.astype(np.float64)))
    assert np.all(np.abs(smoothed - exact) <= bound)


# ---------------------------------------------------------------------------
# §2 per-tensor scale set by the outlier: 80/127 = 0.63.
# ---------------------------------------------------------------------------

def test_per_tensor_scale_example():
    fx = _fixture("per_tensor_scale.txt")
    row = np.array([fx["row"]], np.float32)
    xq, sx = oracle.quantize_act(row, None)
    assert abs(float(sx[0]) - float(fx["scale_approx"][0])) <= \
        float(fx["scale_rel_tol"][0]) * float(fx["scale_approx"][0])
    np.testing.assert_array_equal(xq[0], np.array(fx["codes"], np.int8))


def test_round_half_even_ties():
    fx = _fixture("rounding_ties.txt")
    row = np.array([fx["row"]], np.float32)
    xq, sx = oracle.quantize_act(row, None)
    assert sx[0] == np.float32(1.0)
    np.testing.assert_array_equal(xq[0], np.array(fx["codes"], np.int8))


# ---------------------------------------------------------------------------
# §4 E4M3 format.
# ---------------------------------------------------------------------------

def test_e4m3_fixture_points():
    with open(os.path.join(GOLDEN, "e4m3_points.txt")) as f:
        pts = [l.split() for l in f if l.strip() and not l.startswith("#")]
    vals = np.array([float(v) for v, _ in pts], np.float32)
    codes = oracle.e4m3_encode(vals)
    assert [int(c) for c in codes] == [int(c, 16) for _, c in pts]


def test_e4m3_decode_matches_torch_and_format():
    codes = np.arange(256, dtype=np.uint8)
    dec = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    np.testing.assert_array_equal(np.isnan(dec), nan)
    np.testing.assert_array_equal(dec[~nan], ref[~nan])
    assert np.nanmax(dec) == 448.0 and np.nanmin(dec) == -448.0


def test_e4m3_roundtrip_all_finite_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    vals = oracle.e4m3_decode(codes).astype(np.float32)
    np.testing.assert_array_equal(oracle.e4m3_encode(vals), codes)


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(7)
    finite = oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    mids = ((finite[1:] + finite[:-1]) / 2).astype(np.float32)  # exact ties
    x = np.concatenate([
        rng.uniform(-448, 448, 20000).astype(np.float32),
        (rng.standard_normal(20000) * 0.01).astype(np.float32),
        mids, -mids,
        np.nextafter(mids, np.float32(np.inf)), np.nextafter(mids, np.float32(0)),
    ]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.e4m3_encode(x), ref)


def test_e4m3_saturates_above_range():
    x = np.array([448.0, 449.0, 463.9, 464.0, 480.0, 1e30, -600.0], np.float32)
    np.testing.assert_array_equal(oracle.e4m3_encode(x),
                                  np.array([0x7E] * 6 + [0xFE], np.uint8))


# ---------------------------------------------------------------------------
# bfloat16 rounding (the output format) against torch's conversion.
# ---------------------------------------------------------------------------

def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(8)
    bits = rng.integers(0, 2 ** 32, size=30000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    # exact ties: low 16 bits = 0x8000
    ties = ((rng.integers(0, 2 ** 16, 2000).astype(np.uint32) << 16) | 0x8000).view(np.float32)
    ties = ties[np.isfinite(ties)]
    x = np.concatenate([x, ties, np.float32([0.0, -0.0, 3.4e38, -3.4e38, 1e-45])])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle.f32_to_bf16(x), ref)


def test_bf16_widening_exact():
    h = np.arange(0, 2 ** 16, 97, dtype=np.uint16)
    ref = torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).float().numpy()
    got = oracle.bf16_to_f32(h)
    finite = np.isfinite(ref)
    np.testing.assert_array_equal(got[finite], ref[finite])


# ---------------------------------------------------------------------------
# §3 "Choosing the Smoothing Factor": s_j = max|X_j|^a / max|W_j|^(1-a).
# ---------------------------------------------------------------------------

def test_smooth_factor_hand_values():
    ax = np.float32([16.0, 16.0, 16.0, 16.0, 9.0])
    aw = np.float32([4.0, 4.0, 4.0, 4.0, 1.0])
    assert oracle.smooth_factors(ax, aw, 0.5)[0] == np.float32(2.0)
    assert oracle.smooth_factors(ax, aw, 1.0)[0] == np.float32(16.0)
    assert oracle.smooth_factors(ax, aw, 0.0)[0] == np.float32(0.25)
    # 16^0.75 / 4^0.25 = 8 / sqrt(2) = 4 sqrt(2); swapping alpha and 1-alpha
    # would give 16^0.25 / 4^0.75 = sqrt(2)/2 instead.
    got = oracle.smooth_factors(ax, aw, 0.75)[0]
    assert got == np.float32(4.0 * math.sqrt(2.0))
    assert oracle.smooth_factors(ax, aw, 0.5)[4] == np.float32(3.0)


def test_smooth_factor_zero_amax_is_clamped():
    s = oracle.smooth_factors(np.float32([0.0, 1.0]), np.float32([1.0, 0.0]), 0.5)
    assert np.isfinite(s).all() and (s > 0).all()
    assert abs(float(s[0]) - math.sqrt(1e-5)) <= 1e-7 * math.sqrt(1e-5) + 1e-12
    assert abs(float(s[1]) - 1.0 / math.sqrt(1e-5)) <= 1e-6 / math.sqrt(1e-5)


def test_alpha_half_balances_ranges():
    rng = np.random.default_rng(9)
    ax = rng.uniform(0.1, 100.0, 512).astype(np.float32)
    aw = rng.uniform(0.001, 0.5, 512).astype(np.float32)
    s = oracle.smooth_factors(ax, aw, 0.5).astype(np.float64)
    # after smoothing both channel ranges equal sqrt(ax*aw)
    lhs = ax / s
    rhs = aw * s
    g = np.sqrt(ax.astype(np.float64) * aw.astype(np.float64))
    assert np.all(np.abs(lhs - g) <= 4e-7 * g)
    assert np.all(np.abs(rhs - g) <= 4e-7 * g)


def test_alpha_one_normalizes_calibration_channels():
    case = workloads.TINY
    d = synth.generate(case)
    ax = oracle.amax(d["x_cal"], per_column=True)
    aw = oracle.amax(d["w"], per_column=False)
    s = oracle.smooth_factors(ax, aw, 1.0)
    np.testing.assert_array_equal(s, ax)
    xs = oracle.smooth_act(d["x_cal"], s)
    np.testing.assert_array_equal(np.abs(xs).max(axis=0), np.ones(case.K, np.float32))


def test_alpha_zero_normalizes_weight_rows():
    rng = np.random.default_rng(10)
    w = (rng.standard_normal((40, 24)) * 0.02).astype(np.float32)
    aw = oracle.amax(w, per_column=False)
    s = oracle.smooth_factors(np.ones(40, np.float32), aw, 0.0)
    ws = oracle.smooth_weight(w, s)
    rowmax = np.abs(ws).max(axis=1)
    assert np.all(np.abs(rowmax - 1.0) <= 2.0 ** -22)


# ---------------------------------------------------------------------------
# Calibration amax along each axis, and quantization of weights / activations.
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_amax_axes(dtype):
    rng = np.random.default_rng(11)
    x = rng.standard_normal((37, 53)).astype(np.float32) * 3
    if dtype == "bf16":
        xb = synth.to_bf16_bits(x)
        xf = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).float().numpy()
        src = xb
    else:
        xf = x
        src = x
    np.testing.assert_array_equal(oracle.amax(src, True), np.abs(xf).max(axis=0))
    np.testing.assert_array_equal(oracle.amax(src, False), np.abs(xf).max(axis=1))


def test_amax_of_small_and_zero_channels():
    """Channels whose values all lie below 1 in magnitude, and all-zero ones,
    along both axes (a calibration scaled like layer activations after a
    normalization)."""
    rng = np.random.default_rng(15)
    x = (rng.uniform(-1, 1, (9, 24)) * 1e-3).astype(np.float32)
    x[:, 4] = 0.0
    x[6] = 0.0
    np.testing.assert_array_equal(oracle.amax(x, True), np.abs(x).max(axis=0))
    np.testing.assert_array_equal(oracle.amax(x, False), np.abs(x).max(axis=1))
    assert oracle.amax(x, True)[4] == 0 and oracle.amax(x, False)[6] == 0


def test_quantize_weight_layout_and_scale():
    K, N = 48, 40
    w = np.full((K, N), 0.001, np.float32)
    w[7, 29] = -3.0
    w[:, 5] = 0.0
    wq, sw = oracle.quantize_weight(w, None)
    assert wq.shape == (N, K)
    assert wq[29, 7] == -127
    assert abs(float(sw[29]) - 3.0 / 127) <= 1e-7
    assert sw[5] == 0 and not wq[5].any()
    # every other entry of column 29 is tiny
    assert np.abs(wq[29].astype(int)).sum() == 127


@pytest.mark.parametrize("smooth", [False, True])
def test_weight_quant_error_bound(smooth):
    rng = np.random.default_rng(12)
    K, N = 64, 48
    w = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    s = rng.uniform(0.2, 5.0, K).astype(np.float32) if smooth else None
    wq, sw = oracle.quantize_weight(w, s)
    wt = oracle.smooth_weight(w, s) if smooth else w
    deq = wq.T.astype(np.float64) * sw.astype(np.float64)[None, :]
    err = np.abs(wt.astype(np.float64) - deq)
    assert np.all(err <= sw.astype(np.float64)[None, :] / 2 * (1 + 2.0 ** -20))
    # the largest element of each column lands on +-127
    assert np.all(np.abs(wq.astype(int)).max(axis=1) == 127)


def test_act_quant_error_bound_and_extremes():
    case = workloads.TINY
    d = synth.generate(case)
    x = d["x"]
    s = synth.random_floats(case.K, seed=3, lo=0.5, hi=8.0)
    xq, sx = oracle.quantize_act(x, s)
    xs = oracle.smooth_act(x, s).astype(np.float64)
    deq = xq.astype(np.float64) * sx.astype(np.float64)[:, None]
    assert np.all(np.abs(xs - deq) <= sx.astype(np.float64)[:, None] / 2 * (1 + 2.0 ** -20))
    assert np.all(np.abs(xq.astype(int)).max(axis=1) == 127)
    assert xq.min() >= -127


def test_act_quant_zero_row_and_no_smoothing():
    x = np.zeros((3, 16), np.float32)
    x[1] = np.linspace(-2, 2, 16, dtype=np.float32)
    xq, sx = oracle.quantize_act(x, None)
    assert sx[0] == 0 and sx[2] == 0 and not xq[0].any() and not xq[2].any()
    xq1, sx1 = oracle.quantize_act(x, np.ones(16, np.float32))
    np.testing.assert_array_equal(xq, xq1)
    np.testing.assert_array_equal(sx, sx1)


def test_scale_that_underflows_to_zero_gives_zero_codes():
    """A row / column whose amax / Q underflows to a zero scale (amax a few
    subnormal steps) is stored with scale 0 and all codes 0, although its
    elements are not zero; dividing by that zero scale would give +-inf and
    saturated codes instead."""
    tiny = np.float32(2.0 ** -147)          # amax / 127 rounds to 0 in binary32
    assert np.float32(tiny / np.float32(127.0)) == 0 and tiny > 0
    x = np.zeros((2, 16), np.float32)
    x[0, 3], x[0, 9] = tiny, -tiny
    x[1] = 1.0
    for qt in (oracle.INT8, oracle.E4M3):
        xq, sx = oracle.quantize_act(x, None, qt)
        assert sx[0] == 0 and not xq[0].view(np.uint8).any(), qt
        assert sx[1] > 0
        wq, sw = oracle.quantize_weight(np.ascontiguousarray(x.T), None, qt)
        assert sw[0] == 0 and not wq[0].view(np.uint8).any(), qt


def test_quantize_weight_e4m3_scale_and_extreme():
    """E4M3 weights: sw[n] = amax_n / 448 and the largest element of each
    output channel is stored as +-448 (code 0x7E / 0xFE)."""
    K, N = 32, 24
    rng = np.random.default_rng(14)
    w = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    w[5, 7] = -0.5
    wq, sw = oracle.quantize_weight(w, None, oracle.E4M3)
    amax = np.abs(w).max(axis=0)
    np.testing.assert_array_equal(sw, (amax / np.float32(448.0)).astype(np.float32))
    assert wq[7, 5] == 0xFE
    top = np.abs(w).argmax(axis=0)
    assert np.all((wq[np.arange(N), top] & 0x7F) == 0x7E)


def test_act_quant_e4m3_bound():
    rng = np.random.default_rng(13)
    x = (rng.standard_normal((8, 64)) * 5).astype(np.float32)
    xq, sx = oracle.quantize_act(x, None, oracle.E4M3)
    dec = oracle.e4m3_decode(xq) * sx.astype(np.float64)[:, None]
    xd = x.astype(np.float64)
    # 3 mantissa bits: half-ulp relative error 2^-4 for normals, plus the
    # half subnormal step 2^-10 in units of the scale
    assert np.all(np.abs(xd - dec) <= 2.0 ** -4 * np.abs(xd) + 2.0 ** -10 * sx[:, None] * 1.0001)
    absmax_codes = xq[np.arange(8), np.abs(x).argmax(axis=1)]
    assert np.all((absmax_codes & 0x7F) == 0x7E)


# ---------------------------------------------------------------------------
# 8-bit GEMMs against independent brute force.
# ---------------------------------------------------------------------------

def test_gemm_i8_brute_force_nonsquare():
    xq = synth.random_matrix((7, 48), np.int8, seed=1)
    wq = synth.random_matrix((5, 48), np.int8, seed=2)
    acc = oracle.gemm_i8(xq, wq)
    ref = xq.astype(np.int64) @ wq.astype(np.int64).T
    np.testing.assert_array_equal(acc, ref)


def test_gemm_i8_extremes():
    K = 4096
    xq = np.full((2, K), 127, np.int8)
    xq[1] = -127
    wq = np.full((3, K), 127, np.int8)
    wq[2] = 0
    wq[2, 17] = 1
    acc = oracle.gemm_i8(xq, wq)
    assert acc[0, 0] == K * 127 * 127 and acc[1, 1] == -K * 127 * 127
    assert acc[0, 2] == 127 and acc[1, 2] == -127


def test_gemm_e4m3_exact():
    rng = np.random.default_rng(14)
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    xq = rng.choice(codes, size=(6, 160)).astype(np.uint8)
    wq = rng.choice(codes, size=(9, 160)).astype(np.uint8)
    acc = oracle.gemm_e4m3(xq, wq)
    # all partial sums are exact in binary64, so any summation order gives the
    # same value; numpy's matmul of the decoded values is an independent sum
    ref = oracle.e4m3_decode(xq) @ oracle.e4m3_decode(wq).T
    np.testing.assert_array_equal(acc, ref)


# ---------------------------------------------------------------------------
# Dequantization epilogue.
# ---------------------------------------------------------------------------

def test_epilogue_power_of_two_scales_exact():
    acc = np.array([[3, -1000, 12345], [0, 7, -8]], np.int32)
    sx = np.float32([2.0 ** -7, 0.5])
    sw = np.float32([0.25, 2.0 ** -10, 8.0])
    yf, yb = oracle.epilogue(acc, sx, sw, None)
    exact = acc.astype(np.float64) * sx[:, None].astype(np.float64) * sw[None, :].astype(np.float64)
    np.testing.assert_array_equal(yf.astype(np.float64), exact)
    ref = torch.from_numpy(yf).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(yb, ref)


def test_epilogue_bias_added():
    acc = np.array([[4, 0]], np.int32)
    bias = synth.to_bf16_bits(np.float32([0.5, -1.25]))
    yf, _ = oracle.epilogue(acc, np.float32([0.25]), np.float32([1.0, 1.0]), bias)
    np.testing.assert_array_equal(yf, np.float32([[1.5, -1.25]]))


def test_epilogue_relative_error_bound():
    rng = np.random.default_rng(15)
    acc = rng.integers(-2 ** 28, 2 ** 28, size=(16, 32)).astype(np.int32)
    sx = rng.uniform(0.01, 1, 16).astype(np.float32)
    sw = rng.uniform(1e-4, 1e-2, 32).astype(np.float32)
    yf, _ = oracle.epilogue(acc, sx, sw, None)
    exact = acc.astype(np.float64) * sx[:, None] * sw[None, :]
    # int->float rounding plus two products: below 3 units of 2^-24
    assert np.all(np.abs(yf - exact) <= 3.01 * 2.0 ** -24 * np.abs(exact))


@pytest.mark.parametrize("qt", [oracle.INT8, oracle.E4M3])
def test_linear_at_matches_full_path(qt):
    """The sampled-output function the full-size GPU tests use equals the
    full product at the sampled points, for both code types."""
    case = workloads.TINY
    d = synth.generate(case)
    ax = oracle.amax(d["x_cal"], True)
    aw = oracle.amax(d["w"], False)
    s = oracle.smooth_factors(ax, aw, case.alpha)
    wq, sw = oracle.quantize_weight(d["w"], s, qt)
    bias = synth.to_bf16_bits(synth.random_floats(case.N, seed=4, std=0.1))
    full = oracle.linear(d["x"], s, wq, sw, bias, qt)
    rows = np.array([0, 3, 15, 8, 2, 9], np.int64)
    cols = np.array([0, 63, 41, 7, 3, 12], np.int64)
    acc, yf, yb = oracle.linear_at(full["xq"], full["sx"], wq, sw, bias, rows, cols, qt)
    np.testing.assert_array_equal(acc, full["acc"][rows, cols].astype(np.float64))
    np.testing.assert_array_equal(yf, full["y_f32"][rows, cols])
    np.testing.assert_array_equal(yb, full["y_bf16"][rows, cols])


# ---------------------------------------------------------------------------
# §3: quantization after smoothing gives a smaller error than without.
# ---------------------------------------------------------------------------

def test_smoothing_reduces_quantization_error_on_outlier_data():
    case = workloads.TINY
    d = synth.generate(case)
    x, w = d["x"], d["w"]
    exact = x.astype(np.float64) @ w.astype(np.float64)

    def err(s):
        wq, sw = oracle.quantize_weight(w, s)
        y = oracle.linear(x, s, wq, sw)["y_f32"].astype(np.float64)
        return np.linalg.norm(y - exact) / np.linalg.norm(exact)

    ax = oracle.amax(x, True)
    aw = oracle.amax(w, False)
    s = oracle.smooth_factors(ax, aw, 0.5)
    e_smooth, e_plain = err(s), err(None)
    assert e_smooth < 0.5 * e_plain, (e_smooth, e_plain)
    assert e_smooth < 0.05


# ---------------------------------------------------------------------------
# §4 per-tensor scaling (online, and delayed from the previous step's max).
# ---------------------------------------------------------------------------

def test_per_tensor_example_spans_tokens():
    """The §2 row split into two tokens: one per-tensor scale (80/127) for
    both, so 75 maps to 119 as on the page, where a per-token scale for the
    second token (75/127) would give it the full 127."""
    fx = _fixture("per_tensor_scale.txt")
    row = np.array(fx["row"], np.float32)
    x = row.reshape(2, 4)
    xq, scale, amax = oracle.quantize_act_tensor(x, None, oracle.INT8)
    assert abs(float(scale) - float(fx["scale_approx"][0])) <= \
        float(fx["scale_rel_tol"][0]) * float(fx["scale_approx"][0])
    assert amax == np.float32(80.0)
    np.testing.assert_array_equal(xq.reshape(-1), np.array(fx["codes"], np.int8))
    per_token, _ = oracle.quantize_act(x, None)
    assert per_token[1, 1] == 127 and xq[1, 1] == 119


@pytest.mark.parametrize("qt", [oracle.INT8, oracle.E4M3])
def test_per_tensor_one_token_is_per_token(qt):
    """With a single token the tensor is the row: online per-tensor scaling
    must equal the (separately pinned) per-token quantization."""
    g = np.random.default_rng(5)
    x = (g.standard_normal((1, 96)) * 4).astype(np.float32)
    s = synth.random_floats(96, seed=6, lo=0.1, hi=10.0)
    xq_t, scale, amax = oracle.quantize_act_tensor(x, s, qt)
    xq_r, sx = oracle.quantize_act(x, s, qt)
    np.testing.assert_array_equal(xq_t, xq_r)
    assert scale == sx[0]
    assert amax == np.abs((x / s).astype(np.float32)).max()


@pytest.mark.parametrize("qt", [oracle.INT8, oracle.E4M3])
def test_per_tensor_brute_force(qt):
    """Element by element in numpy binary32: codes of x/s/scale under the
    given (delayed) scale, saturating, and the tensor's max |x/s|."""
    g = np.random.default_rng(7)
    x = (g.standard_normal((5, 24)) * 3).astype(np.float32)
    x[2, 3] = 40.0                                     # beyond the delayed scale
    x[4, 0] = -40.0
    s = synth.random_floats(24, seed=8, lo=0.5, hi=2.0)
    s[3] = 1.0
    s[0] = 1.0
    scale = np.float32(0.05)                           # Q * scale = 6.35 (INT8), 22.4 (E4M3)
    xq, used, amax = oracle.quantize_act_tensor(x, s, qt, scale=scale)
    assert used == scale
    xs = (x / s).astype(np.float32)
    assert amax == np.abs(xs).max()
    for (m, k), v in np.ndenumerate(xs):
        q = np.float32(v / scale)
        if qt == oracle.INT8:
            want = np.int8(min(max(np.rint(q), -127), 127))
            assert xq[m, k] == want, (m, k)
        else:
            assert xq[m, k] == oracle.e4m3_encode(q), (m, k)
    if qt == oracle.INT8:
        assert xq[2, 3] == 127 and xq[4, 0] == -127
    else:
        assert xq[2, 3] == 0x7E and xq[4, 0] == 0xFE   # +-448: satfinite


def test_per_tensor_delayed_with_own_max_is_online_and_zero_scale():
    g = np.random.default_rng(9)
    x = (g.standard_normal((6, 32)) * 2).astype(np.float32)
    xq_o, scale_o, amax = oracle.quantize_act_tensor(x, None, oracle.E4M3)
    assert scale_o == np.float32(amax / np.float32(448.0))
    xq_d, _, _ = oracle.quantize_act_tensor(x, None, oracle.E4M3, scale=scale_o)
    np.testing.assert_array_equal(xq_o, xq_d)
    xq_z, _, amax_z = oracle.quantize_act_tensor(x, None, oracle.INT8, scale=np.float32(0.0))
    assert not xq_z.any() and amax_z == amax


# ---------------------------------------------------------------------------
# The smoothing is offline: 1/s folded once into the layer that produces X.
# ---------------------------------------------------------------------------

def test_fold_worked_example_gain_emits_the_smoothed_values():
    """A producer with unit gain on the worked example's channel, folded with
    s = 8, has gain 1/8 and emits the smoothed values printed in §3."""
    fx = _fixture("worked_example.txt")
    x = np.array(fx["x"], np.float32)
    s = np.array(fx["s"], np.float32)
    g = oracle.fold_smoothing(np.ones(3, np.float32), s)[0]
    np.testing.assert_array_equal(g, np.full(3, 0.125, np.float32))
    np.testing.assert_array_equal((x * g).astype(np.float32),
                                  np.array(fx["x_smoothed"], np.float32))


def test_fold_power_of_two_is_an_exact_scaling():
    """Division by 2^e is the exact scaling by 2^-e, along either axis."""
    rng = np.random.default_rng(61)
    p = rng.standard_normal((5, 40)).astype(np.float32)
    ec = rng.integers(-12, 13, size=40)
    er = rng.integers(-12, 13, size=5)
    sc = np.ldexp(np.ones(40), ec).astype(np.float32)
    sr = np.ldexp(np.ones(5), er).astype(np.float32)
    np.testing.assert_array_equal(oracle.fold_smoothing(p, sc, per_column=True),
                                  np.ldexp(p.astype(np.float64), -ec[None, :]).astype(np.float32))
    np.testing.assert_array_equal(oracle.fold_smoothing(p, sr, per_column=False),
                                  np.ldexp(p.astype(np.float64), -er[:, None]).astype(np.float32))


@pytest.mark.parametrize("bf16", [False, True])
def test_fold_general_s_is_the_correctly_rounded_quotient(bf16):
    """A binary64 quotient of two binary32 values rounded once to binary32 is
    their correctly rounded binary32 quotient (53 >= 2*24 + 2 significant
    bits, so the double rounding is harmless): an independent route to the
    fold's result. bf16 parameters widen exactly first."""
    rng = np.random.default_rng(62)
    p = (rng.standard_normal((7, 33)) * np.exp(rng.uniform(-20, 20, (7, 33)))).astype(np.float32)
    s = np.exp(rng.uniform(np.log(1e-3), np.log(1e3), 33)).astype(np.float32)
    if bf16:
        pin = synth.to_bf16_bits(p)
        pw = oracle.bf16_to_f32(pin)
    else:
        pin = pw = p
    want = (pw.astype(np.float64) / s.astype(np.float64)[None, :]).astype(np.float32)
    np.testing.assert_array_equal(oracle.fold_smoothing(pin, s, per_column=True), want)


def test_fold_axes_are_transposes_of_each_other():
    """Channel = column of p [R,K] and channel = row of p^T [K,R] give
    transposed results (a swapped index would fail on this non-square p)."""
    rng = np.random.default_rng(63)
    p = rng.standard_normal((6, 11)).astype(np.float32)
    s = rng.uniform(0.05, 20.0, 11).astype(np.float32)
    a = oracle.fold_smoothing(p, s, per_column=True)
    b = oracle.fold_smoothing(np.ascontiguousarray(p.T), s, per_column=False)
    np.testing.assert_array_equal(a, b.T)
    assert not np.array_equal(a, p / s[0])


@pytest.mark.parametrize("qt", [oracle.INT8, oracle.E4M3])
def test_folded_producer_feeds_the_same_codes(qt):
    """A gain producer x * g: folded (gain g/s, then quantization without s)
    and unfolded (gain g, then x/s inside the quantization) give the same
    codes and scales when s is a power of two, and X~ within two roundings
    on each side otherwise."""
    rng = np.random.default_rng(64)
    M, K = 9, 64
    x = (rng.standard_normal((M, K)) * 3).astype(np.float32)
    x[:, [5, 40]] *= 50
    g = rng.uniform(0.5, 2.0, K).astype(np.float32)
    s = np.ldexp(np.ones(K), rng.integers(-4, 8, K)).astype(np.float32)
    folded = (x * oracle.fold_smoothing(g, s)[0]).astype(np.float32)
    unfolded = (x * g).astype(np.float32)
    q1, sx1 = oracle.quantize_act(folded, None, qt)
    q2, sx2 = oracle.quantize_act(unfolded, s, qt)
    np.testing.assert_array_equal(q1, q2)
    np.testing.assert_array_equal(sx1, sx2)
    s = rng.uniform(0.05, 20.0, K).astype(np.float32)
    folded = (x * oracle.fold_smoothing(g, s)[0]).astype(np.float64)
    exact = x.astype(np.float64) * g.astype(np.float64) / s.astype(np.float64)
    assert np.all(np.abs(folded - exact) <= 2.0 ** -22 * np.abs(exact))


# ---------------------------------------------------------------------------
# Weight-only quantization (W8A16 / W4A16): infra.bea.ai §1 table (W4A16 row,
# weights dequantized, then a 16-bit multiply), the zenaique flashcard (the
# runtime dequantizes weights on the fly against BF16 activations), the
# grasp.study lesson §1 / §3 (W8A16).
# ---------------------------------------------------------------------------

def test_int4_weight_codes_and_packing_by_hand():
    """A column with amax 7 has scale 1: codes are the half-even roundings
    clamped to +-7. The 8 codes of one k-group form one little-endian word,
    even k in bits 0,4,8,12 and odd k in bits 16,20,24,28 (two's complement)."""
    w = np.zeros((8, 3), np.float32)
    w[:, 0] = [7.0, -3.5, 2.5, 0.5, -6.49, 1.0, 3.0, -6.6]  # ties to even: -3.5 -> -4, 2.5 -> 2
    w[7, 1] = -14.0                                           # amax 14 -> scale 2; -14 / 2 = -7
    wq4, sw = oracle.quantize_weight_i4(w)
    assert sw.tolist() == [1.0, 2.0, 0.0]
    # codes (7, -4, 2, 0, -6, 1, 3, -7): even k 7, 2, -6, 3 -> 0x3A27; odd k -4, 0, 1, -7 -> 0x910C
    assert wq4[0].tolist() == [0x27, 0x3A, 0x0C, 0x91]
    assert wq4[1].tolist() == [0x00, 0x00, 0x00, 0x90]      # code -7 at k = 7 (bits 28..31)
    assert not wq4[2].any()                                   # an all-zero channel
    np.testing.assert_array_equal(oracle.unpack_i4(wq4)[0], [7, -4, 2, 0, -6, 1, 3, -7])


@pytest.mark.parametrize("bf16", [False, True])
def test_int4_weight_quant_brute_force(bf16):
    w = synth.random_floats((64, 40), seed=41, std=0.02)
    w[:, 3] = 0.0
    w[5, 7] = 0.5                                  # one dominant weight per channel
    if bf16:
        w = synth.to_bf16_bits(w)
    wf = oracle.bf16_to_f32_array(w) if bf16 else w
    amax = np.abs(wf).max(axis=0)
    scale = (amax / np.float32(7.0)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0))
    codes = np.clip(np.rint(wf / safe[None, :]), -7, 7).astype(np.int8).T
    codes[scale == 0] = 0
    wq4, sw = oracle.quantize_weight_i4(w)
    np.testing.assert_array_equal(sw, scale)
    np.testing.assert_array_equal(oracle.unpack_i4(wq4), codes)
    nib = codes.astype(np.int64).reshape(codes.shape[0], -1, 8) & 0xF   # [N, K/8, 8]
    words = np.zeros(nib.shape[:2], np.int64)
    for j in range(4):
        words |= nib[:, :, 2 * j] << (4 * j)
        words |= nib[:, :, 2 * j + 1] << (16 + 4 * j)
    np.testing.assert_array_equal(wq4, words.astype("<u4").view(np.uint8).reshape(wq4.shape))
    # the largest weight of a channel maps to +-7 and the error is half a step
    assert (np.abs(oracle.unpack_i4(wq4)[7]).max() == 7)
    err = np.abs(wf.T - codes * sw[:, None])
    assert (err <= sw[:, None] / 2 * (1 + 2 ** -20)).all()


@pytest.mark.parametrize("bits", [8, 4])
def test_weight_only_gemm_brute_force(bits):
    M, K, N = 5, 96, 24
    x = synth.to_bf16_bits(synth.random_floats((M, K), seed=42, std=1.0) *
                           np.float32(3.0))
    w = synth.random_floats((K, N), seed=43, std=0.02)
    bias = synth.to_bf16_bits(synth.random_floats(N, seed=44, std=0.05))
    if bits == 8:
        wq, sw = oracle.quantize_weight(w, None)
        codes = wq
    else:
        wq, sw = oracle.quantize_weight_i4(w)
        codes = oracle.unpack_i4(wq)
    xf = oracle.bf16_to_f32_array(x).astype(np.float64)
    ref = xf @ (codes.astype(np.float64) * sw.astype(np.float64)[:, None]).T
    ref += oracle.bf16_to_f32_array(bias).astype(np.float64)[None, :]
    y = oracle.gemm_weight_only(x, wq, sw, bias, bits)
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-13)
    y0 = oracle.gemm_weight_only(x, wq, sw, None, bits)
    np.testing.assert_allclose(y - y0, np.broadcast_to(
        oracle.bf16_to_f32_array(bias).astype(np.float64), y.shape), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("bits", [8, 4])
def test_weight_only_one_hot_row_reads_one_dequantized_weight(bits):
    K, N = 32, 16
    w = synth.random_floats((K, N), seed=45, std=0.02)
    wq, sw = oracle.quantize_weight(w, None) if bits == 8 else oracle.quantize_weight_i4(w)
    codes = wq if bits == 8 else oracle.unpack_i4(wq)
    x = np.zeros((K, K), np.float32)
    x[np.arange(K), np.arange(K)] = 1.0            # row j is e_j
    y = oracle.gemm_weight_only(synth.to_bf16_bits(x), wq, sw, None, bits)
    np.testing.assert_array_equal(y, (codes.astype(np.float64) * sw.astype(np.float64)[:, None]).T)


def test_weight_only_on_integer_activations_is_the_int8_gemm_scaled():
    """With integer activations (|x| <= 127, exact in bf16) the weight-only
    product equals the INT8 GEMM of the same codes times the channel scale."""
    M, K, N = 7, 160, 40
    xi = synth.random_matrix((M, K), np.int8, seed=46)
    w = synth.random_floats((K, N), seed=47, std=0.02)
    wq, sw = oracle.quantize_weight(w, None)
    y = oracle.gemm_weight_only(synth.to_bf16_bits(xi.astype(np.float32)), wq, sw, None, 8)
    acc = oracle.gemm_i8(xi, wq).astype(np.float64)
    np.testing.assert_array_equal(y, acc * sw.astype(np.float64)[None, :])


# ---------------------------------------------------------------------------
# The producer of X with the smoothing folded in: RMS normalization, then
# per-token quantization ("Weight-Activation Quantization" §3 "Step 1" and the
# grasp.study lesson §2: the smoothing is applied offline, with no runtime
# overhead). Pinned against exact rational arithmetic, closed forms, exact
# scalings and the per-token quantization already pinned above.
# ---------------------------------------------------------------------------

def _rms_reference(xb, g, eps):
    """r and xn from the definition, the sum of squares in exact rational
    arithmetic (every element here is within 48 binades of the row's
    largest), then the binary64 steps in Python floats (IEEE, rounded once
    each) and the binary32 products in numpy float32."""
    from fractions import Fraction
    xf = oracle.bf16_to_f32_array(xb)
    M, K = xb.shape
    r = np.empty(M, np.float32)
    for m in range(M):
        ss = sum((Fraction(float(v)) ** 2 for v in xf[m]), Fraction(0))
        mean = float(ss) / float(K)              # float(Fraction) is correctly rounded
        t = math.sqrt(mean + float(np.float32(eps)))
        r[m] = np.float32(1.0 / t)
    xn = (xf * r[:, None]).astype(np.float32) * g.astype(np.float32)[None, :]
    return r, xn.astype(np.float32)


@pytest.mark.parametrize("K", [64, 384, 1024])
def test_rmsnorm_matches_exact_rational_sum_of_squares(K):
    x = synth.random_floats((6, K), seed=70 + K, std=1.0)
    x[:, 5] *= 80.0                                    # an outlier channel
    x[2] *= 1e-3                                       # a small row
    xb = synth.to_bf16_bits(x)
    g = synth.random_floats(K, seed=71, lo=0.25, hi=3.0)
    for eps in (1e-6, 1e-2):
        xq, sx, r, xn = oracle.rmsnorm_quantize_act(xb, g, eps)
        r_ref, xn_ref = _rms_reference(xb, g, eps)
        np.testing.assert_array_equal(r.view(np.uint32), r_ref.view(np.uint32))
        np.testing.assert_array_equal(xn.view(np.uint32), xn_ref.view(np.uint32))
        # then exactly the per-token quantization of xn, without smoothing
        for qt in (oracle.INT8, oracle.E4M3):
            q2, s2 = oracle.quantize_act(xn_ref, None, qt)
            q1, s1, _, _ = oracle.rmsnorm_quantize_act(xb, g, eps, qt)
            np.testing.assert_array_equal(q1.view(np.uint8), q2.view(np.uint8))
            np.testing.assert_array_equal(s1, s2)


def test_rmsnorm_single_value_closed_form():
    """One nonzero x = 2 in a row of 64: mean square 4/64 = 1/16, 1/rms = 4,
    so xn = 2 * 4 * g exactly (eps far below the binary64 resolution of 1/16)."""
    K = 64
    x = np.zeros((1, K), np.float32)
    x[0, 9] = 2.0
    g = synth.random_floats(K, seed=72, lo=0.5, hi=2.0)
    xq, sx, r, xn = oracle.rmsnorm_quantize_act(synth.to_bf16_bits(x), g, 1e-38)
    assert r[0] == np.float32(4.0)
    expect = np.zeros(K, np.float32)
    expect[9] = np.float32(8.0) * g[9]
    np.testing.assert_array_equal(xn[0], expect)
    assert xq[0, 9] == 127 and not xq[0, np.arange(K) != 9].any()


def test_rmsnorm_is_exactly_homogeneous_under_powers_of_two():
    """Scaling a row by 2^j (exact in bf16) scales 1/rms by 2^-j and leaves
    xn and the codes bit for bit unchanged (eps negligible)."""
    x = synth.random_floats((4, 256), seed=73, std=1.0)
    g = synth.random_floats(256, seed=74, lo=0.5, hi=2.0)
    q0, s0, r0, xn0 = oracle.rmsnorm_quantize_act(synth.to_bf16_bits(x), g, 1e-38)
    for j in (-9, 7):
        q1, s1, r1, xn1 = oracle.rmsnorm_quantize_act(synth.to_bf16_bits(x * 2.0 ** j), g, 1e-38)
        np.testing.assert_array_equal(r1, r0 * np.float32(2.0 ** -j))
        np.testing.assert_array_equal(xn1, xn0)
        np.testing.assert_array_equal(q1, q0)


def test_rmsnorm_zero_row_and_eps():
    """An all-zero row: 1/rms = 1/sqrt(eps) (binary64, then binary32), zero
    codes and scale 0."""
    x = np.zeros((2, 32), np.float32)
    x[1, 3] = 1.0
    eps = np.float32(1e-2)
    xq, sx, r, xn = oracle.rmsnorm_quantize_act(synth.to_bf16_bits(x), np.ones(32, np.float32), eps)
    assert r[0] == np.float32(1.0 / math.sqrt(float(eps)))
    assert sx[0] == 0.0 and not xq[0].any()
    assert r[1] == np.float32(1.0 / math.sqrt(1.0 / 32.0 + float(eps)))


@pytest.mark.parametrize("qt", [oracle.INT8, oracle.E4M3])
def test_rmsnorm_with_folded_gain_equals_smoothing_after_the_norm(qt):
    """With power-of-two smoothing factors, the norm with the folded gain
    gamma / s gives the codes and scales of the per-token quantization of the
    norm's output (gain gamma) smoothed by s at run time: the fold moves the
    division, exactly."""
    K = 128
    x = synth.random_floats((5, K), seed=75, std=1.0)
    x[:, 17] *= 50.0
    xb = synth.to_bf16_bits(x)
    gamma = synth.random_floats(K, seed=76, lo=0.5, hi=2.0)
    s = (2.0 ** np.random.default_rng(77).integers(-6, 7, K)).astype(np.float32)
    g_folded = oracle.fold_smoothing(gamma, s)[0]
    q1, s1, _, _ = oracle.rmsnorm_quantize_act(xb, g_folded, 1e-6, qt)
    _, _, _, xn_gamma = oracle.rmsnorm_quantize_act(xb, gamma, 1e-6, qt)
    q2, s2 = oracle.quantize_act(xn_gamma, s, qt)
    np.testing.assert_array_equal(q1.view(np.uint8), q2.view(np.uint8))
    np.testing.assert_array_equal(s1, s2)


def test_rmsnorm_drops_only_terms_far_below_the_row_maximum():
    """Elements more than 48 binades below the row's largest do not enter the
    sum of squares (each is below 2^-94 of the largest square); elements
    within that range do, exactly."""
    K = 64
    x = np.zeros((3, K), np.float32)
    x[:, 0] = 2.0 ** 20
    x[1, 1:] = 2.0 ** -40          # 60 binades below: dropped
    x[2, 1:4] = 2.0 ** 10          # 10 binades below: kept
    xq, sx, r, xn = oracle.rmsnorm_quantize_act(synth.to_bf16_bits(x), np.ones(K, np.float32), 1e-38)
    assert r[1] == r[0]
    ss = 2.0 ** 40 + 3 * 2.0 ** 20
    assert r[2] == np.float32(1.0 / math.sqrt(ss / K))
