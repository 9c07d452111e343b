"""Stage-by-stage parity of the CUDA path against the CPU oracle.

Each GPU stage gets exactly the inputs the oracle gets (seeded synthetic
data, or the oracle's own outputs of the previous stage), so a one-ulp
difference upstream cannot cascade. The bar: bit-exact INT8 / E4M3 codes,
scales, int32 accumulators and INT8-path outputs; smoothing factors within
2 ulp; the FP8 GEMM within 1e-3 of the exact sum on the normalized metric.
"""
import numpy as np
import pytest
import torch

import oracle
from w8a8_smoothquant_int8_02_b200 import ops, synth

from _gpu_util import dev, fp8_normalized_error, host, sample_points, ulp_distance

pytestmark = pytest.mark.gpu

E4M3_FINITE = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)


def _x(shape, seed, dtype, outliers=True):
    x = synth.random_floats(shape, seed=seed, std=1.0)
    if outliers:
        g = np.random.default_rng(seed + 1000)
        ch = g.choice(shape[1], size=max(1, shape[1] // 64), replace=False)
        x[:, ch] *= g.uniform(20, 100, ch.size).astype(np.float32)
    return synth.to_bf16_bits(x) if dtype == "bf16" else x


# ------------------------------------------------------------------ a1 / a2 --

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("rows,cols", [(1, 64), (37, 200), (512, 4096), (3000, 8)])
def test_calibrate_amax(dtype, rows, cols):
    x = _x((rows, cols), seed=rows + cols, dtype=dtype)
    xd = dev(x)
    np.testing.assert_array_equal(host(ops.calibrate_amax(xd, "column")), oracle.amax(x, True))
    np.testing.assert_array_equal(host(ops.calibrate_amax(xd, "row")), oracle.amax(x, False))


def test_calibrate_amax_accumulates_over_batches():
    a = _x((64, 128), seed=1, dtype="bf16")
    b = _x((40, 128), seed=2, dtype="bf16")
    out = ops.calibrate_amax(dev(a), "column")
    ops.calibrate_amax(dev(b), "column", out=out, accumulate=True)
    ref = np.maximum(oracle.amax(a, True), oracle.amax(b, True))
    np.testing.assert_array_equal(host(out), ref)
    assert ops.device_status() == ops.SQ_OK


# ----------------------------------------------------------------------- a3 --

def reciprocals(s):
    """The documented content of s_inv: the IEEE binary32 reciprocal inside
    [2^-20, 2^20], NaN outside."""
    s = np.asarray(s, np.float32)
    inside = (s >= np.float32(2.0 ** -20)) & (s <= np.float32(2.0 ** 20))
    return np.where(inside, np.float32(1.0) / np.where(inside, s, 1), np.float32(np.nan)).astype(np.float32)


@pytest.mark.parametrize("alpha", [0.0, 0.5, 0.85, 1.0])
def test_smooth_factors(alpha):
    g = np.random.default_rng(3)
    ax = g.uniform(0.01, 100, 4096).astype(np.float32)
    aw = g.uniform(1e-4, 0.2, 4096).astype(np.float32)
    ax[:3] = 0.0
    aw[3:6] = 0.0
    s_d, inv_d = ops.smooth_factors(dev(ax), dev(aw), alpha, with_inverse=True)
    got = host(s_d)
    ref = oracle.smooth_factors(ax, aw, alpha)
    d = ulp_distance(got, ref)
    assert d.max() <= 2, d.max()
    assert (d == 0).mean() >= 0.99
    np.testing.assert_array_equal(host(inv_d), reciprocals(got))


# ----------------------------------------------------------------------- a4 --

@pytest.mark.parametrize("qtype", ["i8", "e4m3"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("smooth", [True, False])
@pytest.mark.parametrize("K,N", [(64, 64), (208, 200), (4096, 256), (96, 8)])
def test_quantize_weight(qtype, dtype, smooth, K, N):
    w = synth.random_floats((K, N), seed=K * 7 + N, std=0.02)
    w[:, 0] = 0.0  # an all-zero output channel
    w = synth.to_bf16_bits(w) if dtype == "bf16" else w
    s = synth.random_floats(K, seed=K, lo=0.05, hi=20.0) if smooth else None
    qt = oracle.E4M3 if qtype == "e4m3" else oracle.INT8
    wq_ref, sw_ref = oracle.quantize_weight(w, s, qt)
    wq, sw = ops.quantize_weight(dev(w), None if s is None else dev(s), qtype)
    np.testing.assert_array_equal(host(sw), sw_ref)
    np.testing.assert_array_equal(host(wq).view(np.uint8), wq_ref.view(np.uint8))


# ----------------------------------------------------------------------- a5 --

@pytest.mark.parametrize("qtype", ["i8", "e4m3"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("smooth", [True, False])
@pytest.mark.parametrize("M,K", [(1, 64), (17, 96), (129, 4096), (16, 8192), (3, 14336), (5, 16),
                                 (2, 20000), (2, 65536)])
def test_quantize_act(qtype, dtype, smooth, M, K):
    x = _x((M, K), seed=M * 31 + K, dtype=dtype)
    s = synth.random_floats(K, seed=K + 1, lo=0.05, hi=20.0) if smooth else None
    qt = oracle.E4M3 if qtype == "e4m3" else oracle.INT8
    xq_ref, sx_ref = oracle.quantize_act(x, s, qt)
    variants = [None] if s is None else [None, reciprocals(s)]
    for s_inv in variants:
        xq, sx = ops.quantize_act(dev(x), None if s is None else dev(s), qtype,
                                  s_inv=None if s_inv is None else dev(s_inv))
        np.testing.assert_array_equal(host(sx), sx_ref)
        np.testing.assert_array_equal(host(xq).view(np.uint8), xq_ref.view(np.uint8))


def test_quantize_act_zero_rows_and_ties():
    x = np.zeros((4, 32), np.float32)
    x[1, :10] = [2.5, 3.5, -2.5, 126.5, 127.0, -126.5, 0.5, -0.5, 1.5, 0.49999997]
    x[3] = np.linspace(-1e-3, 1e-3, 32, dtype=np.float32)
    for qtype, qt in (("i8", oracle.INT8), ("e4m3", oracle.E4M3)):
        xq_ref, sx_ref = oracle.quantize_act(x, None, qt)
        xq, sx = ops.quantize_act(dev(x), None, qtype)
        np.testing.assert_array_equal(host(sx), sx_ref)
        np.testing.assert_array_equal(host(xq).view(np.uint8), xq_ref.view(np.uint8))


def test_quantize_act_empty_is_noop():
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    xq, sx = ops.quantize_act(x, None, "i8")
    assert xq.shape == (0, 64) and sx.shape == (0,)
    assert ops.device_status() == ops.SQ_OK


# ------------------------------------------------------------------ a6 INT8 --

GEMM_SHAPES = [(1, 16, 32), (17, 64, 64), (129, 200, 96), (128, 128, 128), (300, 392, 4096),
               (256, 256, 208), (7, 8, 16), (640, 136, 1040)]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
@pytest.mark.parametrize("with_bias", [False, True])
def test_gemm_w8a8(M, N, K, with_bias):
    xq = synth.random_matrix((M, K), np.int8, seed=M + K)
    wq = synth.random_matrix((N, K), np.int8, seed=N + 2 * K)
    sx = synth.random_floats(M, seed=5, lo=1e-3, hi=0.5)
    sw = synth.random_floats(N, seed=6, lo=1e-4, hi=1e-2)
    bias = synth.to_bf16_bits(synth.random_floats(N, seed=7, std=0.1)) if with_bias else None
    acc_ref = oracle.gemm_i8(xq, wq)
    yf_ref, yb_ref = oracle.epilogue(acc_ref, sx, sw, bias)
    d = [dev(a) for a in (xq, sx, wq, sw)]
    b = None if bias is None else dev(bias)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    yf = ops.gemm_w8a8(*d, bias=b, out_dtype=torch.float32, acc=acc)
    yb = ops.gemm_w8a8(*d, bias=b, out_dtype=torch.bfloat16)
    assert ops.device_status() == ops.SQ_OK
    np.testing.assert_array_equal(host(acc), acc_ref)
    np.testing.assert_array_equal(host(yf), yf_ref)
    np.testing.assert_array_equal(host(yb), yb_ref)


@pytest.mark.parametrize("split", [True, False])
@pytest.mark.parametrize("tile", ops.GEMM_TILES)
@pytest.mark.parametrize("M,N,K", [(300, 392, 4096), (129, 200, 96), (513, 520, 208),
                                   (1, 16, 32), (256, 448, 1024), (1100, 904, 272)])
@pytest.mark.parametrize("qtype", ["i8", "e4m3"])
def test_gemm_every_tile_shape(tile, M, N, K, qtype, split, monkeypatch):
    """Every compiled tile shape (1-CTA and SM-pair) on ragged sizes; with
    split=True the last partial round is always split."""
    monkeypatch.setenv("SQ_GEMM_FORCE_SPLIT", "1")
    g = np.random.default_rng(M + N + K)
    if qtype == "i8":
        xq = synth.random_matrix((M, K), np.int8, seed=M * 3 + K)
        wq = synth.random_matrix((N, K), np.int8, seed=N * 5 + K)
    else:
        codes = E4M3_FINITE[np.abs(oracle.e4m3_decode(E4M3_FINITE)) <= 64.0]
        xq = g.choice(codes, size=(M, K)).astype(np.uint8)
        wq = g.choice(codes, size=(N, K)).astype(np.uint8)
    sx = synth.random_floats(M, seed=31, lo=1e-3, hi=0.5)
    sw = synth.random_floats(N, seed=32, lo=1e-4, hi=1e-2)
    bias = synth.to_bf16_bits(synth.random_floats(N, seed=33, std=0.1))
    d = [dev(a) for a in (xq, sx, wq, sw)]
    with ops.gemm_tile(tile):
        if qtype == "i8":
            acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
            yf = ops.gemm_w8a8(*d, bias=dev(bias), out_dtype=torch.float32, acc=acc, split=split)
            yb = ops.gemm_w8a8(*d, bias=dev(bias), split=split)
        else:
            yf = ops.gemm_fp8(*d, bias=dev(bias), out_dtype=torch.float32, split=split)
            yb = ops.gemm_fp8(*d, bias=dev(bias), split=split)
    assert ops.device_status() == ops.SQ_OK
    if qtype == "i8":
        acc_ref = oracle.gemm_i8(xq, wq)
        yf_ref, yb_ref = oracle.epilogue(acc_ref, sx, sw, bias)
        np.testing.assert_array_equal(host(acc), acc_ref)
        np.testing.assert_array_equal(host(yf), yf_ref)
        np.testing.assert_array_equal(host(yb), yb_ref)
    else:
        yf_ref, _ = oracle.epilogue(oracle.gemm_e4m3(xq, wq), sx, sw, bias)
        rows, cols = np.divmod(np.arange(M * N, dtype=np.int64), N)
        e = fp8_normalized_error(host(yf).reshape(-1), yf_ref.reshape(-1), xq, wq, sx, sw, bias,
                                 rows, cols)
        assert e.max() <= 1e-3, e.max()
        np.testing.assert_array_equal(host(yb), oracle.f32_to_bf16(host(yf)))


@pytest.mark.parametrize("M,N,K", [(512, 4096, 1024), (300, 1000, 1040), (129, 8192, 2048),
                                   (1024, 2048, 1024)])
@pytest.mark.parametrize("qtype", ["i8", "e4m3"])
def test_gemm_one_wave(M, N, K, qtype):
    """The one-wave GEMM (every 128 x 128 output tile on its own SM, four
    MMA-issuing threads per tile, each with its own accumulator, added in a
    fixed order): ragged M, N and K, full-range E4M3 codes."""
    if qtype == "i8":
        xq = synth.random_matrix((M, K), np.int8, seed=M * 7 + K)
        wq = synth.random_matrix((N, K), np.int8, seed=N * 11 + K)
    else:
        g = np.random.default_rng(M + 2 * N + K)
        xq = g.choice(E4M3_FINITE, size=(M, K)).astype(np.uint8)
        wq = g.choice(E4M3_FINITE, size=(N, K)).astype(np.uint8)
    sx = synth.random_floats(M, seed=61, lo=1e-6, hi=1e-3)
    sw = synth.random_floats(N, seed=62, lo=1e-6, hi=1e-3)
    bias = synth.to_bf16_bits(synth.random_floats(N, seed=63, std=0.1))
    d = [dev(a) for a in (xq, sx, wq, sw)]
    if qtype == "i8":
        acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
        yf = ops.gemm_w8a8(*d, bias=dev(bias), out_dtype=torch.float32, acc=acc)
        yb = ops.gemm_w8a8(*d, bias=dev(bias))
    else:
        yf = ops.gemm_fp8(*d, bias=dev(bias), out_dtype=torch.float32)
        yb = ops.gemm_fp8(*d, bias=dev(bias))
    assert ops.device_status() == ops.SQ_OK
    if qtype == "i8":
        acc_ref = oracle.gemm_i8(xq, wq)
        yf_ref, yb_ref = oracle.epilogue(acc_ref, sx, sw, bias)
        np.testing.assert_array_equal(host(acc), acc_ref)
        np.testing.assert_array_equal(host(yf), yf_ref)
        np.testing.assert_array_equal(host(yb), yb_ref)
    else:
        yf_ref, _ = oracle.epilogue(oracle.gemm_e4m3(xq, wq), sx, sw, bias)
        rows, cols = np.divmod(np.arange(M * N, dtype=np.int64), N)
        e = fp8_normalized_error(host(yf).reshape(-1), yf_ref.reshape(-1), xq, wq, sx, sw, bias,
                                 rows, cols)
        assert e.max() <= 1e-3, e.max()
        np.testing.assert_array_equal(host(yb), oracle.f32_to_bf16(host(yf)))


def test_split_tiles_leave_workspace_clean_and_match_whole_tiles(monkeypatch):
    """Stream-K split tiles give the same bits as whole tiles (INT8 partial
    sums are exact) and the workspace counters are zero again afterwards."""
    monkeypatch.setenv("SQ_GEMM_FORCE_SPLIT", "1")
    M, N, K = 1000, 2056, 2048
    xq = synth.random_matrix((M, K), np.int8, seed=41)
    wq = synth.random_matrix((N, K), np.int8, seed=42)
    sx = synth.random_floats(M, seed=43, lo=1e-3, hi=0.5)
    sw = synth.random_floats(N, seed=44, lo=1e-4, hi=1e-2)
    d = [dev(a) for a in (xq, sx, wq, sw)]
    ref = oracle.epilogue(oracle.gemm_i8(xq, wq), sx, sw)[0]
    for tile in ops.GEMM_TILES:
        with ops.gemm_tile(tile):
            for _ in range(3):
                y = ops.gemm_w8a8(*d, out_dtype=torch.float32, split=True)
                np.testing.assert_array_equal(host(y), ref)
        assert ops.device_status() == ops.SQ_OK
        counters = host(ops.workspace()[:4096])
        assert not counters.any(), tile


def test_gemm_w8a8_extreme_accumulators():
    M, N, K = 130, 136, 16384
    xq = np.full((M, K), 127, np.int8)
    xq[1::2] = -127
    wq = np.full((N, K), 127, np.int8)
    wq[5] = -127
    wq[7] = 0
    wq[7, 1234] = 1
    sx = np.ones(M, np.float32)
    sw = np.ones(N, np.float32)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    ops.gemm_w8a8(dev(xq), dev(sx), dev(wq), dev(sw), out_dtype=torch.float32, acc=acc)
    a = host(acc)
    assert a[0, 0] == K * 127 * 127 and a[1, 0] == -K * 127 * 127 and a[1, 5] == K * 127 * 127
    assert a[0, 7] == 127 and a[1, 7] == -127
    np.testing.assert_array_equal(a, oracle.gemm_i8(xq, wq))


def test_gemm_w8a8_maximum_k():
    """The largest K the int32 accumulator admits (K * 127^2 < 2^31, K a
    multiple of 16): all-extreme rows reach +-2,147,350,544 exactly, and the
    K tail (K mod 128 = 16) is summed."""
    M, N, K = 3, 16, 133136
    assert K * 127 * 127 < 2 ** 31 <= (K + 16) * 127 * 127
    xq = np.full((M, K), 127, np.int8)
    xq[1] = -127
    xq[2] = synth.random_matrix((1, K), np.int8, seed=91)[0]
    wq = np.full((N, K), 127, np.int8)
    wq[3] = -127
    wq[4] = synth.random_matrix((1, K), np.int8, seed=92)[0]
    wq[5] = 0
    wq[5, K - 1] = 7                   # only the last element of the tail
    sx = np.ones(M, np.float32)
    sw = np.ones(N, np.float32)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    ops.gemm_w8a8(dev(xq), dev(sx), dev(wq), dev(sw), out_dtype=torch.float32, acc=acc)
    assert ops.device_status() == ops.SQ_OK
    a = host(acc)
    assert a[0, 0] == K * 127 * 127 and a[1, 0] == -K * 127 * 127 and a[0, 3] == -K * 127 * 127
    assert a[0, 5] == 7 * 127 and a[1, 5] == -7 * 127
    np.testing.assert_array_equal(a, oracle.gemm_i8(xq, wq))


def test_gemm_does_not_write_outside_output():
    M, N, K = 100, 72, 64
    xq = synth.random_matrix((M, K), np.int8, seed=11)
    wq = synth.random_matrix((N, K), np.int8, seed=12)
    sx = synth.random_floats(M, seed=13, lo=0.01, hi=0.1)
    sw = synth.random_floats(N, seed=14, lo=0.01, hi=0.1)
    guard = 4096
    buf = torch.full((M * N + 2 * guard,), -7777.0, dtype=torch.float32, device="cuda")
    out = buf[guard:guard + M * N].view(M, N)
    ops.gemm_w8a8(dev(xq), dev(sx), dev(wq), dev(sw), out=out)
    h = host(buf)
    assert (h[:guard] == -7777.0).all() and (h[guard + M * N:] == -7777.0).all()
    np.testing.assert_array_equal(host(out), oracle.epilogue(oracle.gemm_i8(xq, wq), sx, sw)[0])


# ------------------------------------------------------------------ a7 FP8 --

@pytest.mark.parametrize("M,N,K", [(1, 16, 32), (17, 64, 64), (129, 200, 96), (300, 392, 4096),
                                   (256, 256, 14336)])
@pytest.mark.parametrize("with_bias", [False, True])
def test_gemm_fp8(M, N, K, with_bias):
    g = np.random.default_rng(M * N + K)
    mag = np.abs(oracle.e4m3_decode(E4M3_FINITE))
    codes = E4M3_FINITE[(mag <= 64.0)]
    xq = g.choice(codes, size=(M, K)).astype(np.uint8)
    wq = g.choice(codes, size=(N, K)).astype(np.uint8)
    sx = synth.random_floats(M, seed=21, lo=1e-3, hi=0.5)
    sw = synth.random_floats(N, seed=22, lo=1e-4, hi=1e-2)
    bias = synth.to_bf16_bits(synth.random_floats(N, seed=23, std=0.1)) if with_bias else None
    acc_ref = oracle.gemm_e4m3(xq, wq)
    yf_ref, _ = oracle.epilogue(acc_ref, sx, sw, bias)
    yf = ops.gemm_fp8(dev(xq), dev(sx), dev(wq), dev(sw), bias=None if bias is None else dev(bias),
                      out_dtype=torch.float32)
    yb = ops.gemm_fp8(dev(xq), dev(sx), dev(wq), dev(sw), bias=None if bias is None else dev(bias))
    assert ops.device_status() == ops.SQ_OK
    rows, cols = np.divmod(np.arange(M * N, dtype=np.int64), N)
    e = fp8_normalized_error(host(yf).reshape(-1), yf_ref.reshape(-1), xq, wq, sx, sw, bias, rows, cols)
    assert e.max() <= 1e-3, e.max()
    # the bf16 output is the nearest-even rounding of the same binary32 values
    # (the tensor-core summation order is fixed for a given launch shape)
    np.testing.assert_array_equal(host(yb), oracle.f32_to_bf16(host(yf)))


# ------------------------------------------- few tokens: weight streaming --

SKINNY_SHAPES = [(1, 8, 16), (5, 136, 1040), (16, 1000, 208), (16, 4096, 8192), (3, 28672, 256)]


@pytest.mark.parametrize("M,N,K", SKINNY_SHAPES)
@pytest.mark.parametrize("with_bias", [False, True])
def test_gemm_few_tokens_int8(M, N, K, with_bias, monkeypatch):
    """M <= 16 runs the weight-streaming kernel (operand roles swapped): int32
    accumulators, binary32 and bf16 outputs bit for bit against the oracle
    and against the tiled kernel forced on the same inputs."""
    xq = synth.random_matrix((M, K), np.int8, seed=M + 3 * K)
    wq = synth.random_matrix((N, K), np.int8, seed=N + 5 * K)
    xq[0, :8] = 127
    wq[:, :8] = -127
    sx = synth.random_floats(M, seed=31, lo=1e-3, hi=0.5)
    sw = synth.random_floats(N, seed=32, lo=1e-4, hi=1e-2)
    bias = synth.to_bf16_bits(synth.random_floats(N, seed=33, std=0.1)) if with_bias else None
    acc_ref = oracle.gemm_i8(xq, wq)
    yf_ref, yb_ref = oracle.epilogue(acc_ref, sx, sw, bias)
    d = [dev(a) for a in (xq, sx, wq, sw)]
    b = None if bias is None else dev(bias)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    yf = ops.gemm_w8a8(*d, bias=b, out_dtype=torch.float32, acc=acc)
    yb = ops.gemm_w8a8(*d, bias=b, out_dtype=torch.bfloat16)
    yn = ops.gemm_w8a8_noalloc(*d, bias=b)
    assert ops.device_status() == ops.SQ_OK
    np.testing.assert_array_equal(host(acc), acc_ref)
    np.testing.assert_array_equal(host(yf), yf_ref)
    np.testing.assert_array_equal(host(yb), yb_ref)
    np.testing.assert_array_equal(host(yn), yb_ref)
    monkeypatch.setenv("SQ_GEMM_TILE", "c1n128")
    yt = ops.gemm_w8a8(*d, bias=b, out_dtype=torch.bfloat16)
    assert torch.equal(yt.view(torch.int16), yb.view(torch.int16))


@pytest.mark.parametrize("M,N,K", SKINNY_SHAPES)
def test_gemm_few_tokens_fp8(M, N, K):
    g = np.random.default_rng(M * 7 + N + K)
    mag = np.abs(oracle.e4m3_decode(E4M3_FINITE))
    codes = E4M3_FINITE[(mag <= 64.0)]
    xq = g.choice(codes, size=(M, K)).astype(np.uint8)
    wq = g.choice(codes, size=(N, K)).astype(np.uint8)
    sx = synth.random_floats(M, seed=34, lo=1e-3, hi=0.5)
    sw = synth.random_floats(N, seed=35, lo=1e-4, hi=1e-2)
    bias = synth.to_bf16_bits(synth.random_floats(N, seed=36, std=0.1))
    yf_ref, _ = oracle.epilogue(oracle.gemm_e4m3(xq, wq), sx, sw, bias)
    yf = ops.gemm_fp8(dev(xq), dev(sx), dev(wq), dev(sw), bias=dev(bias), out_dtype=torch.float32)
    yb = ops.gemm_fp8(dev(xq), dev(sx), dev(wq), dev(sw), bias=dev(bias))
    assert ops.device_status() == ops.SQ_OK
    if M * N <= 50000:
        rows, cols = np.divmod(np.arange(M * N, dtype=np.int64), N)
    else:
        rows, cols = sample_points(M, N, seed=37)
    yfh = host(yf)
    e = fp8_normalized_error(yfh[rows, cols], yf_ref[rows, cols], xq, wq, sx, sw, bias, rows, cols)
    assert e.max() <= 1e-3, e.max()
    np.testing.assert_array_equal(host(yb), oracle.f32_to_bf16(yfh))


def test_gemm_few_tokens_does_not_write_outside_output():
    M, N, K = 7, 200, 96
    xq = synth.random_matrix((M, K), np.int8, seed=41)
    wq = synth.random_matrix((N, K), np.int8, seed=42)
    sx = synth.random_floats(M, seed=43, lo=0.01, hi=0.1)
    sw = synth.random_floats(N, seed=44, lo=0.01, hi=0.1)
    guard = 4096
    buf = torch.full((M * N + 2 * guard,), -7777.0, dtype=torch.float32, device="cuda")
    out = buf[guard:guard + M * N].view(M, N)
    ops.gemm_w8a8(dev(xq), dev(sx), dev(wq), dev(sw), out=out)
    h = host(buf)
    assert (h[:guard] == -7777.0).all() and (h[guard + M * N:] == -7777.0).all()
    np.testing.assert_array_equal(host(out), oracle.epilogue(oracle.gemm_i8(xq, wq), sx, sw)[0])


# --------------------------------------------------------- the whole layer --

@pytest.mark.parametrize("qtype", ["i8", "e4m3"])
def test_linear_matches_oracle(qtype):
    M, K, N = 77, 320, 136
    x = _x((M, K), seed=99, dtype="bf16")
    w = synth.to_bf16_bits(synth.random_floats((K, N), seed=98, std=0.02))
    bias = synth.to_bf16_bits(synth.random_floats(N, seed=97, std=0.01))
    qt = oracle.E4M3 if qtype == "e4m3" else oracle.INT8
    s = oracle.smooth_factors(oracle.amax(x, True), oracle.amax(w, False), 0.5)
    wq, sw = oracle.quantize_weight(w, s, qt)
    ref = oracle.linear(x, s, wq, sw, bias, qt)
    y = ops.linear(dev(x), dev(s), dev(wq), dev(sw), dev(bias), qtype, out_dtype=torch.float32,
                   s_inv=dev(reciprocals(s)))
    assert ops.device_status() == ops.SQ_OK
    if qtype == "i8":
        np.testing.assert_array_equal(host(y), ref["y_f32"])
    else:
        rows, cols = np.divmod(np.arange(M * N, dtype=np.int64), N)
        e = fp8_normalized_error(host(y).reshape(-1), ref["y_f32"].reshape(-1), ref["xq"], wq,
                                 ref["sx"], sw, bias, rows, cols)
        assert e.max() <= 1e-3


def test_prepare_pipeline_matches_oracle():
    x_cal = _x((64, 256), seed=5, dtype="bf16")
    w = synth.to_bf16_bits(synth.random_floats((256, 64), seed=6, std=0.02))
    p = ops.prepare(dev(w), dev(x_cal), alpha=0.5, qtype="i8")
    ax, aw = oracle.amax(x_cal, True), oracle.amax(w, False)
    np.testing.assert_array_equal(host(p["amax_x"]), ax)
    np.testing.assert_array_equal(host(p["amax_w"]), aw)
    s = oracle.smooth_factors(ax, aw, 0.5)
    assert ulp_distance(host(p["s"]), s).max() <= 2
    np.testing.assert_array_equal(host(p["s_inv"]), reciprocals(host(p["s"])))


def test_fast_division_is_exact_on_every_bf16_significand():
    """The reciprocal-product division used for bf16 activations equals the
    IEEE division on all 2^30 (x, s) significand pairs, both signs."""
    assert ops.selftest_fast_division() == 0


@pytest.mark.parametrize("qtype", ["i8", "e4m3"])
def test_quantize_act_fast_path_edge_values(qtype):
    """bf16 rows with zeros of both signs, subnormals, huge values, exact
    ties after smoothing, and smoothing factors outside the fast window."""
    K = 256
    g = np.random.default_rng(77)
    x = (g.standard_normal((6, K)) * 3).astype(np.float32)
    x[0, :8] = [0.0, -0.0, 1e-40, -1e-40, 3e38, -3e38, 2.0 ** -130, 1.0]
    x[1] = np.float32(2.0) ** g.integers(-20, 20, K).astype(np.float32)
    x[2] = 0.0
    x[3, :4] = [127.0, 63.5, -0.5, 1.5]
    x[4] *= 1e-38
    s = synth.random_floats(K, seed=78, lo=0.05, hi=20.0)
    # channels 1..3 lie outside the fast-division window; no quotient overflows
    s[:4] = [1.0, 2.0 ** -30, 2.0 ** 30, 2.0 ** -25]
    s[4:8] = 2.0 ** g.integers(0, 5, 4).astype(np.float32)
    xb = synth.to_bf16_bits(x)
    qt = oracle.E4M3 if qtype == "e4m3" else oracle.INT8
    for smooth, inv in ((s, reciprocals(s)), (s, None), (None, None)):
        xq_ref, sx_ref = oracle.quantize_act(xb, smooth, qt)
        xq, sx = ops.quantize_act(dev(xb), None if smooth is None else dev(smooth), qtype,
                                  s_inv=None if inv is None else dev(inv))
        np.testing.assert_array_equal(host(sx), sx_ref)
        np.testing.assert_array_equal(host(xq).view(np.uint8), xq_ref.view(np.uint8))


@pytest.mark.parametrize("qtype", ["i8", "e4m3"])
@pytest.mark.parametrize("K", [64, 208, 4096, 4112, 14336, 16384])
def test_quantize_act_streaming_rows_edge_values(qtype, K):
    """Many bf16 rows (the persistent streaming kernel): ordinary rows mixed
    with rows that leave its fast window (all zeros, all -0, tiny, huge,
    subnormal) and rows whose elements are zeros of both signs, tiny values
    or exact ties after smoothing; once with every smoothing factor inside
    the fast-division window, once with some outside it, once unsmoothed."""
    M = 700
    g = np.random.default_rng(K)
    x = (g.standard_normal((M, K)) * 3).astype(np.float32)
    x[5] = 0.0
    x[6] = -0.0
    x[7] *= 1e-25                      # amax below the fast window
    x[8] *= 1e28                       # amax above it; no quotient overflows,
    x[8, 20] = 3e31                    # inputs must keep every x/s finite
    x[8, 40] = 1e28
    x[9] = 1e-40                       # subnormal bf16 everywhere
    x[10, :8] = [0.0, -0.0, 1e-30, -1e-30, 1e-40, -1e-40, 2.0 ** -100, -(2.0 ** -90)]
    x[11, ::3] = -0.0
    x[12, :6] = [127.0, 63.5, -0.5, 1.5, 2.5, -126.5]   # ties when s_k = 1
    x[13:20] = np.round(x[13:20] * 2) / 2                # many half-integers
    x[20, -1] = 300.0                                    # amax in the last chunk
    s_in = synth.random_floats(K, seed=K + 3, lo=0.05, hi=20.0)
    s_in[:6] = 1.0
    s_in[6:14] = 2.0 ** g.integers(-3, 4, 8).astype(np.float32)
    # row 12: |x/s| <= ~50 beyond its first six elements, so its amax is 127
    x[12, 6:] = np.clip(x[12, 6:], -1, 1) * s_in[6:] * 50
    s_out = s_in.copy()
    s_out[min(K - 1, 40)] = 2.0 ** -30                   # outside [2^-20, 2^20]
    xb = synth.to_bf16_bits(x)
    qt = oracle.E4M3 if qtype == "e4m3" else oracle.INT8
    # with and without the caller's reciprocals (rows longer than 8192 take a
    # different form when they are given)
    for smooth, inv in ((s_in, None), (s_out, None), (None, None), (s_in, reciprocals(s_in)),
                        (s_out, reciprocals(s_out))):
        xq_ref, sx_ref = oracle.quantize_act(xb, smooth, qt)
        xq, sx = ops.quantize_act(dev(xb), None if smooth is None else dev(smooth), qtype,
                                  s_inv=None if inv is None else dev(inv))
        assert ops.device_status() == ops.SQ_OK
        np.testing.assert_array_equal(host(sx), sx_ref)
        np.testing.assert_array_equal(host(xq).view(np.uint8), xq_ref.view(np.uint8))


@pytest.mark.parametrize("qtype", ["i8", "e4m3"])
@pytest.mark.parametrize("M,K", [(40000, 1024), (12000, 4096), (9000, 4112), (5000, 8192),
                                 (2000, 14336)])
def test_quantize_act_many_rows_per_cta(qtype, M, K):
    """Enough rows that every persistent CTA of the many-row kernel handles
    many of them (its ring slots are refilled and its per-row buffers reused
    several times), with the edge rows of the test above repeated every 500
    rows; with and without the caller's reciprocals."""
    g = np.random.default_rng(M + K)
    x = (g.standard_normal((M, K)) * 3).astype(np.float32)
    ch = g.choice(K, size=K // 100, replace=False)
    x[:, ch] *= g.uniform(20, 100, ch.size).astype(np.float32)
    for r0 in range(0, M - 16, 500):
        x[r0 + 0] = 0.0
        x[r0 + 1] = -0.0
        x[r0 + 2] *= 1e-25
        x[r0 + 3] *= 1e28
        x[r0 + 4] = 1e-40
        x[r0 + 5, :8] = [0.0, -0.0, 1e-30, -1e-30, 1e-40, -1e-40, 2.0 ** -100, -(2.0 ** -90)]
        x[r0 + 6, :6] = [127.0, 63.5, -0.5, 1.5, 2.5, -126.5]
        x[r0 + 7:r0 + 12] = np.round(x[r0 + 7:r0 + 12] * 2) / 2
        x[r0 + 12, -1] = 3000.0
    s = synth.random_floats(K, seed=K + 5, lo=0.05, hi=20.0)
    s[:6] = 1.0
    xb = synth.to_bf16_bits(x)
    qt = oracle.E4M3 if qtype == "e4m3" else oracle.INT8
    xd = dev(xb)
    for smooth, inv in ((s, reciprocals(s)), (s, None), (None, None)):
        xq_ref, sx_ref = oracle.quantize_act(xb, smooth, qt)
        xq, sx = ops.quantize_act(xd, None if smooth is None else dev(smooth), qtype,
                                  s_inv=None if inv is None else dev(inv))
        assert ops.device_status() == ops.SQ_OK
        np.testing.assert_array_equal(host(sx), sx_ref)
        np.testing.assert_array_equal(host(xq).view(np.uint8), xq_ref.view(np.uint8))


# ---------------------------------------------------------- failure path --

def test_bounded_wait_reports_timeout_and_context_survives():
    assert ops.device_status() == ops.SQ_OK
    ops.probe_wait_timeout(20_000_000)  # 20 ms
    assert ops.device_status() == ops.SQ_ERR_TIMEOUT
    assert ops.device_status() == ops.SQ_OK  # read-and-clear
    # the context is still usable
    x = _x((4, 64), seed=1, dtype="bf16")
    xq, sx = ops.quantize_act(dev(x), None, "i8")
    np.testing.assert_array_equal(host(xq), oracle.quantize_act(x, None)[0])
