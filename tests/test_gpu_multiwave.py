"""GEMM launches in which every CTA computes several output tiles, compared
element by element with the CPU oracle.

The persistent kernel walks tiles in rounds over all SMs; the second and
later tiles of a CTA reuse its tensor-memory accumulators (two buffers,
alternating), flip the phases of every pipeline barrier and move through the
raster groups. The shape here gives every compiled tile shape at least three
tiles per CTA (or SM pair), with ragged M, N and K tails, and runs each with
whole tiles and with the split (stream-K) last wave.

Bar: INT8 -- int32 accumulators, binary32 and bf16 outputs bit for bit
("Weight-Activation Quantization" §3 "Step 2": Y = dequantize(X_int8 @
W_int8)). FP8 -- codes drawn from every finite E4M3 value (magnitudes up to
448, subnormals included, §4 "FP8 W8A8"), binary32 output within 1e-3 of the
exact sum on the normalized metric, and bf16 output the nearest-even
rounding of the binary32 output.
"""
import numpy as np
import pytest
import torch

import oracle
from w8a8_smoothquant_int8_02_b200 import ops, synth

from _gpu_util import dev, fp8_error_denominator, fp8_normalized_error_full, host

pytestmark = pytest.mark.gpu

M, N, K = 2085, 7176, 272           # ragged: M % 128 = 37, N % 8 == 0, K % 128 = 16
SMS = 148
TILE_GEOM = {"c1n128": (1, 128, 128), "c1n224": (1, 128, 224), "c1n256": (1, 128, 256),
             "c2n224": (2, 256, 224), "c2n256": (2, 256, 256)}
E4M3_FINITE = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)


@pytest.fixture(scope="module")
def int8_case():
    xq = synth.random_matrix((M, K), np.int8, seed=501)
    wq = synth.random_matrix((N, K), np.int8, seed=502)
    xq[3, :] = 127                   # extreme rows and columns
    wq[5, :] = -127
    sx = synth.random_floats(M, seed=503, lo=1e-3, hi=0.5)
    sw = synth.random_floats(N, seed=504, lo=1e-4, hi=1e-2)
    bias = synth.to_bf16_bits(synth.random_floats(N, seed=505, std=0.1))
    acc = oracle.gemm_i8(xq, wq)
    yf, yb = oracle.epilogue(acc, sx, sw, bias)
    return dict(xq=xq, wq=wq, sx=sx, sw=sw, bias=bias, acc=acc, yf=yf, yb=yb)


@pytest.fixture(scope="module")
def fp8_case():
    g = np.random.default_rng(506)
    xq = g.choice(E4M3_FINITE, size=(M, K)).astype(np.uint8)
    wq = g.choice(E4M3_FINITE, size=(N, K)).astype(np.uint8)
    xq[7, :] = 0x7E                  # +448 everywhere in one row
    wq[9, :] = 0xFE                  # -448 everywhere in one column
    sx = synth.random_floats(M, seed=507, lo=1e-6, hi=1e-3)
    sw = synth.random_floats(N, seed=508, lo=1e-6, hi=1e-3)
    bias = synth.to_bf16_bits(synth.random_floats(N, seed=509, std=0.1))
    yf, _ = oracle.epilogue(oracle.gemm_e4m3(xq, wq), sx, sw, bias)
    den = fp8_error_denominator(xq, wq, sx, sw, bias)
    return dict(xq=xq, wq=wq, sx=sx, sw=sw, bias=bias, yf=yf, den=den)


def test_shape_gives_every_tile_shape_several_tiles_per_unit():
    for name, (cg, bm, bn) in TILE_GEOM.items():
        tiles = -(-M // bm) * -(-N // bn)
        assert tiles / (SMS // cg) >= 3.0, name


@pytest.fixture
def force_split(monkeypatch):
    """Split the last partial round on every tile shape (the library
    otherwise splits only where it pays)."""
    monkeypatch.setenv("SQ_GEMM_FORCE_SPLIT", "1")


@pytest.mark.parametrize("split", [False, True])
@pytest.mark.parametrize("tile", ops.GEMM_TILES)
def test_int8_multiwave_bit_exact(int8_case, tile, split, force_split):
    c = int8_case
    d = [dev(c[k]) for k in ("xq", "sx", "wq", "sw")]
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    with ops.gemm_tile(tile):
        yf = ops.gemm_w8a8(*d, bias=dev(c["bias"]), out_dtype=torch.float32, acc=acc, split=split)
        yb = ops.gemm_w8a8(*d, bias=dev(c["bias"]), split=split)
    assert ops.device_status() == ops.SQ_OK
    np.testing.assert_array_equal(host(acc), c["acc"])
    np.testing.assert_array_equal(host(yf).view(np.uint32), c["yf"].view(np.uint32))
    np.testing.assert_array_equal(host(yb), c["yb"])


@pytest.mark.parametrize("split", [False, True])
@pytest.mark.parametrize("tile", ops.GEMM_TILES)
def test_fp8_multiwave_full_range_codes(fp8_case, tile, split, force_split):
    c = fp8_case
    d = [dev(c[k]) for k in ("xq", "sx", "wq", "sw")]
    with ops.gemm_tile(tile):
        yf = ops.gemm_fp8(*d, bias=dev(c["bias"]), out_dtype=torch.float32, split=split)
        yb = ops.gemm_fp8(*d, bias=dev(c["bias"]), split=split)
    assert ops.device_status() == ops.SQ_OK
    got = host(yf)
    e = fp8_normalized_error_full(got, c["yf"], den=c["den"])
    assert e.max() <= 1e-3, e.max()
    np.testing.assert_array_equal(host(yb), oracle.f32_to_bf16(got))
