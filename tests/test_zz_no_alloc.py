"""The allocation-free GEMM entry point (sq_gemm_w8a8_noalloc).

Some callers cannot allocate device memory while they run (a runtime that
reserves all device memory for its own pool, or latency-critical code that
cannot afford cudaMalloc's synchronization), so they cannot hand the GEMM a
workspace; this entry point uses a fixed array inside the library instead.
The test calls it through the C ABI twice in a row and checks each output
against the existing entry point (sq_gemm_w8a8 with a caller workspace) and
against the CPU oracle: INT8 results must agree bit for bit, the tolerance
all INT8 GEMM tests use. One case forces a tile shape and a tile count just
above a whole number of waves, so the split tiles (the part that uses the
fixed array) certainly run. It is named to run last and also passes alone in
a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from w8a8_smoothquant_int8_02_b200 import ops, synth

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _bits(t):
    return t.view(torch.int32 if t.dtype == torch.float32 else torch.int16).cpu().numpy()


@pytest.mark.parametrize("M,N,K,out_dtype,tile", [
    (1000, 2056, 2048, torch.float32, None),
    (4096, 4096, 1024, torch.bfloat16, None),
    # 128 x 128 tiles: 7 x 43 = 301 tiles on 148 SMs, two whole waves plus 5
    # tiles, so the last part is split along K through the fixed array
    (896, 5504, 512, torch.float32, "c1n128"),
])
def test_noalloc_matches_workspace_entry_point_twice(M, N, K, out_dtype, tile):
    lib = ops.load()
    xq_h = synth.random_matrix((M, K), np.int8, seed=71)
    wq_h = synth.random_matrix((N, K), np.int8, seed=72)
    sx_h = synth.random_floats(M, seed=73, lo=1e-3, hi=0.5)
    sw_h = synth.random_floats(N, seed=74, lo=1e-4, hi=1e-2)
    bias_h = synth.to_bf16_bits(synth.random_floats(N, seed=75, std=0.1))
    xq, wq, sx, sw = _dev(xq_h), _dev(wq_h), _dev(sx_h), _dev(sw_h)
    bias = torch.from_numpy(bias_h.view(np.int16)).view(torch.bfloat16).cuda()
    yf_ref, yb_ref = oracle.epilogue(oracle.gemm_i8(xq_h, wq_h), sx_h, sw_h, bias_h)
    oracle_bits = yf_ref.view(np.int32) if out_dtype == torch.float32 else yb_ref.view(np.int16)
    yt = ops.SQ_F32 if out_dtype == torch.float32 else ops.SQ_BF16
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    P = ctypes.c_void_p
    with ops.gemm_tile(tile):
        ref = ops.gemm_w8a8(xq, sx, wq, sw, bias, out_dtype=out_dtype, split=True)
        np.testing.assert_array_equal(_bits(ref), oracle_bits)
        for call in range(2):
            y = torch.full((M, N), float("nan"), dtype=out_dtype, device="cuda")
            st = lib.sq_gemm_w8a8_noalloc(P(xq.data_ptr()), P(sx.data_ptr()), P(wq.data_ptr()),
                                          P(sw.data_ptr()), P(bias.data_ptr()), M, N, K,
                                          P(y.data_ptr()), yt, stream)
            assert st == ops.SQ_OK, ops.status_string(st)
            assert ops.device_status() == ops.SQ_OK
            got = _bits(y)
            assert np.array_equal(got, _bits(ref)), call
            np.testing.assert_array_equal(got, oracle_bits)
