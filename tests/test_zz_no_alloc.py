"""The allocation-free GEMM entry point (sq_gemm_w8a8_noalloc).

Some callers cannot allocate device memory while they run (a runtime that
reserves all device memory for its own pool, or latency-critical code that
cannot afford cudaMalloc's synchronization), so they cannot hand the GEMM a
workspace; this entry point uses a fixed array inside the library instead.
The test calls it through the C ABI twice in a row and checks each output
against the existing entry point (sq_gemm_w8a8 with a caller workspace):
INT8 results must agree bit for bit, the tolerance all INT8 GEMM tests use.
It is named to run last and also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from w8a8_smoothquant_int8_02_b200 import ops, synth

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("M,N,K,out_dtype", [(1000, 2056, 2048, torch.float32),
                                             (4096, 4096, 1024, torch.bfloat16)])
def test_noalloc_matches_workspace_entry_point_twice(M, N, K, out_dtype):
    lib = ops.load()
    xq = _dev(synth.random_matrix((M, K), np.int8, seed=71))
    wq = _dev(synth.random_matrix((N, K), np.int8, seed=72))
    sx = _dev(synth.random_floats(M, seed=73, lo=1e-3, hi=0.5))
    sw = _dev(synth.random_floats(N, seed=74, lo=1e-4, hi=1e-2))
    bias = torch.from_numpy(synth.to_bf16_bits(synth.random_floats(N, seed=75, std=0.1))
                            .view(np.int16)).view(torch.bfloat16).cuda()
    ref = ops.gemm_w8a8(xq, sx, wq, sw, bias, out_dtype=out_dtype, split=True)
    yt = ops.SQ_F32 if out_dtype == torch.float32 else ops.SQ_BF16
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    P = ctypes.c_void_p
    for call in range(2):
        y = torch.full((M, N), float("nan"), dtype=out_dtype, device="cuda")
        st = lib.sq_gemm_w8a8_noalloc(P(xq.data_ptr()), P(sx.data_ptr()), P(wq.data_ptr()),
                                      P(sw.data_ptr()), P(bias.data_ptr()), M, N, K,
                                      P(y.data_ptr()), yt, stream)
        assert st == ops.SQ_OK, ops.status_string(st)
        assert ops.device_status() == ops.SQ_OK
        assert torch.equal(y.view(torch.int32 if out_dtype == torch.float32 else torch.int16),
                           ref.view(torch.int32 if out_dtype == torch.float32 else torch.int16)), call
