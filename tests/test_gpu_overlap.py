"""Activation passes that overlap the previous batch's GEMM (SQ_OVERLAP_PREVIOUS).

Consecutive independent batches, each: the activation pass (smoothing +
per-token quantization, or the fused RMS normalization + quantization) into
one of two code buffers, then the 8-bit GEMM on it. With the flag the pass of
batch i+1 may start while the GEMM of batch i is still running (its last
round of tiles leaves SMs idle) and completes after it. Every batch's codes,
scales and GEMM output must equal those of the same calls without the flag,
and the first batch's codes the oracle's.
"""
import numpy as np
import pytest
import torch

import oracle
from w8a8_smoothquant_int8_02_b200 import ops, synth

from _gpu_util import dev, host

pytestmark = pytest.mark.gpu


def _batches(n, M, K, seed):
    return [synth.to_bf16_bits(synth.random_floats((M, K), seed=seed + i, std=1.0 + i))
            for i in range(n)]


def _run(kind, xs, s, g, wq, sw, qt, overlap, n_buf=2):
    M, K = xs[0].shape
    xqs = [torch.empty((M, K), dtype=torch.int8 if qt == "i8" else torch.uint8, device="cuda")
           for _ in range(n_buf)]
    sxs = [torch.empty(M, dtype=torch.float32, device="cuda") for _ in range(n_buf)]
    gemm = ops.gemm_w8a8 if qt == "i8" else ops.gemm_fp8
    xd = [dev(x) for x in xs]
    ys = [torch.empty((M, wq.shape[0]), dtype=torch.float32, device="cuda") for _ in xs]
    torch.cuda.synchronize()
    # nothing but the two calls per batch on the stream, so that each pass
    # follows the previous batch's GEMM directly
    for i, x in enumerate(xd):
        b = i % n_buf
        if kind == "norm":
            ops.rmsnorm_quantize_act(x, g, 1e-5, qt, xq=xqs[b], sx=sxs[b], overlap=overlap)
        else:
            ops.quantize_act(x, s, qt, xq=xqs[b], sx=sxs[b], overlap=overlap)
        gemm(xqs[b], sxs[b], wq, sw, out=ys[i])
    torch.cuda.synchronize()
    assert ops.device_status() == ops.SQ_OK
    # the buffers hold the last n_buf batches' codes, in batch order
    last = [(len(xs) - n_buf + j) % n_buf for j in range(n_buf)]
    return ys, [xqs[b] for b in last], [sxs[b] for b in last]


@pytest.mark.parametrize("kind", ["smooth", "norm"])
@pytest.mark.parametrize("qt", ["i8", "e4m3"])
def test_overlapped_passes_match_serial(kind, qt):
    # 2048 tokens: the many-row forms of both passes; N = 4096: the persistent
    # GEMM in more than one round of tiles, so its last round leaves SMs idle
    M, K, N = 2048, 1024, 4096
    xs = _batches(6, M, K, seed=300)
    w = synth.random_floats((K, N), seed=301, std=0.02)
    s = synth.random_floats(K, seed=302, lo=0.5, hi=4.0)
    gamma = synth.random_floats(K, seed=303, lo=0.5, hi=2.0)
    qcode = oracle.INT8 if qt == "i8" else oracle.E4M3
    wq, sw = oracle.quantize_weight(w, None, qcode)
    wq_d, sw_d, s_d, g_d = dev(wq), dev(sw), dev(s), dev(gamma)
    ref = _run(kind, xs, s_d, g_d, wq_d, sw_d, qt, overlap=False)
    got = _run(kind, xs, s_d, g_d, wq_d, sw_d, qt, overlap=True)
    for i in range(len(xs)):
        np.testing.assert_array_equal(host(got[0][i]).view(np.uint32),
                                      host(ref[0][i]).view(np.uint32))
    for j in range(2):
        np.testing.assert_array_equal(host(got[1][j]).view(np.uint8), host(ref[1][j]).view(np.uint8))
        np.testing.assert_array_equal(host(got[2][j]), host(ref[2][j]))
    # the last batch against the oracle: codes, scales, and the INT8 output
    if kind == "norm":
        q5, s5, _, _ = oracle.rmsnorm_quantize_act(xs[-1], gamma, 1e-5, qcode)
    else:
        q5, s5 = oracle.quantize_act(xs[-1], s, qcode)
    np.testing.assert_array_equal(host(got[1][1]).view(np.uint8), q5.view(np.uint8))
    np.testing.assert_array_equal(host(got[2][1]), s5)
    if qt == "i8":
        y5, _ = oracle.epilogue(oracle.gemm_i8(q5, wq), s5, sw, None)
        np.testing.assert_array_equal(host(got[0][-1]), y5)


def test_overlap_flag_in_a_graph():
    """The bench's form: steps captured in a CUDA graph with the flag set, two
    code buffers, replayed twice; outputs equal the serial calls."""
    M, K, N = 1024, 2048, 2048
    xs = _batches(4, M, K, seed=310)
    w = synth.random_floats((K, N), seed=311, std=0.02)
    s = synth.random_floats(K, seed=312, lo=0.5, hi=4.0)
    wq, sw = oracle.quantize_weight(w, None)
    wq_d, sw_d, s_d = dev(wq), dev(sw), dev(s)
    ref = _run("smooth", xs, s_d, None, wq_d, sw_d, "i8", overlap=False)
    xd = [dev(x) for x in xs]
    xqs = [torch.empty((M, K), dtype=torch.int8, device="cuda") for _ in range(2)]
    sxs = [torch.empty(M, dtype=torch.float32, device="cuda") for _ in range(2)]
    ys = [torch.empty((M, N), dtype=torch.float32, device="cuda") for _ in range(4)]

    def steps():
        for i in range(4):
            b = i % 2
            ops.quantize_act(xd[i], s_d, "i8", xq=xqs[b], sx=sxs[b], overlap=True)
            ops.gemm_w8a8(xqs[b], sxs[b], wq_d, sw_d, out=ys[i])

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        steps()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        steps()
    for _ in range(2):
        for y in ys:
            y.zero_()
        graph.replay()
        torch.cuda.synchronize()
        for i in range(4):
            np.testing.assert_array_equal(host(ys[i]).view(np.uint32), host(ref[0][i]).view(np.uint32))
    assert ops.device_status() == ops.SQ_OK
