"""The workloads at full size, in the launch configuration bench.py
times (tile shape chosen by problem size), against the CPU oracle.

Per workload: calibration amaxes bit-exact, smoothing factors within 2 ulp,
weight codes / scales and activation codes / scales bit-exact (each GPU
stage fed the oracle's inputs), and every element of the GEMM output
against the oracle's full GEMM and epilogue: bit-exact for INT8, within
1e-3 of the exact sum (normalized) for FP8.
"""
import numpy as np
import pytest
import torch

import oracle
from w8a8_smoothquant_int8_02_b200 import ops, synth, workloads

from _gpu_util import (dev, fp8_normalized_error_full, host, ulp_distance,
                       weight_only_error_denominator)

pytestmark = pytest.mark.gpu


def _reciprocals(s):
    s = np.asarray(s, np.float32)
    inside = (s >= np.float32(2.0 ** -20)) & (s <= np.float32(2.0 ** 20))
    return np.where(inside, np.float32(1.0) / np.where(inside, s, 1), np.float32(np.nan)).astype(np.float32)


def _weight_only_end_to_end(case):
    """Weight-only workloads: per-channel weight codes and scales bit-exact,
    then every output element of the GEMM within 1e-3 of the binary64 product
    (normalized by sw * sum_k |x q| + |bias|), bf16 the rounding of binary32."""
    bits = workloads.WEIGHT_ONLY_BITS[case.qtype]
    d = synth.generate(case)
    x, w, bias = d["x"], d["w"], d["bias"]
    if bits == 8:
        wq_ref, sw_ref = oracle.quantize_weight(w, None)
    else:
        wq_ref, sw_ref = oracle.quantize_weight_i4(w)
    wq_d, sw_d = ops.quantize_weight(dev(w), None, "i8" if bits == 8 else "i4")
    np.testing.assert_array_equal(host(sw_d), sw_ref)
    np.testing.assert_array_equal(host(wq_d).view(np.uint8), wq_ref.view(np.uint8))
    bias_d = None if bias is None else dev(bias)
    xd = dev(x)
    yf = ops.gemm_weight_only(xd, wq_d, sw_d, bias_d, bits, out_dtype=torch.float32)
    yb = ops.gemm_weight_only(xd, wq_d, sw_d, bias_d, bits)
    assert ops.device_status() == ops.SQ_OK
    y_ref = oracle.gemm_weight_only(x, wq_ref, sw_ref, bias, bits)
    codes = wq_ref if bits == 8 else oracle.unpack_i4(wq_ref)
    den = weight_only_error_denominator(x, codes, sw_ref, bias)
    got = host(yf)
    e = np.abs(got.astype(np.float64) - y_ref) / den
    assert e.max() <= 1e-3, e.max()
    np.testing.assert_array_equal(host(yb), oracle.f32_to_bf16(got))


@pytest.mark.parametrize("name", list(workloads.ALL))
def test_workload_end_to_end(name):
    case = workloads.ALL[name]
    if case.qtype in workloads.WEIGHT_ONLY_BITS:
        _weight_only_end_to_end(case)
        return
    qt = oracle.E4M3 if case.qtype == "e4m3" else oracle.INT8
    d = synth.generate(case)
    x, x_cal, w, bias = d["x"], d["x_cal"], d["w"], d["bias"]
    M, K, N = case.M, case.K, case.N

    # ---- offline preparation ----
    w_d = dev(w)
    s = None
    if case.norm_eps:
        # calibration on the normalization's output, s, and the gain with 1/s
        # folded in; the later stages take the oracle's s (stage-wise parity)
        xn_cal = oracle.rmsnorm_quantize_act(x_cal, d["gamma"], case.norm_eps)[3]
        ax = oracle.amax(xn_cal, True)
        aw = oracle.amax(w, False)
        s = oracle.smooth_factors(ax, aw, case.alpha)
        p = ops.prepare_rmsnorm(w_d, dev(x_cal), dev(d["gamma"]), case.norm_eps,
                                alpha=case.alpha, qtype=case.qtype)
        np.testing.assert_array_equal(host(p["amax_x"]), ax)
        np.testing.assert_array_equal(host(p["amax_w"]), aw)
        assert ulp_distance(host(p["s"]), s).max() <= 2
        g_ref = oracle.fold_smoothing(d["gamma"], s)[0]
        g_d = ops.fold_smoothing(dev(d["gamma"]), dev(s))
        np.testing.assert_array_equal(host(g_d), g_ref)
    elif case.smooth:
        ax = oracle.amax(x_cal, True)
        aw = oracle.amax(w, False)
        s = oracle.smooth_factors(ax, aw, case.alpha)
        p = ops.prepare(w_d, dev(x_cal), alpha=case.alpha, qtype=case.qtype)
        np.testing.assert_array_equal(host(p["amax_x"]), ax)
        np.testing.assert_array_equal(host(p["amax_w"]), aw)
        assert ulp_distance(host(p["s"]), s).max() <= 2
    s_d = None if s is None else dev(s)
    s_inv_d = None if s is None else dev(_reciprocals(s))

    wq_ref, sw_ref = oracle.quantize_weight(w, s, qt)
    wq_d, sw_d = ops.quantize_weight(w_d, s_d, case.qtype)
    del w_d
    np.testing.assert_array_equal(host(sw_d), sw_ref)
    np.testing.assert_array_equal(host(wq_d).view(np.uint8), wq_ref.view(np.uint8))

    if case.act_scaling == "tensor":
        # ---- runtime: per-tensor delayed scaling, the first step's max from
        # the calibration tokens (online), then one delayed step ----
        _, _, amax_cal = oracle.quantize_act_tensor(x_cal, s, qt)
        _, _, amax_cal_d = ops.quantize_act_tensor(dev(x_cal), s_d, case.qtype, s_inv=s_inv_d)
        assert host(amax_cal_d)[0] == amax_cal
        scale = np.float32(amax_cal) / np.float32(448.0 if qt == oracle.E4M3 else 127.0)
        xq_ref, used, amax_x = oracle.quantize_act_tensor(x, s, qt, scale=scale)
        sx_ref = np.full(M, used, np.float32)
        xq_d, sx_d, amax_d = ops.quantize_act_tensor(dev(x), s_d, case.qtype, amax_prev=amax_cal_d,
                                                     s_inv=s_inv_d)
        assert host(amax_d)[0] == amax_x
    elif case.norm_eps:
        # ---- runtime: the fused normalization + per-token quantization ----
        xq_ref, sx_ref, _, _ = oracle.rmsnorm_quantize_act(x, g_ref, case.norm_eps, qt)
        xq_d, sx_d = ops.rmsnorm_quantize_act(dev(x), g_d, case.norm_eps, case.qtype)
    else:
        # ---- runtime: activation smoothing + per-token quantization ----
        xq_ref, sx_ref = oracle.quantize_act(x, s, qt)
        xq_d, sx_d = ops.quantize_act(dev(x), s_d, case.qtype, s_inv=s_inv_d)
    np.testing.assert_array_equal(host(sx_d), sx_ref)
    np.testing.assert_array_equal(host(xq_d).view(np.uint8), xq_ref.view(np.uint8))

    # ---- runtime: 8-bit GEMM + epilogue, on the oracle's operands ----
    bias_d = None if bias is None else dev(bias)
    gemm = ops.gemm_w8a8 if case.qtype == "i8" else ops.gemm_fp8
    ops_x, ops_w = dev(xq_ref), dev(wq_ref)
    # as bench.py launches it: with the workspace, the library splitting the
    # last partial round of tiles where that pays
    yf = gemm(ops_x, dev(sx_ref), ops_w, dev(sw_ref), bias_d, out_dtype=torch.float32, split=True)
    yb = gemm(ops_x, dev(sx_ref), ops_w, dev(sw_ref), bias_d, split=True)
    assert ops.device_status() == ops.SQ_OK
    # every output element against the oracle's full GEMM and epilogue
    if case.qtype == "i8":
        acc_ref = oracle.gemm_i8(xq_ref, wq_ref)
        yf_ref, yb_ref = oracle.epilogue(acc_ref, sx_ref, sw_ref, bias)
        del acc_ref
        yf_got = host(yf)
        np.testing.assert_array_equal(yf_got.view(np.uint32), yf_ref.view(np.uint32))
        np.testing.assert_array_equal(host(yb), yb_ref)
    else:
        yf_ref, _ = oracle.epilogue(oracle.gemm_e4m3(xq_ref, wq_ref), sx_ref, sw_ref, bias)
        yf_got = host(yf)
        e = fp8_normalized_error_full(yf_got, yf_ref, xq_ref, wq_ref, sx_ref, sw_ref, bias)
        assert e.max() <= 1e-3, e.max()
        np.testing.assert_array_equal(host(yb), oracle.f32_to_bf16(yf_got))
    del yf_ref

    # ---- the fused forward through one C call (same operands; per-token) ----
    if case.act_scaling == "tensor" or case.norm_eps:
        return
    y2 = ops.linear(dev(x), s_d, ops_w, dev(sw_ref), bias_d, case.qtype,
                    out_dtype=torch.float32, s_inv=s_inv_d, split=True)
    assert ops.device_status() == ops.SQ_OK
    np.testing.assert_array_equal(host(y2).view(np.uint32), yf_got.view(np.uint32))
