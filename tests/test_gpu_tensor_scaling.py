"""Per-tensor activation scaling ("Weight-Activation Quantization" §4:
per-tensor scaling online, or delayed from the previous step's max) on the
GPU against the CPU oracle: codes, the broadcast scale and the tensor max
bit for bit, for both code types, both input types, with and without
smoothing, on ragged and full-width shapes, plus the edge cases of delayed
scaling (saturation, a zero or out-of-window scale, tiny and signed-zero
inputs) and a two-step delayed sequence.
"""
import numpy as np
import pytest
import torch

import oracle
from w8a8_smoothquant_int8_02_b200 import ops, synth

from _gpu_util import dev, host

pytestmark = pytest.mark.gpu

Q = {"i8": np.float32(127.0), "e4m3": np.float32(448.0)}


def _qt(qtype):
    return oracle.E4M3 if qtype == "e4m3" else oracle.INT8


def _check(x, s, qtype, amax_prev=None, s_inv=None):
    """Run both sides; returns the GPU's tensor max for chaining."""
    scale = None if amax_prev is None else np.float32(amax_prev) / Q[qtype]
    xq_ref, used, amax_ref = oracle.quantize_act_tensor(x, s, _qt(qtype), scale=scale)
    prev_d = None if amax_prev is None else torch.tensor([amax_prev], dtype=torch.float32,
                                                         device="cuda")
    xq, sx, amax = ops.quantize_act_tensor(dev(x), None if s is None else dev(s), qtype,
                                           amax_prev=prev_d,
                                           s_inv=None if s_inv is None else dev(s_inv))
    assert ops.device_status() == ops.SQ_OK
    M = x.shape[0]
    np.testing.assert_array_equal(host(sx), np.full(M, used, np.float32))
    assert host(amax)[0] == amax_ref, (host(amax)[0], amax_ref)
    np.testing.assert_array_equal(host(xq).view(np.uint8), xq_ref.view(np.uint8))
    return host(amax)[0]


def _x(shape, seed, dtype):
    g = np.random.default_rng(seed)
    x = (g.standard_normal(shape) * 2).astype(np.float32)
    ch = g.choice(shape[1], size=max(1, shape[1] // 64), replace=False)
    x[:, ch] *= g.uniform(20, 100, ch.size).astype(np.float32)
    return synth.to_bf16_bits(x) if dtype == "bf16" else x


def _reciprocals(s):
    s = np.asarray(s, np.float32)
    inside = (s >= np.float32(2.0 ** -20)) & (s <= np.float32(2.0 ** 20))
    return np.where(inside, np.float32(1.0) / np.where(inside, s, 1), np.float32(np.nan)).astype(np.float32)


@pytest.mark.parametrize("qtype", ["i8", "e4m3"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("smooth", [True, False])
@pytest.mark.parametrize("M,K", [(1, 64), (37, 208), (700, 4096), (16, 8192), (300, 14336),
                                 (3, 65536)])
def test_online_and_delayed(qtype, dtype, smooth, M, K):
    x = _x((M, K), seed=M + K, dtype=dtype)
    s = synth.random_floats(K, seed=K + 5, lo=0.05, hi=20.0) if smooth else None
    amax = _check(x, s, qtype)                                   # online
    _check(x, s, qtype, amax_prev=amax * np.float32(0.5),        # delayed: half the max, saturates
           s_inv=None if s is None else _reciprocals(s))
    _check(x, s, qtype, amax_prev=amax * np.float32(3.0))        # delayed: headroom


@pytest.mark.parametrize("qtype", ["i8", "e4m3"])
def test_delayed_edge_cases(qtype):
    K = 256
    g = np.random.default_rng(21)
    x = (g.standard_normal((40, K)) * 3).astype(np.float32)
    x[0, :8] = [0.0, -0.0, 1e-30, -1e-30, 1e-40, -1e-40, 2.0 ** -100, -(2.0 ** -90)]
    x[1] = -0.0
    x[2, :6] = [127.0, 63.5, -0.5, 1.5, 2.5, -126.5]
    x[3] *= 1e-20
    xb = synth.to_bf16_bits(x)
    s = synth.random_floats(K, seed=22, lo=0.05, hi=20.0)
    s[:6] = 1.0
    for amax_prev in (np.float32(127.0), np.float32(0.0), np.float32(1e-3), np.float32(2.0 ** 110),
                      np.float32(2.0 ** -70), np.float32(448.0)):
        _check(xb, None, qtype, amax_prev=amax_prev)
        _check(xb, s, qtype, amax_prev=amax_prev)
    # a smoothing factor outside the fast-division window
    s2 = s.copy()
    s2[40] = 2.0 ** -30
    _check(xb, s2, qtype, amax_prev=np.float32(50.0))


def test_two_delayed_steps_chain_the_max():
    """Step 1 online on one batch, step 2 on the next batch with step 1's max:
    each output feeds the next step exactly as the oracle's scale does."""
    x1 = _x((512, 1024), seed=31, dtype="bf16")
    x2 = _x((512, 1024), seed=32, dtype="bf16")
    a1 = _check(x1, None, "e4m3")
    a2 = _check(x2, None, "e4m3", amax_prev=a1)
    _check(x1, None, "e4m3", amax_prev=a2)


def test_empty_batch_sets_the_max_to_zero():
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    out = torch.full((1,), 7.0, dtype=torch.float32, device="cuda")
    xq, sx, amax = ops.quantize_act_tensor(x, None, "e4m3", amax_out=out)
    assert xq.shape == (0, 64) and sx.shape == (0,)
    assert host(amax)[0] == 0.0
    assert ops.device_status() == ops.SQ_OK


def test_module_delayed_scaling_over_calls():
    """SmoothQuantLinear(act_scaling='tensor', smooth=False): the first call
    scales by the calibration max, each later call by the previous call's
    max; outputs against the oracle (exact E4M3 sums, normalized error)."""
    from w8a8_smoothquant_int8_02_b200.ops import SmoothQuantLinear
    from _gpu_util import fp8_normalized_error
    K, N = 512, 384
    g = np.random.default_rng(41)
    w = (g.standard_normal((K, N)) * 0.02).astype(np.float32)
    x_cal = _x((64, K), seed=42, dtype="bf16")
    batches = [_x((96, K), seed=43 + i, dtype="bf16") for i in range(3)]
    layer = SmoothQuantLinear(dev(synth.to_bf16_bits(w)), dev(x_cal), qtype="e4m3",
                              act_scaling="tensor", smooth=False)
    wb = synth.to_bf16_bits(w)
    wq_ref, sw_ref = oracle.quantize_weight(wb, None, oracle.E4M3)
    _, _, prev = oracle.quantize_act_tensor(x_cal, None, oracle.E4M3)
    for xb in batches:
        assert host(layer.last_amax)[0] == prev
        y = layer(dev(xb), out_dtype=torch.float32)
        scale = np.float32(prev) / np.float32(448.0)
        xq_ref, used, prev = oracle.quantize_act_tensor(xb, None, oracle.E4M3, scale=scale)
        rows, cols = np.divmod(np.arange(96 * N, dtype=np.int64), N)
        sx_ref = np.full(96, used, np.float32)
        _, yf_ref, _ = oracle.linear_at(xq_ref, sx_ref, wq_ref, sw_ref, None, rows, cols,
                                        oracle.E4M3)
        got = host(y)[rows, cols]
        e = fp8_normalized_error(got, yf_ref, xq_ref, wq_ref, sx_ref, sw_ref, None, rows, cols)
        assert e.max() <= 1e-3, e.max()
    assert ops.device_status() == ops.SQ_OK
