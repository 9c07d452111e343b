"""Host-side logic of bench.py (no GPU): the L2-defeating rotation, the
metric names, which activation kernel each workload launches, the
source-hash guard on profiled DRAM traffic, and the reference arm's
arithmetic on a tiny case."""
import importlib.util
import os
import shutil
import sys

import pytest

from w8a8_smoothquant_int8_02_b200 import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name", list(workloads.ALL))
def test_rotation_exceeds_l2(bench, name):
    case = workloads.ALL[name]
    per_set = case.M * case.K * 2 + case.N * case.K
    r = bench.rotate_count(case)
    assert r >= 1
    assert r * per_set >= 1.5 * bench.L2_BYTES or per_set >= 1.5 * bench.L2_BYTES


def test_metric_names(bench):
    assert bench.metric_for(workloads.MLP_UP) == bench.METRIC
    assert "FP8" in bench.metric_for(workloads.FP8_DOWN)
    assert "per-tensor" in bench.metric_for(workloads.FP8_TENSOR)
    assert "M512 K4096 N4096" in bench.metric_for(workloads.PREFILL)
    assert "RMSNorm" in bench.metric_for(workloads.MLP_UP_RMSNORM)


def test_activation_kernel_per_workload(bench):
    assert bench.quant_kernel_name(workloads.TINY) == "quant_act_kernel"              # fp32 input
    assert bench.quant_kernel_name(workloads.MLP_UP) == "quant_act_stream_kernel"
    assert bench.quant_kernel_name(workloads.FP8_DOWN) == "quant_act_stream_kernel"
    assert bench.quant_kernel_name(workloads.DECODE) == "quant_act_fast_kernel"      # 16 rows
    assert bench.quant_kernel_name(workloads.FP8_TENSOR) == "quant_act_tensor_kernel"
    assert bench.quant_kernel_name(workloads.MLP_UP_RMSNORM) == "rmsnorm_quant_warp_kernel"


def test_profiled_traffic_is_guarded_by_the_kernel_source(bench, tmp_path, monkeypatch):
    """Traffic is reported only for a workload that was captured and only
    while the kernel's sources hash as they did at capture time."""
    assert bench.profiled_traffic("gemm", "prefill_512x4096x4096") is None
    # a copy of the tree whose GEMM source differs by one byte reports null
    fake = tmp_path / "root"
    csrc = fake / "w8a8_smoothquant_int8_02_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in ("sq_gemm.cu", "sq_common.cuh", "sq_quant.cu"):
        shutil.copy(os.path.join(ROOT, "w8a8_smoothquant_int8_02_b200", "csrc", f), csrc / f)
    monkeypatch.setattr(bench, "ROOT", str(fake))
    key = ("gemm", "mlp_up_4096x4096x14336")
    if key in bench.PROFILED_TRAFFIC:
        expected = bench.profiled_traffic(*key)
        with open(csrc / "sq_gemm.cu", "a") as f:
            f.write("\n")
        assert bench.profiled_traffic(*key) is None
        assert expected is None or expected > 0


def test_reference_arm_cpu_baseline_on_tiny(bench):
    """The oracle leg runs on a tiny case and reports a positive rate with
    its sample described."""
    from w8a8_smoothquant_int8_02_b200 import synth
    case = workloads.TINY
    d = synth.generate(case)
    out = bench.cpu_baseline(case, d, budget_s=0.05)
    assert out["kind"] == "oracle" and out["value"] > 0 and out["cores"] >= 1
    assert "token rows" in out["sample"]
    tensor = workloads.FP8_TENSOR
    small = synth.LinearCase(**{**tensor.__dict__, "M": 8, "K": 64, "N": 32, "cal_tokens": 16,
                                "name": "fp8_tensor_small"})
    d2 = synth.generate(small)
    out2 = bench.cpu_baseline(small, d2, budget_s=0.05)
    assert out2["value"] > 0
    normed = workloads.MLP_UP_RMSNORM
    small3 = synth.LinearCase(**{**normed.__dict__, "M": 8, "K": 64, "N": 32, "cal_tokens": 16,
                                 "name": "mlp_up_rmsnorm_small"})
    d3 = synth.generate(small3)
    assert d3["gamma"].shape == (64,) and d3["gamma"].min() >= 0.5
    out3 = bench.cpu_baseline(small3, d3, budget_s=0.05)
    assert out3["value"] > 0 and "RMS normalization" in out3["sample"]


def test_reference_arm_line(bench, capsys, monkeypatch):
    """--impl reference prints one JSON line for the selected workload with
    the base contract's keys; ranks other than 0 print nothing."""
    import argparse
    import json
    args = argparse.Namespace(workload="tiny_16x64x64", steps=3, warmup=3, ref_rows=8)
    bench.run_reference(args)
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["metric"] == bench.metric_for(workloads.TINY)
    assert line["config"]["workload"] == "tiny_16x64x64"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.run_reference(args)
    assert capsys.readouterr().out == ""


def test_gemm_roofline_bound_follows_the_ridge_point(bench):
    """The decode shape (few tokens, the weight streamed once) is reported
    against HBM; the MLP-up and prefill shapes against the tensor peak."""
    def entry(case):
        M, K, N = case.M, case.K, case.N
        nbytes = M * K + N * K + M * N * 2 + 4 * (M + N)
        return bench.gemm_roofline(case.ops, nbytes, 0.1, 3285.6, 2840.0, 6538.0, None)
    assert entry(workloads.DECODE)["bound"] == "hbm"
    assert entry(workloads.DECODE)["unit"] == "GB/s"
    assert entry(workloads.MLP_UP)["bound"] == "tensor"
    assert entry(workloads.PREFILL)["bound"] == "tensor"
    e = entry(workloads.MLP_UP)
    assert abs(e["frac"] - e["achieved"] / 3285.6) < 1e-12


def test_gemm_kernel_per_workload(bench):
    """At most 16 tokens run the weight-streaming kernel unless a tile shape
    is forced; single-wave problems (prefill: 4 x 32 tiles of 128 x 128) the
    four-issuer kernel; weight-only workloads their own kernel; every other
    workload the tiled kernel."""
    assert bench.gemm_kind(workloads.DECODE) == ("gemm_skinny", "gemm_skinny_kernel")
    assert bench.gemm_kind(workloads.TINY) == ("gemm_skinny", "gemm_skinny_kernel")
    assert bench.gemm_kind(workloads.DECODE, "c1n224") == ("gemm", "gemm_w8a8_kernel")
    assert bench.gemm_kind(workloads.MLP_UP) == ("gemm", "gemm_w8a8_kernel")
    assert bench.gemm_kind(workloads.PREFILL) == ("gemm_small", "gemm_small_kernel")
    assert bench.gemm_kind(workloads.PREFILL, "c2n256") == ("gemm", "gemm_w8a8_kernel")
    assert bench.gemm_kind(workloads.DECODE_W4A16) == ("gemm_wonly", "gemm_wonly_kernel")


def test_single_wave_rule_matches_the_library(bench):
    """bench.py names the four-issuer kernel by the same tile and K rule the
    library dispatches on (128 x 128 tiles, at most one per SM, K of at least
    two 128-byte k-blocks per issuing thread)."""
    import re
    src = open(os.path.join(ROOT, "w8a8_smoothquant_int8_02_b200", "csrc",
                            "sq_gemm_small.cu")).read()
    assert int(re.search(r"constexpr int kSmTile = (\d+);", src).group(1)) == 128
    assert int(re.search(r"constexpr int kSmIssuers = (\d+);", src).group(1)) * 2 * 128 == 1024
    from w8a8_smoothquant_int8_02_b200 import synth
    at = workloads.PREFILL.__dict__
    assert bench.gemm_kind(synth.LinearCase(**{**at, "K": 1008}))[0] == "gemm"
    assert bench.gemm_kind(synth.LinearCase(**{**at, "M": 640}))[0] == "gemm"   # 5 x 32 > 148


def test_few_token_threshold_matches_the_library(bench):
    """bench.py names the kernel by the same token threshold the library
    dispatches on."""
    import re
    src = open(os.path.join(ROOT, "w8a8_smoothquant_int8_02_b200", "csrc",
                            "sq_gemm_skinny.cu")).read()
    mp = int(re.search(r"constexpr int kSkMP = (\d+);", src).group(1))
    assert mp == bench.SKINNY_MAX_M
    from w8a8_smoothquant_int8_02_b200 import synth
    at = workloads.DECODE.__dict__
    assert bench.gemm_kind(synth.LinearCase(**{**at, "M": mp}))[0] == "gemm_skinny"
    assert bench.gemm_kind(synth.LinearCase(**{**at, "M": mp + 1}))[0] == "gemm"


def test_bench_line_carries_every_contract_key():
    """The JSON line bench.py prints (the dict literal in run_ours and the
    one in run_reference) names every key of the measurement contract."""
    import ast
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    required = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"}
    found = {}
    for fn in (n for n in tree.body if isinstance(n, ast.FunctionDef)
               and n.name in ("run_ours", "run_reference")):
        for node in ast.walk(fn):
            if isinstance(node, ast.Assign) and any(getattr(t, "id", None) == "line"
                                                    for t in node.targets):
                assert isinstance(node.value, ast.Dict)
                found[fn.name] = {k.value for k in node.value.keys
                                  if isinstance(k, ast.Constant)}
    assert required | {"roofline", "clocks", "gpu_launches"} <= found["run_ours"]
    assert required | {"impl"} <= found["run_reference"]


def test_gpu_count_must_match_the_process_count(bench, monkeypatch):
    """--gpus N without N processes stops before touching a GPU."""
    import argparse
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    args = argparse.Namespace(gpus=2, tile=None, workload="tiny_16x64x64")
    with pytest.raises(SystemExit, match="torch.distributed.run"):
        bench.run_ours(args)
    # one GPU, one process: the check passes (and, without a GPU here, the
    # first CUDA call is what stops it)
    import torch
    if not torch.cuda.is_available():
        args.gpus = 1
        with pytest.raises(Exception) as exc:
            bench.run_ours(args)
        assert not isinstance(exc.value, SystemExit)
