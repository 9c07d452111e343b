"""Benchmark of the SmoothQuant W8A8 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = the runtime hot path of one layer over one batch: the fused
activation smoothing + per-token INT8 quantization kernel followed by the
INT8 tcgen05 GEMM with its dequantization (+bias) epilogue, at
M=4096 tokens, K=4096, N=14336 (an MLP up-projection). Weights are prepared
offline (calibration, smoothing factors, per-channel INT8 quantization) and
are not timed.

Metric: TOPS of the whole step (2*M*N*K ops / step time) and its fraction of
the INT8 dense tensor-core peak. Inputs are resident in HBM when the timed
region starts; three rotating input sets (X and Wq, 277 MB in all, more than
the 126 MB L2) keep each step from reading the previous step's data out of L2.
Rank 0 prints one JSON line. Under torchrun every rank runs its own
independent copy of the workload (weak scaling, no collective on the data
path); time is the max over ranks.

--impl reference times the plain CPU oracle on this host's cores on a bounded
sample of the same workload (the oracle is the reference arm here).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W8A8 smooth+quant+GEMM TOPS and % of INT8 TC peak at M4096 K4096 N14336"
UNIT = "TOPS"
L2_BYTES = 126 * 2 ** 20
# B200 dense INT8 / FP8 tensor-core rate from NVIDIA's datasheet (9 POPS is
# with 2:4 sparsity); reported beside the measured-peak fraction
DATASHEET_8BIT_TOPS = 4500.0


def weight_bits(case):
    """Weight bits of a weight-only workload (W8A16 / W4A16), else None."""
    return {"w8": 8, "w4": 4}.get(case.qtype)


def metric_for(case):
    if case.norm_eps:
        return (f"W8A8 RMSNorm+quant+GEMM TOPS and % of INT8 TC peak at "
                f"M{case.M} K{case.K} N{case.N}")
    if case.name.startswith("mlp_up"):
        return METRIC
    if weight_bits(case):
        return (f"W{weight_bits(case)}A16 weight-only GEMM TOPS and % of HBM roofline at "
                f"M{case.M} K{case.K} N{case.N}")
    if case.act_scaling == "tensor":
        return (f"W8A8 per-tensor FP8 quant+GEMM TOPS and % of FP8 TC peak at "
                f"M{case.M} K{case.K} N{case.N}")
    kind = "FP8" if case.qtype == "e4m3" else "INT8"
    return (f"W8A8 smooth+quant+GEMM TOPS and % of {kind} TC peak at "
            f"M{case.M} K{case.K} N{case.N}")


def rotate_count(case):
    """Input sets to rotate through so that the inputs of one step are not
    left in L2 by the previous steps (X and Wq of all sets > 1.5 x L2)."""
    per_set = case.M * case.K * 2 + case.N * case.K * (weight_bits(case) or 8) // 8
    if per_set >= 1.5 * L2_BYTES:
        return 1
    return max(2, -(-int(1.5 * L2_BYTES) // per_set))


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# one ncu capture of those two counters on bench.py's own command per
# workload (profiles/dram_bytes_per_launch_all_workloads.md), keyed by the
# sha256 prefix of the kernel's sources at capture time: a kernel changed
# since reports null.
PROFILED_TRAFFIC = {
    ("quant", "mlp_up_4096x4096x14336"): (33.648384e6 + 0.000512e6, "a01687d33b9f4575"),
    ("gemm", "mlp_up_4096x4096x14336"): (75.845376e6 + 79.977984e6, "634da0a9c1526fe2"),
    ("quant", "fp8_down_4096x14336x4096"): (117.751296e6 + 30.796800e6, "a01687d33b9f4575"),
    ("gemm", "fp8_down_4096x14336x4096"): (258.229248e6 + 39.162880e6, "634da0a9c1526fe2"),
    ("gemm", "fp8_tensor_4096x4096x14336"): (75.746048e6 + 82.847488e6, "634da0a9c1526fe2"),
    ("quant", "fp8_tensor_4096x4096x14336"): (33.578496e6 + 0.000000e6, "a01687d33b9f4575"),
    ("quant", "prefill_512x4096x4096"): (4.288512e6 + 0.000000e6, "a01687d33b9f4575"),
    ("gemm_small", "prefill_512x4096x4096"): (18.911488e6 + 0.000000e6, "2c1a43c91e6b64ee"),
    ("quant", "decode_16x8192x28672"): (0.362752e6 + 0.000000e6, "a01687d33b9f4575"),
    ("gemm_skinny", "decode_16x8192x28672"): (235.150080e6 + 0.125440e6, "5b049eeaf965ee9c"),
    ("gemm_wonly", "decode_w8a16_16x8192x28672"): (237.157632e6 + 3.582976e6, "cc74ba938948939e"),
    ("gemm_wonly", "decode_w4a16_16x8192x28672"): (119.395584e6 + 3.497472e6, "cc74ba938948939e"),
    ("norm", "mlp_up_rmsnorm_4096x4096x14336"): (33.629440e6 + 0.000512e6, "0162f0c1de1cb81e"),
    ("gemm", "mlp_up_rmsnorm_4096x4096x14336"): (75.863552e6 + 79.571968e6, "634da0a9c1526fe2"),
}
KERNEL_SOURCES = {"gemm": ("sq_gemm.cu", "sq_common.cuh"),
                  "gemm_wonly": ("sq_gemm_wonly.cu", "sq_common.cuh"),
                  "gemm_small": ("sq_gemm_small.cu", "sq_common.cuh"),
                  "gemm_skinny": ("sq_gemm_skinny.cu", "sq_common.cuh"),
                  "quant": ("sq_quant.cu", "sq_common.cuh"),
                  "norm": ("sq_norm.cu", "sq_common.cuh")}


def profiled_traffic(kind, workload):
    """Bytes per launch from the capture, or None if there is none for this
    workload or the kernel's sources changed since (or a tile is forced)."""
    import hashlib
    entry = PROFILED_TRAFFIC.get((kind, workload))
    if entry is None or (kind.startswith("gemm") and os.environ.get("SQ_GEMM_TILE")):
        return None
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, "w8a8_smoothquant_int8_02_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return entry[0] if h.hexdigest()[:16] == entry[1] else None


def gemm_roofline(ops, nbytes, ms, tops_peak, tops_peak_sus, hbm_gbs, traffic,
                  kernel="gemm_w8a8_kernel", peak_src="measured"):
    """The GEMM's roofline entry: against the 8-bit tensor peak when its
    arithmetic intensity (ops per compulsory byte) is above the ridge point
    of the two measured peaks, else against HBM bandwidth (the few-token
    decode shape, which streams the weight once)."""
    if ops / nbytes >= tops_peak * 1e12 / (hbm_gbs * 1e9):
        tops = ops / (ms * 1e-3) / 1e12
        return {"bound": "tensor", "kernel": kernel, "achieved": tops,
                "peak": tops_peak, "unit": "TFLOP/s", "frac": tops / tops_peak,
                "frac_of_sustained": tops / tops_peak_sus,
                "ops_note": f"8-bit multiply-add counted as 2 ops; peak = 2 x {peak_src} bf16 "
                            "dense (burst)",
                "traffic": traffic, "ms_per_launch": ms}
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "kernel": kernel, "achieved": gbs, "peak": hbm_gbs,
            "unit": "GB/s", "frac": gbs / hbm_gbs,
            "bytes_note": "compulsory bytes: Xq + Wq read once, Y written, scales and bias",
            "traffic": traffic, "ms_per_launch": ms}


SKINNY_MAX_M = 16  # the library's weight-streaming GEMM takes M <= 16 (sq_gemm_skinny.cu)


def gemm_kind(case, forced_tile=None):
    """Which GEMM kernel the library runs for this workload: the weight-only
    kernel for W8A16 / W4A16, the weight-streaming form for at most 16 tokens,
    the four-issuer form when the 128 x 128 tiles fit in one wave (unless a
    tile shape is forced), else the tiled kernel. Returns (traffic key,
    kernel name)."""
    if weight_bits(case):
        return "gemm_wonly", "gemm_wonly_kernel"
    if case.M <= SKINNY_MAX_M and not forced_tile:
        return "gemm_skinny", "gemm_skinny_kernel"
    tiles = -(-case.M // 128) * -(-case.N // 128)
    if tiles <= 148 and case.K >= 1024 and not forced_tile:
        return "gemm_small", "gemm_small_kernel"
    return "gemm", "gemm_w8a8_kernel"


def quant_kernel_name(case):
    """The activation kernel sq_quantize_act launches for this workload: for
    bf16 input the persistent streaming form when there are many rows, one
    CTA per row otherwise; the generic kernel for fp32 input."""
    sms = 148
    if weight_bits(case):
        return None
    if case.norm_eps:
        # one warp per row for many rows of at most 8192 elements, else the
        # block-per-row streaming form
        return ("rmsnorm_quant_warp_kernel" if case.K <= 8192 and case.M >= 4 * sms
                else "rmsnorm_quant_stream_kernel")
    if case.act_scaling == "tensor":
        return "quant_act_tensor_kernel"
    if case.x_dtype != "bf16" or case.K // 8 > 256 * 8:
        return "quant_act_kernel"
    if case.K // 8 <= 2048 and case.M >= 2 * sms:
        return "quant_act_stream_kernel"
    return "quant_act_fast_kernel"


def path_desc(case):
    if case.norm_eps:
        return "fused RMS normalization + act quant, 8-bit GEMM + epilogue"
    return ("weight-only GEMM on bf16 activations + epilogue" if weight_bits(case)
            else "act quant + 8-bit GEMM + epilogue")


def launches_per_step(case):
    """Kernels of this library launched per step: the activation kernel and
    the GEMM (the weight-only GEMM alone for W8A16 / W4A16)."""
    return 1 if weight_bits(case) else 2


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sus=float(d["bf16_tflops_sustained"]), src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


class ClockSampler:
    """nvidia-smi sampled every 100 ms in the background (clocks + throttle reasons)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        self.t_start = time.time()

    def stop(self, t0: float, t1: float) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        # samples are ~100 ms apart starting at t_start; keep those in the timed window
        n = len(rows)
        span = max(time.time() - self.t_start, 1e-3)
        ts = [self.t_start + span * (i + 0.5) / n for i in range(n)]
        sel = [r for r, t in zip(rows, ts) if t0 - 0.05 <= t <= t1 + 0.05] or rows
        sm = [float(r[1]) for r in sel if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in sel if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[j] for r in sel for j in range(4) if r[5 + j].lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(sel)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


REF_BUDGET_S = 120.0


def run_reference(args):
    """The reference arm: the CPU oracle on the same workload as our arm, a
    bounded sample of its token rows per step (full K and N)."""
    import oracle
    from w8a8_smoothquant_int8_02_b200 import synth, workloads

    ws, rank, _ = _dist()
    if rank != 0:
        return
    case = workloads.ALL[args.workload]
    d = synth.generate(case)
    s, wq, sw, scale = _oracle_prep(case, d)
    bias = d["bias"]
    # one untimed row sizes the per-step sample so that the K steps take
    # about REF_BUDGET_S seconds at most (at least one row per step)
    t0 = time.perf_counter()
    _oracle_runtime(case, np.ascontiguousarray(d["x"][:1]), s, wq, sw, bias, scale)
    t_row = max(time.perf_counter() - t0, 1e-6)
    rows = max(1, min(args.ref_rows, case.M, int(REF_BUDGET_S / (args.steps * t_row))))
    xs = np.ascontiguousarray(d["x"][:rows])
    _oracle_runtime(case, xs, s, wq, sw, bias, scale)   # warm-up at the sample size
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_runtime(case, xs, s, wq, sw, bias, scale)
    dt = time.perf_counter() - t0
    ops = 2.0 * rows * case.N * case.K * args.steps
    val = ops / dt / 1e12
    line = {
        "impl": "reference", "metric": metric_for(case), "value": val, "unit": UNIT,
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if weight_bits(case) else ("i8" if case.qtype == "i8" else "e4m3"),
        "data": f"synthetic, seeded: {case.note}",
        "config": {"workload": case.name, "M": case.M, "K": case.K, "N": case.N,
                   "alpha": case.alpha if case.smooth else None,
                   "act_scaling": ("per-tensor, delayed" if case.act_scaling == "tensor"
                                   else "per-token, from the fused RMS normalization"
                                   if case.norm_eps else "per-token"),
                   "bias": bias is not None, "out": "bf16"},
        "cpu_baseline": {"value": val, "unit": UNIT, "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"{rows} of {case.M} token rows per step through the runtime "
                                   f"path ({path_desc(case)}), full K and N"},
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _oracle_prep(case, d):
    """The oracle's offline preparation for a workload: (s or None, wq, sw,
    per-tensor scale or None)."""
    import oracle
    if weight_bits(case) == 8:
        wq, sw = oracle.quantize_weight(d["w"], None)
        return None, wq, sw, None
    if weight_bits(case) == 4:
        wq, sw = oracle.quantize_weight_i4(d["w"])
        return None, wq, sw, None
    qt = oracle.E4M3 if case.qtype == "e4m3" else oracle.INT8
    if case.norm_eps:
        # calibration on the normalization's output; the returned "s" is the
        # gain with 1/s folded in, the runtime path's only per-channel input
        xn_cal = oracle.rmsnorm_quantize_act(d["x_cal"], d["gamma"], case.norm_eps)[3]
        s = oracle.smooth_factors(oracle.amax(xn_cal, True), oracle.amax(d["w"], False),
                                  case.alpha)
        wq, sw = oracle.quantize_weight(d["w"], s, qt)
        return oracle.fold_smoothing(d["gamma"], s)[0], wq, sw, None
    s = None
    if case.smooth:
        s = oracle.smooth_factors(oracle.amax(d["x_cal"], True), oracle.amax(d["w"], False),
                                  case.alpha)
    wq, sw = oracle.quantize_weight(d["w"], s, qt)
    scale = None
    if case.act_scaling == "tensor":
        _, scale, _ = oracle.quantize_act_tensor(d["x_cal"], s, qt)
    return s, wq, sw, scale


def _oracle_runtime(case, xs, s, wq, sw, bias, scale):
    """The oracle's runtime path on token rows xs: activation quantization,
    8-bit GEMM, epilogue (the weight-only product for W8A16 / W4A16)."""
    import oracle
    if weight_bits(case):
        return oracle.gemm_weight_only(xs, wq, sw, bias, weight_bits(case))
    qt = oracle.E4M3 if case.qtype == "e4m3" else oracle.INT8
    if case.norm_eps:     # s is the folded gain here
        xq, sx, _, _ = oracle.rmsnorm_quantize_act(xs, s, case.norm_eps, qt)
        acc = oracle.gemm_e4m3(xq, wq) if qt == oracle.E4M3 else oracle.gemm_i8(xq, wq)
        return oracle.epilogue(acc, sx, sw, bias)
    if scale is None:
        return oracle.linear(xs, s, wq, sw, bias, qt)
    xq, sc, _ = oracle.quantize_act_tensor(xs, s, qt, scale=scale)
    acc = oracle.gemm_e4m3(xq, wq) if qt == oracle.E4M3 else oracle.gemm_i8(xq, wq)
    sx = np.full(xs.shape[0], sc, np.float32)
    return oracle.epilogue(acc, sx, sw, bias)


def cpu_baseline(case, d, budget_s: float):
    """Oracle throughput on a bounded sample of the workload (rank 0, N=1 only).
    The oracle prepares its own weights (untimed), then runs the runtime path
    (activation quant + 8-bit GEMM + epilogue) on as many token rows as fit
    in about `budget_s` seconds."""
    import oracle
    s, wq, sw, scale = _oracle_prep(case, d)
    # grow the sample until it takes about budget_s (a small first sample
    # underestimates the per-row rate: thread start-up, rows < threads)
    rows2, dt = 2, 0.0
    for _ in range(4):
        xs = np.ascontiguousarray(d["x"][:rows2])
        t0 = time.perf_counter()
        _oracle_runtime(case, xs, s, wq, sw, d["bias"], scale)
        dt = time.perf_counter() - t0
        if dt >= 0.5 * budget_s or rows2 >= case.M:
            break
        rows2 = int(max(rows2 + 1, min(case.M, rows2 * budget_s / max(dt, 1e-3))))
    return {"value": 2.0 * rows2 * case.N * case.K / dt / 1e12, "unit": UNIT,
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{rows2} of {case.M} token rows through the runtime path "
                      f"({path_desc(case)}), full K={case.K} and N={case.N}; {dt:.1f} s"}


def run_ours(args):
    import torch
    import torch.distributed as dist

    from w8a8_smoothquant_int8_02_b200 import dist as sqdist, ops, synth, workloads

    ws, rank, local = _dist()
    if args.gpus != ws:
        raise SystemExit(f"--gpus {args.gpus} but {ws} process(es): launch N > 1 GPUs with "
                         f"python -m torch.distributed.run --nproc-per-node {args.gpus} bench.py "
                         f"--gpus {args.gpus}")
    if args.tile:
        os.environ["SQ_GEMM_TILE"] = args.tile
    torch.cuda.set_device(local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    ops.load()
    case = workloads.ALL[args.workload]
    M, K, N = case.M, case.K, case.N
    qt = case.qtype
    ROTATE = rotate_count(case)
    dev = torch.device("cuda", local)
    d = synth.generate(case)

    def to_dev(a):
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(a).to(dev)

    # ---- offline preparation (untimed) ----
    w = to_dev(d["w"])
    wbits = weight_bits(case)
    g_fold = None
    if wbits:
        s = s_inv = None
        wq0, sw = ops.quantize_weight(w, None, "i8" if wbits == 8 else "i4")
    elif case.norm_eps:
        p = ops.prepare_rmsnorm(w, to_dev(d["x_cal"]), to_dev(d["gamma"]), case.norm_eps,
                                alpha=case.alpha, qtype=qt)
        s = s_inv = None
        g_fold, wq0, sw = p["g"], p["wq"], p["sw"]
    elif case.smooth:
        p = ops.prepare(w, to_dev(d["x_cal"]), alpha=case.alpha, qtype=qt)
        s, s_inv, wq0, sw = p["s"], p["s_inv"], p["wq"], p["sw"]
    else:
        s = s_inv = None
        wq0, sw = ops.quantize_weight(w, None, qt)
    tensor = case.act_scaling == "tensor"
    # per-tensor (delayed) scaling: step i reads the max written by step i-1;
    # the first step's comes from the calibration tokens
    amax_b = torch.zeros(2, dtype=torch.float32, device=dev)
    if tensor:
        ops.quantize_act_tensor(to_dev(d["x_cal"]), s, qt, amax_out=amax_b[0:1], s_inv=s_inv)
    bias = to_dev(d["bias"]) if d["bias"] is not None else None
    gemm = ops.gemm_w8a8 if qt == "i8" else ops.gemm_fp8
    if wbits:
        def gemm(xin, sx_, wq_, sw_, bias_, out, split=False):  # noqa: E306
            return ops.gemm_weight_only(xin, wq_, sw_, bias_, wbits, out=out)
    del w
    xs = [to_dev(d["x"])] + [None] * (ROTATE - 1)
    wqs = [wq0] + [None] * (ROTATE - 1)
    for r in range(1, ROTATE):
        xs[r] = xs[0].clone()
        wqs[r] = wq0.clone()
    xq = torch.empty((M, K), dtype=torch.int8 if qt == "i8" else torch.uint8, device=dev)
    sx = torch.empty(M, dtype=torch.float32, device=dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    # consecutive steps are independent batches: with two code buffers the
    # activation pass of step i+1 may run in the SMs that step i's GEMM leaves
    # idle in its last round of tiles (SQ_OVERLAP_PREVIOUS); it completes only
    # after that GEMM, so the steps still finish in order
    overlap = not (wbits or tensor or args.no_overlap)
    nbuf = 2 if overlap else 1
    xqs = [xq] + [torch.empty_like(xq) for _ in range(nbuf - 1)]
    sxs = [sx] + [torch.empty_like(sx) for _ in range(nbuf - 1)]

    def quantize(i, ov=False):
        r, b = i % ROTATE, i % nbuf
        if tensor:
            ops.quantize_act_tensor(xs[r], s, qt, amax_prev=amax_b[i % 2:i % 2 + 1], xq=xqs[b],
                                    sx=sxs[b], amax_out=amax_b[(i + 1) % 2:(i + 1) % 2 + 1],
                                    s_inv=s_inv)
        elif g_fold is not None:
            ops.rmsnorm_quantize_act(xs[r], g_fold, case.norm_eps, qt, xq=xqs[b], sx=sxs[b],
                                     overlap=ov)
        else:
            ops.quantize_act(xs[r], s, qt, xq=xqs[b], sx=sxs[b], s_inv=s_inv, overlap=ov)

    split = not args.no_split

    def step(i):
        if wbits:
            gemm(xs[i % ROTATE], None, wqs[i % ROTATE], sw, bias, out=y)
            return
        quantize(i, overlap)
        gemm(xqs[i % nbuf], sxs[i % nbuf], wqs[i % ROTATE], sw, bias, out=y, split=split)

    for i in range(max(3, args.warmup)):
        step(i)
    st = ops.device_status()
    if st != ops.SQ_OK:
        raise RuntimeError(f"device status after warm-up: {ops.status_string(st)}")

    # ---- per-kernel attribution (untimed for the headline): events around
    # each launch, which also keeps the two kernels from overlapping ----
    # A spin kernel ahead of every few steps lets the host queue their
    # launches before the GPU reaches them, so that the host's per-launch work
    # does not show up as idle time between the events of a short kernel.
    A_steps = min(args.steps, 200)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(A_steps)]
    torch.cuda.synchronize()
    for i in range(A_steps):
        r = i % ROTATE
        if i % 8 == 0:
            torch.cuda._sleep(4_000_000)  # about 2 ms of GPU time
        ev[i][0].record(stream)
        if not wbits:
            quantize(i)
        ev[i][1].record(stream)
        gemm(xs[r] if wbits else xqs[i % nbuf], sxs[i % nbuf], wqs[r], sw, bias, out=y,
             split=split)
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    t_quant = float(np.mean([e[0].elapsed_time(e[1]) for e in ev]))
    t_gemm = float(np.mean([e[1].elapsed_time(e[2]) for e in ev]))

    # ---- the steps as one CUDA graph: ROTATE consecutive steps (one per
    # input set) captured once and replayed, so the host's per-launch work
    # (argument checks, tensor-map encoding, Python) stays out of the timed
    # region; the kernels and their programmatic dependencies are the same.
    # Falls back to launching the steps one by one if capture fails. ----
    graph = None
    tail = None
    K_steps = args.steps
    g_steps = ROTATE * max(1, 6 // ROTATE)
    tail_steps = K_steps % g_steps

    def capture(n_steps, first):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            for i in range(first, first + n_steps):
                step(i)
        return g

    if not args.no_graph:
        try:
            side = torch.cuda.Stream(device=dev)
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                for i in range(g_steps):          # warm the capture stream's state
                    step(i)
            stream.wait_stream(side)
            torch.cuda.synchronize()
            graph = capture(g_steps, 0)
            # the last K mod g steps, so that exactly K steps are timed
            tail = capture(tail_steps, 0) if tail_steps else None
            torch.cuda.synchronize()
            graph.replay()
            if tail is not None:
                tail.replay()
            torch.cuda.synchronize()
            if ops.device_status() != ops.SQ_OK:
                raise RuntimeError("device status after a graph replay")
        except Exception as exc:  # noqa: BLE001 - report and run without the graph
            print(f"graph capture unavailable ({exc}); launching steps one by one",
                  file=sys.stderr)
            graph = tail = None

    def run_steps(n):
        if graph is not None:
            for _ in range(n // g_steps):
                graph.replay()
            if n % g_steps:
                tail.replay()
        else:
            for i in range(n):
                step(i)

    # ---- timed region: exactly K steps back to back, events only at both ends ----
    sampler = ClockSampler(local) if not args.no_clocks else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    run_steps(K_steps)
    end.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    if ws > 1:
        dist.barrier()
    clocks = sampler.stop(t_wall0, t_wall1) if sampler else None
    st = ops.device_status()
    if st != ops.SQ_OK:
        raise RuntimeError(f"device status after timed region: {ops.status_string(st)}")
    elapsed_ms = start.elapsed_time(end)
    elapsed_ms = sqdist.max_over_ranks(elapsed_ms, device=dev)

    # ---- sustained: the same steps repeated for about args.sustained_s
    # seconds (clocks settle under the power cap), timed the same way ----
    sustained = None
    if args.sustained_s > 0:
        n_sus = max(g_steps, int(args.sustained_s * 1e3 / max(elapsed_ms / K_steps, 1e-3)))
        n_sus = (n_sus + g_steps - 1) // g_steps * g_steps
        sampler2 = ClockSampler(local) if not args.no_clocks else None
        if sampler2:
            sampler2.start()
            time.sleep(0.3)
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t_s0 = time.time()
        a_ev = torch.cuda.Event(enable_timing=True)
        b_ev = torch.cuda.Event(enable_timing=True)
        a_ev.record(stream)
        run_steps(n_sus)
        b_ev.record(stream)
        torch.cuda.synchronize()
        t_s1 = time.time()
        if ws > 1:
            dist.barrier()
        clocks2 = sampler2.stop(t_s0, t_s1) if sampler2 else None
        sus_ms = sqdist.max_over_ranks(a_ev.elapsed_time(b_ev), device=dev)
        if ops.device_status() != ops.SQ_OK:
            raise RuntimeError("device status after the sustained run")
        sustained = {"value": ws * case.ops * n_sus / (sus_ms * 1e-3) / 1e12, "unit": UNIT,
                     "steps": n_sus, "seconds": sus_ms * 1e-3, "ms_per_step": sus_ms / n_sus,
                     "clocks": clocks2}

    # ---- end to end through the public API with host buffers: every step
    # copies its input X from pinned host memory and its output Y back, in a
    # three-stage pipeline (H2D of step i+1 and D2H of step i-1 overlap the
    # kernels of step i, on their own streams, with double-buffered device
    # copies of X and Y) ----
    e2e = None
    if not args.no_e2e:
        x_host = torch.empty((M, K), dtype=torch.bfloat16, pin_memory=True)
        x_host.copy_(xs[0].cpu())
        y_host = [torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
        x_dev = [torch.empty_like(xs[0]) for _ in range(2)]
        y_dev = [y, torch.empty_like(y)]
        e_steps = max(3, min(args.steps, args.e2e_steps))
        s_h2d, s_comp, s_d2h = (torch.cuda.Stream(device=dev) for _ in range(3))

        def compute(xd, yd):
            if wbits:
                gemm(xd, None, wq0, sw, bias, out=yd)
            elif tensor:
                ops.quantize_act_tensor(xd, s, qt, amax_prev=amax_b[0:1], xq=xq, sx=sx,
                                        amax_out=amax_b[1:2], s_inv=s_inv)
                gemm(xq, sx, wq0, sw, bias, out=yd, split=split)
            elif g_fold is not None:
                ops.rmsnorm_quantize_act(xd, g_fold, case.norm_eps, qt, xq=xq, sx=sx)
                gemm(xq, sx, wq0, sw, bias, out=yd, split=split)
            else:
                ops.linear(xd, s, wq0, sw, bias, qt, out=yd, xq_buf=xq, sx_buf=sx, s_inv=s_inv,
                           split=split)

        def run_pipeline(n):
            ev = [[torch.cuda.Event() for _ in range(3)] for _ in range(n)]
            for i in range(n):
                bb = i % 2
                with torch.cuda.stream(s_h2d):
                    if i >= 2:
                        s_h2d.wait_event(ev[i - 2][1])        # x_dev[bb] read by step i-2
                    x_dev[bb].copy_(x_host, non_blocking=True)
                    ev[i][0].record(s_h2d)
                with torch.cuda.stream(s_comp):
                    s_comp.wait_event(ev[i][0])
                    if i >= 2:
                        s_comp.wait_event(ev[i - 2][2])       # y_dev[bb] copied out by step i-2
                    compute(x_dev[bb], y_dev[bb])
                    ev[i][1].record(s_comp)
                with torch.cuda.stream(s_d2h):
                    s_d2h.wait_event(ev[i][1])
                    y_host[bb].copy_(y_dev[bb], non_blocking=True)
                    ev[i][2].record(s_d2h)

        run_pipeline(3)
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(s_h2d)
        run_pipeline(e_steps)
        b.record(s_d2h)
        torch.cuda.synchronize()
        e_ms = sqdist.max_over_ranks(a.elapsed_time(b), device=dev)
        step_s = e_ms * 1e-3 / e_steps
        e2e = {"value": ws * case.ops * e_steps / (e_ms * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2,
               "steps": e_steps, "pipeline": "H2D / kernels / D2H on three streams",
               # the copies' achieved rates over the step (each direction has
               # its own PCIe link budget): the larger one bounds the step
               "h2d_gbs": M * K * 2 / step_s / 1e9, "d2h_gbs": M * N * 2 / step_s / 1e9,
               "bound": ("D2H copy of Y" if M * N >= M * K else "H2D copy of X")}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(case, d, args.cpu_budget)

    if rank == 0:
        pk = _peaks()
        g_kind, g_name = gemm_kind(case, os.environ.get("SQ_GEMM_TILE"))
        int8_peak = 2.0 * pk["bf16"]        # dense INT8 / FP8 = 2x dense bf16 (4.5 vs 2.25 P)
        int8_peak_sus = 2.0 * pk["bf16_sus"]
        gemm_tops = case.ops / (t_gemm * 1e-3) / 1e12
        value = ws * case.ops * K_steps / (elapsed_ms * 1e-3) / 1e12
        # read X (bf16) + s (or the folded gain), write Xq + sx (per-tensor: + the scale, + the max)
        q_bytes = M * K * 2 + M * K + M * 4 + (K * 4 if case.smooth else 0)
        g_bytes = M * K + N * K + M * N * 2 + 4 * (M + N) + (2 * N if bias is not None else 0)
        if wbits:
            # bf16 X, the packed weight codes once, Y bf16, scales and bias
            g_bytes = (M * K * 2 + N * K * wbits // 8 + M * N * 2 + 4 * N
                       + (2 * N if bias is not None else 0))
        w_set = N * K * (wbits or 8) // 8
        line = {
            "metric": metric_for(case), "value": value, "unit": UNIT, "n_gpus": ws,
            "steps": K_steps, "warmup": args.warmup, "ms_per_step": elapsed_ms / K_steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if wbits else ("i8" if qt == "i8" else "e4m3"),
            "data": f"synthetic, seeded: {case.note}",
            "config": {"workload": case.name, "M": M, "K": K, "N": N,
                       "alpha": case.alpha if case.smooth else None,
                       "act_scaling": ("none (weight-only)" if wbits else
                                       "per-tensor, delayed" if tensor else
                                       "per-token, from the fused RMS normalization"
                                       if case.norm_eps else "per-token"),
                       "bias": bias is not None, "out": "bf16",
                       "l2": (f"{ROTATE} rotating input sets (X + Wq, "
                              f"{ROTATE * (M * K * 2 + w_set) / 2 ** 20:.0f} MiB) > 126 MiB L2"),
                       "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU",
                       "launch": ((f"CUDA graph of {g_steps} steps, replayed"
                                   + (f", then one of {tail_steps}" if tail_steps else ""))
                                  if graph is not None else "one launch per kernel"),
                       "gemm_workspace": ("passed: the last partial round of tiles is split where that pays" if split else "not passed"),
                       "gemm_tile": os.environ.get("SQ_GEMM_TILE", "auto"),
                       "overlap": ("the activation pass of step i+1 may run in the SMs step i's "
                                   "GEMM leaves idle (two code buffers, SQ_OVERLAP_PREVIOUS)"
                                   if overlap else "none")},
            "frac_of_int8_peak": None if wbits else value / ws / int8_peak,
            "frac_of_datasheet": None if wbits else value / ws / DATASHEET_8BIT_TOPS,
            "int8_peak_tops": int8_peak,
            "datasheet_8bit_tops": DATASHEET_8BIT_TOPS,
            "int8_peak_source": f"2 x {pk['src']} bf16 dense ({pk['bf16']} TFLOP/s burst)",
            "gemm_hbm_gbs": g_bytes / (t_gemm * 1e-3) / 1e9,
            "roofline": gemm_roofline(case.ops, g_bytes, t_gemm, int8_peak, int8_peak_sus,
                                      pk["hbm"], profiled_traffic(g_kind, case.name), g_name,
                                      pk["src"]),
            "roofline_quant": None if wbits else {
                "bound": "hbm", "kernel": quant_kernel_name(case),
                "achieved": q_bytes / (t_quant * 1e-3) / 1e9, "peak": pk["hbm"],
                "unit": "GB/s", "frac": q_bytes / (t_quant * 1e-3) / 1e9 / pk["hbm"],
                "traffic": profiled_traffic("norm" if case.norm_eps else "quant", case.name),
                "ms_per_launch": t_quant},
            "gpu_launches": launches_per_step(case) * K_steps,
            "clocks": clocks,
            "sustained": sustained,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()


def measure_peaks(args):
    """Black-box 8-bit tensor-core rates of cuBLAS on this GPU (no code of this
    repository on the path): torch._int_mm (INT8 x INT8 -> int32) and
    torch._scaled_mm (E4M3 x E4M3 -> bf16, per-tensor scales), each at
    8192^3 and at every workload shape with at least 17 tokens. One JSON line
    per (kind, shape): mean CUDA-event time of `steps` launches after
    `warmup`, TOPS, and the SM clocks sampled meanwhile."""
    import torch
    from w8a8_smoothquant_int8_02_b200 import workloads

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    shapes = [("cube_8192", 8192, 8192, 8192)]
    shapes += [(c.name, c.M, c.K, c.N) for c in workloads.ALL.values() if c.M > 16]
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    for name, M, K, N in shapes:
        for kind in ("int8", "e4m3"):
            a8 = torch.randint(-127, 128, (M, K), dtype=torch.int8, device=dev, generator=g)
            b8 = torch.randint(-127, 128, (N, K), dtype=torch.int8, device=dev, generator=g)
            if kind == "int8":
                fn = lambda: torch._int_mm(a8, b8.t())  # noqa: E731
            else:
                af = (a8.float() / 32).to(torch.float8_e4m3fn)
                bf = (b8.float() / 32).to(torch.float8_e4m3fn)
                one = torch.ones((), dtype=torch.float32, device=dev)
                fn = lambda: torch._scaled_mm(af, bf.t(), scale_a=one, scale_b=one,  # noqa: E731
                                              out_dtype=torch.bfloat16)
            for _ in range(max(3, args.warmup)):
                fn()
            torch.cuda.synchronize()
            n = max(20, args.steps)
            sampler = ClockSampler(0) if not args.no_clocks else None
            if sampler:
                sampler.start()
                time.sleep(0.3)
            t0 = time.time()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(n):
                fn()
            e1.record()
            torch.cuda.synchronize()
            t1 = time.time()
            clocks = sampler.stop(t0, t1) if sampler else None
            ms = e0.elapsed_time(e1) / n
            print(json.dumps({"peak_probe": f"cublas_{kind}", "shape": name, "M": M, "K": K,
                              "N": N, "us_per_launch": ms * 1e3,
                              "tops": 2.0 * M * N * K / (ms * 1e-3) / 1e12, "launches": n,
                              "clocks": clocks}), flush=True)
            del a8, b8
            torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--ref-rows", type=int, default=8)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the timed steps one by one instead of replaying a CUDA graph")
    ap.add_argument("--workload", default="mlp_up_4096x4096x14336",
                    help="one of the workloads in workloads.py (default: the MLP up-projection)")
    ap.add_argument("--no-overlap", action="store_true",
                    help="keep each step's activation pass from starting before the previous "
                         "step's GEMM has completed (by default it may use the SMs that GEMM "
                         "leaves idle in its last round of tiles)")
    ap.add_argument("--no-split", action="store_true",
                    help="launch the GEMM without its workspace (by default the library may split "
                         "the last partial round of tiles along K over all SMs where that pays)")
    ap.add_argument("--sustained-s", type=float, default=1.5,
                    help="seconds of extra replays for the sustained figure (0: skip)")
    ap.add_argument("--measure-peaks", action="store_true",
                    help="time the library-free 8-bit peaks instead: cuBLAS INT8 (torch._int_mm) "
                         "and FP8 (torch._scaled_mm) as black boxes at 8192^3 and each workload")
    ap.add_argument("--tile", default=None, help="force a GEMM tile shape (c1n128, c1n224, c1n256, "
                    "c2n224, c2n256); default: chosen by problem size")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.measure_peaks:
        measure_peaks(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
