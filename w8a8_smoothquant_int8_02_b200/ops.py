"""Python binding of libsq.so (the C ABI in include/sq.h).

Argument marshalling only: every step of the layer runs in the CUDA library.
torch supplies device memory and the current stream. If the library cannot
be built or loaded, every call raises -- there is no CPU fallback.

Layouts follow include/sq.h: X [M,K], W [K,N], Wq [N,K] (K contiguous),
Y [M,N], all row-major; bf16 tensors are passed as torch.bfloat16, E4M3 codes
as torch.uint8 or torch.float8_e4m3fn.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import build as _build

(SQ_OK, SQ_ERR_INVALID_ARG, SQ_ERR_MISALIGNED, SQ_ERR_UNSUPPORTED, SQ_ERR_CUDA, SQ_ERR_TIMEOUT,
 SQ_ERR_SCRATCH_TOO_SMALL) = range(7)
SQ_F32, SQ_BF16, SQ_I8, SQ_E4M3, SQ_I32, SQ_I4 = range(6)
SQ_AMAX_PER_COLUMN, SQ_AMAX_PER_ROW = 0, 1
SQ_OVERLAP_PREVIOUS = 1

EXPORTED = (
    "sq_status_string", "sq_abi_version", "sq_get_device_status", "sq_calibrate_amax",
    "sq_smooth_factors", "sq_quantize_weight", "sq_quantize_act", "sq_gemm_w8a8",
    "sq_gemm_fp8", "sq_linear", "sq_probe_wait_timeout", "sq_selftest_fast_division",
    "sq_gemm_workspace_bytes", "sq_gemm_w8a8_noalloc", "sq_quantize_act_tensor",
    "sq_fold_smoothing", "sq_gemm_weight_only", "sq_rmsnorm_quantize_act",
)

_lock = threading.Lock()
_lib = None


class SQError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


def library_path() -> str:
    return _build.LIB


def load(build_if_needed: bool = True) -> ctypes.CDLL:
    """Load libsq.so (building it first with nvcc if it is missing or stale)."""
    global _lib
    with _lock:
        if _lib is None:
            if build_if_needed and _build.is_stale():
                _build.build()
            if not os.path.exists(_build.LIB):
                raise RuntimeError(f"libsq.so not found at {_build.LIB}; build it with "
                                   "`python -m w8a8_smoothquant_int8_02_b200.build`")
            lib = ctypes.CDLL(_build.LIB)
            P, I64, I, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
            U32 = ctypes.c_uint32
            lib.sq_status_string.argtypes = [I]
            lib.sq_status_string.restype = ctypes.c_char_p
            lib.sq_abi_version.restype = I
            lib.sq_get_device_status.argtypes = [P]
            lib.sq_calibrate_amax.argtypes = [P, I, I64, I64, I, P, I, P]
            lib.sq_smooth_factors.argtypes = [P, P, I64, D, P, P, P]
            lib.sq_quantize_weight.argtypes = [P, I, I64, I64, P, I, P, P, P]
            lib.sq_quantize_act.argtypes = [P, I, I64, I64, P, P, I, P, P, U32, P]
            lib.sq_fold_smoothing.argtypes = [P, I, I64, I64, P, I, P, P]
            SZ = ctypes.c_size_t
            lib.sq_gemm_w8a8.argtypes = [P, P, P, P, P, I64, I64, I64, P, I, P, P, SZ, P]
            lib.sq_gemm_fp8.argtypes = [P, P, P, P, P, I64, I64, I64, P, I, P, SZ, P]
            lib.sq_linear.argtypes = [P, I, P, P, P, P, P, I, I64, I64, I64, P, P, P, I, P, SZ, P]
            lib.sq_gemm_w8a8_noalloc.argtypes = [P, P, P, P, P, I64, I64, I64, P, I, P]
            lib.sq_gemm_weight_only.argtypes = [P, P, I, P, P, I64, I64, I64, P, I, P]
            lib.sq_rmsnorm_quantize_act.argtypes = [P, P, ctypes.c_float, I64, I64, I, P, P, P, U32, P]
            lib.sq_gemm_workspace_bytes.argtypes = []
            lib.sq_gemm_workspace_bytes.restype = SZ
            lib.sq_probe_wait_timeout.argtypes = [I64, P]
            lib.sq_selftest_fast_division.argtypes = [ctypes.POINTER(ctypes.c_int64), P]
            for name in EXPORTED:
                if name not in ("sq_status_string", "sq_abi_version", "sq_gemm_workspace_bytes"):
                    getattr(lib, name).restype = I
            _lib = lib
    return _lib


def status_string(st: int) -> str:
    return load().sq_status_string(int(st)).decode()


def _check(st: int, what: str):
    if st != SQ_OK:
        raise SQError(st, what)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device=None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _fdtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SQ_BF16
    if t.dtype == torch.float32:
        return SQ_F32
    raise TypeError(f"expected a bfloat16 or float32 tensor, got {t.dtype}")


def _qtype(q: str) -> int:
    if q in ("i8", "int8"):
        return SQ_I8
    if q in ("e4m3", "fp8"):
        return SQ_E4M3
    if q in ("i4", "int4"):
        return SQ_I4
    raise ValueError(f"qtype must be 'i8', 'e4m3' or 'i4', got {q!r}")


def _cuda(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("all tensors must be CUDA tensors")
            if not t.is_contiguous():
                raise ValueError("all tensors must be contiguous")


def _codes(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.uint8) if t.dtype == torch.float8_e4m3fn else t


# ---------------------------------------------------------------- stages --

def calibrate_amax(x: torch.Tensor, axis: str = "column", out: torch.Tensor | None = None,
                   accumulate: bool = False) -> torch.Tensor:
    """a1/a2: per-column ("column", over rows) or per-row ("row") max |x|."""
    _cuda(x, out)
    rows, cols = x.shape
    ax = SQ_AMAX_PER_COLUMN if axis == "column" else SQ_AMAX_PER_ROW
    n = cols if ax == SQ_AMAX_PER_COLUMN else rows
    if out is None:
        out = torch.empty(n, dtype=torch.float32, device=x.device)
    _check(load().sq_calibrate_amax(_p(x), _fdtype(x), rows, cols, ax, _p(out), int(accumulate),
                                    _stream(x.device)), "sq_calibrate_amax")
    return out


def fold_smoothing(p: torch.Tensor, s: torch.Tensor, axis: str = "column",
                   out: torch.Tensor | None = None) -> torch.Tensor:
    """Offline: the producer's per-channel parameters divided by s (float32),
    so that it emits X~ = X diag(s)^-1 and the quantization runs without s.
    axis "column": channel = column of p (a gain vector, or a producer weight
    [R,K] in the [in,out] layout); "row": channel = row (a weight stored
    [K,R]). A 1-D p holds one value per channel."""
    _cuda(p, s, out)
    if axis not in ("column", "row"):
        raise ValueError("axis must be 'column' or 'row'")
    if p.dim() == 1:
        rows, cols = (1, p.numel()) if axis == "column" else (p.numel(), 1)
    elif p.dim() == 2:
        rows, cols = p.shape
    else:
        raise ValueError("p must be 1-D or 2-D")
    if s.dtype != torch.float32 or s.numel() != (cols if axis == "column" else rows):
        raise ValueError("s must be float32 with one entry per channel")
    if out is None:
        out = torch.empty(p.shape, dtype=torch.float32, device=p.device)
    elif out.shape != p.shape or out.dtype != torch.float32:
        raise ValueError("out must be float32 with p's shape")
    ax = SQ_AMAX_PER_COLUMN if axis == "column" else SQ_AMAX_PER_ROW
    _check(load().sq_fold_smoothing(_p(p), _fdtype(p), rows, cols, _p(s), ax, _p(out),
                                    _stream(p.device)), "sq_fold_smoothing")
    return out


def smooth_factors(amax_x: torch.Tensor, amax_w: torch.Tensor, alpha: float,
                   with_inverse: bool = False):
    """a3: s = max(ax,1e-5)^alpha / max(aw,1e-5)^(1-alpha) (binary64 -> binary32).
    with_inverse=True also returns s_inv (the reciprocals sq_quantize_act uses)."""
    _cuda(amax_x, amax_w)
    s = torch.empty_like(amax_x)
    s_inv = torch.empty_like(amax_x) if with_inverse else None
    _check(load().sq_smooth_factors(_p(amax_x), _p(amax_w), amax_x.numel(), float(alpha), _p(s),
                                    _p(s_inv), _stream(amax_x.device)), "sq_smooth_factors")
    return (s, s_inv) if with_inverse else s


def quantize_weight(w: torch.Tensor, s: torch.Tensor | None, qtype: str = "i8"):
    """a4: returns (wq [N,K] int8 / uint8-E4M3, sw [N] float32); qtype "i4"
    (weight-only, s None): wq [N,K/2] uint8, two codes per byte."""
    _cuda(w, s)
    K, N = w.shape
    qt = _qtype(qtype)
    if qt == SQ_I4:
        wq = torch.empty((N, K // 2), dtype=torch.uint8, device=w.device)
    else:
        wq = torch.empty((N, K), dtype=torch.int8 if qt == SQ_I8 else torch.uint8,
                         device=w.device)
    sw = torch.empty(N, dtype=torch.float32, device=w.device)
    _check(load().sq_quantize_weight(_p(w), _fdtype(w), K, N, _p(s), qt, _p(wq), _p(sw),
                                     _stream(w.device)), "sq_quantize_weight")
    return wq, sw


def quantize_act(x: torch.Tensor, s: torch.Tensor | None, qtype: str = "i8", xq=None, sx=None,
                 s_inv: torch.Tensor | None = None, overlap: bool = False):
    """a5: fused smoothing + per-token quantization; returns (xq [M,K], sx [M]).
    s_inv (from smooth_factors(..., with_inverse=True)) only makes it faster.
    overlap=True passes SQ_OVERLAP_PREVIOUS: the caller guarantees that the
    kernel before it on the stream neither writes x, s, s_inv nor touches xq,
    sx (e.g. the previous batch's GEMM reading another xq buffer); the pass may
    then run in the SMs that kernel leaves idle."""
    _cuda(x, s, xq, sx, s_inv)
    M, K = x.shape
    qt = _qtype(qtype)
    if xq is None:
        xq = torch.empty((M, K), dtype=torch.int8 if qt == SQ_I8 else torch.uint8, device=x.device)
    if sx is None:
        sx = torch.empty(M, dtype=torch.float32, device=x.device)
    _check(load().sq_quantize_act(_p(x), _fdtype(x), M, K, _p(s), _p(s_inv), qt, _p(xq), _p(sx),
                                  SQ_OVERLAP_PREVIOUS if overlap else 0, _stream(x.device)),
           "sq_quantize_act")
    return xq, sx


def quantize_act_tensor(x: torch.Tensor, s: torch.Tensor | None, qtype: str = "e4m3",
                        amax_prev: torch.Tensor | None = None, xq=None, sx=None, amax_out=None,
                        s_inv: torch.Tensor | None = None):
    """Smoothing + per-tensor quantization: one scale for the whole tensor,
    RN(amax_prev / Q) (delayed scaling from the previous step's max) or, with
    amax_prev None, this tensor's own max / Q (online). Returns (xq [M,K],
    sx [M] = the scale in every entry, amax_out [1] = this tensor's
    max|x/s|, the next step's amax_prev)."""
    _cuda(x, s, xq, sx, s_inv, amax_prev, amax_out)
    M, K = x.shape
    qt = _qtype(qtype)
    if xq is None:
        xq = torch.empty((M, K), dtype=torch.int8 if qt == SQ_I8 else torch.uint8, device=x.device)
    if sx is None:
        sx = torch.empty(M, dtype=torch.float32, device=x.device)
    if amax_out is None:
        amax_out = torch.empty(1, dtype=torch.float32, device=x.device)
    _check(load().sq_quantize_act_tensor(_p(x), _fdtype(x), M, K, _p(s), _p(s_inv), qt,
                                         _p(amax_prev), _p(xq), _p(sx), _p(amax_out),
                                         _stream(x.device)), "sq_quantize_act_tensor")
    return xq, sx, amax_out


_workspaces: dict = {}


def workspace(device=None) -> torch.Tensor:
    """The per-device GEMM workspace (zero-filled once; the GEMMs keep it
    zeroed). Calls on one device share it, so they must not run
    concurrently on different streams."""
    dev = torch.device("cuda", torch.cuda.current_device() if device is None else
                       torch.device(device).index or 0)
    ws = _workspaces.get(dev)
    if ws is None:
        with torch.cuda.device(dev):
            n = int(load().sq_gemm_workspace_bytes())
        ws = torch.zeros(n, dtype=torch.uint8, device=dev)
        _workspaces[dev] = ws
    return ws


def _ws_args(use_split, device):
    """(pointer, bytes) of the workspace, or (None, 0) to run without split tiles."""
    if not use_split:
        return None, 0
    ws = workspace(device)
    return _p(ws), ws.numel()


def gemm_w8a8(xq, sx, wq, sw, bias=None, out_dtype=torch.bfloat16, out=None, acc=None,
              split=False):
    """a6: INT8 tensor-core GEMM + dequant epilogue. Returns y (and fills acc if given).
    split=True passes the workspace so the last partial wave of tiles may be
    split along K over all SMs (same results; opt-in: on B200 it has not yet
    beaten whole tiles on the measured shapes)."""
    _cuda(xq, sx, wq, sw, bias, out, acc)
    M, K = xq.shape
    N = wq.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=xq.device)
    wsp, wsn = _ws_args(split, xq.device)
    _check(load().sq_gemm_w8a8(_p(xq), _p(sx), _p(wq), _p(sw), _p(bias), M, N, K, _p(out),
                               _fdtype(out), _p(acc), wsp, wsn, _stream(xq.device)),
           "sq_gemm_w8a8")
    return out


def gemm_w8a8_noalloc(xq, sx, wq, sw, bias=None, out_dtype=torch.bfloat16, out=None):
    """sq_gemm_w8a8_noalloc: the INT8 GEMM with the library's fixed scratch array
    instead of a caller workspace (allocates nothing itself; `out` may be given)."""
    _cuda(xq, sx, wq, sw, bias, out)
    M, K = xq.shape
    N = wq.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=xq.device)
    _check(load().sq_gemm_w8a8_noalloc(_p(xq), _p(sx), _p(wq), _p(sw), _p(bias), M, N, K,
                                       _p(out), _fdtype(out), _stream(xq.device)),
           "sq_gemm_w8a8_noalloc")
    return out


def gemm_fp8(xq, sx, wq, sw, bias=None, out_dtype=torch.bfloat16, out=None, split=False):
    """a7: FP8 E4M3 tensor-core GEMM + dequant epilogue."""
    xq, wq = _codes(xq), _codes(wq)
    _cuda(xq, sx, wq, sw, bias, out)
    M, K = xq.shape
    N = wq.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=xq.device)
    wsp, wsn = _ws_args(split, xq.device)
    _check(load().sq_gemm_fp8(_p(xq), _p(sx), _p(wq), _p(sw), _p(bias), M, N, K, _p(out),
                              _fdtype(out), wsp, wsn, _stream(xq.device)), "sq_gemm_fp8")
    return out


def gemm_weight_only(x, wq, sw, bias=None, bits=8, out_dtype=torch.bfloat16, out=None):
    """Weight-only W8A16 (bits 8: wq int8 [N,K]) or W4A16 (bits 4: wq packed
    uint8 [N,K/2]) linear layer on bf16 activations x [M,K]."""
    _cuda(x, wq, sw, bias, out)
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    M, K = x.shape
    N = wq.shape[0]
    if bits not in (8, 4):
        raise ValueError("bits must be 8 or 4")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x.device)
    _check(load().sq_gemm_weight_only(_p(x), _p(wq), SQ_I8 if bits == 8 else SQ_I4, _p(sw),
                                      _p(bias), M, N, K, _p(out), _fdtype(out),
                                      _stream(x.device)), "sq_gemm_weight_only")
    return out


def rmsnorm_quantize_act(x, g, eps, qtype="i8", xq=None, sx=None, xn=None, want_xn=False,
                         overlap=False):
    """The producer of X with the smoothing folded in: RMS normalization of the
    bf16 rows of x [M,K] with gain g [K] (gamma / s, see fold_smoothing), fused
    with per-token quantization. Returns (xq [M,K] codes, sx [M]); with
    want_xn (or an xn buffer given) also the normalization's output xn [M,K]
    float32, the input of the offline calibration. overlap: as quantize_act."""
    _cuda(x, g, xq, sx, xn)
    if x.dtype != torch.bfloat16 or g.dtype != torch.float32:
        raise TypeError("x must be bfloat16 and g float32")
    M, K = x.shape
    qt = SQ_I8 if qtype == "i8" else SQ_E4M3
    if xq is None:
        xq = torch.empty((M, K), dtype=torch.int8 if qt == SQ_I8 else torch.uint8,
                         device=x.device)
    if sx is None:
        sx = torch.empty(M, dtype=torch.float32, device=x.device)
    if xn is None and want_xn:
        xn = torch.empty((M, K), dtype=torch.float32, device=x.device)
    _check(load().sq_rmsnorm_quantize_act(_p(x), _p(g), float(eps), M, K, qt, _p(xq), _p(sx),
                                          _p(xn), SQ_OVERLAP_PREVIOUS if overlap else 0,
                                          _stream(x.device)), "sq_rmsnorm_quantize_act")
    return (xq, sx, xn) if xn is not None else (xq, sx)


def linear(x, s, wq, sw, bias=None, qtype="i8", out_dtype=torch.bfloat16, out=None,
           xq_buf=None, sx_buf=None, s_inv=None, split=False):
    """Runtime forward: quantize_act then the 8-bit GEMM, one C call."""
    wq = _codes(wq)
    _cuda(x, s, wq, sw, bias, out, xq_buf, sx_buf, s_inv)
    M, K = x.shape
    N = wq.shape[0]
    qt = _qtype(qtype)
    if xq_buf is None:
        xq_buf = torch.empty((M, K), dtype=torch.int8 if qt == SQ_I8 else torch.uint8,
                             device=x.device)
    if sx_buf is None:
        sx_buf = torch.empty(M, dtype=torch.float32, device=x.device)
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x.device)
    wsp, wsn = _ws_args(split, x.device)
    _check(load().sq_linear(_p(x), _fdtype(x), _p(s), _p(s_inv), _p(wq), _p(sw), _p(bias), qt,
                            M, N, K, _p(xq_buf), _p(sx_buf), _p(out), _fdtype(out), wsp, wsn,
                            _stream(x.device)),
           "sq_linear")
    return out


def device_status(device=None) -> int:
    """Synchronize the current stream and return (and clear) the status word.
    After a timeout the GEMM workspace may hold partial counters: it is
    zero-filled again here, as its contract requires."""
    st = int(load().sq_get_device_status(_stream(device)))
    if st == SQ_ERR_TIMEOUT:
        for ws in _workspaces.values():
            ws.zero_()
        torch.cuda.synchronize()
    return st


def selftest_fast_division(device=None) -> int:
    """Exhaustive check of the activation-smoothing division shortcut; returns
    the number of (x, s) significand pairs where it differs from IEEE division."""
    n = ctypes.c_int64(-1)
    _check(load().sq_selftest_fast_division(ctypes.byref(n), _stream(device)),
           "sq_selftest_fast_division")
    return int(n.value)


def probe_wait_timeout(timeout_ns: int, device=None):
    _check(load().sq_probe_wait_timeout(int(timeout_ns), _stream(device)), "sq_probe_wait_timeout")


# GEMM tile shapes compiled into libsq.so (CTAs per tile x N per tile).
GEMM_TILES = ("c1n128", "c1n224", "c1n256", "c2n224", "c2n256")


class gemm_tile:
    """Context manager forcing one GEMM tile shape (testing / tuning); the
    library otherwise picks the shape from the problem size."""

    def __init__(self, name: str | None):
        if name is not None and name not in GEMM_TILES:
            raise ValueError(f"unknown tile {name!r}; choose from {GEMM_TILES}")
        self.name = name

    def __enter__(self):
        self.prev = os.environ.get("SQ_GEMM_TILE")
        if self.name is None:
            os.environ.pop("SQ_GEMM_TILE", None)
        else:
            os.environ["SQ_GEMM_TILE"] = self.name
        return self

    def __exit__(self, *exc):
        if self.prev is None:
            os.environ.pop("SQ_GEMM_TILE", None)
        else:
            os.environ["SQ_GEMM_TILE"] = self.prev


# ------------------------------------------------------------ a layer API --

def prepare(w: torch.Tensor, x_cal: torch.Tensor, alpha: float = 0.5, qtype: str = "i8"):
    """Offline preparation of one layer: calibrate, smoothing factors, quantized weights."""
    ax = calibrate_amax(x_cal, "column")
    aw = calibrate_amax(w, "row")
    s, s_inv = smooth_factors(ax, aw, alpha, with_inverse=True)
    wq, sw = quantize_weight(w, s, qtype)
    return dict(s=s, s_inv=s_inv, wq=wq, sw=sw, amax_x=ax, amax_w=aw)


def prepare_rmsnorm(w: torch.Tensor, x_cal: torch.Tensor, gamma: torch.Tensor, eps: float,
                    alpha: float = 0.5, qtype: str = "i8"):
    """Offline preparation of a layer fed by an RMS normalization: the
    calibration runs on the normalization's output (gain gamma), then s, the
    quantized weights, and the gain with 1/s folded in (g = gamma / s) for
    rmsnorm_quantize_act at runtime."""
    _, _, xn = rmsnorm_quantize_act(x_cal, gamma, eps, qtype, want_xn=True)
    p = prepare(w, xn, alpha, qtype)
    p["g"] = fold_smoothing(gamma, p["s"])
    return p


class SmoothQuantLinear:
    """A prepared W8A8 linear layer: y = x @ W (+ bias).

    act_scaling "token" (default): SmoothQuant, per-token activation scales.
    act_scaling "tensor": one scale for the whole activation tensor, taken
    from the previous call's max (delayed scaling; the first call's from the
    calibration tokens); smooth=False skips the smoothing factors (native
    FP8 without SmoothQuant)."""

    def __init__(self, w: torch.Tensor, x_cal: torch.Tensor, alpha: float = 0.5,
                 qtype: str = "i8", bias: torch.Tensor | None = None,
                 act_scaling: str = "token", smooth: bool = True):
        if act_scaling not in ("token", "tensor"):
            raise ValueError("act_scaling must be 'token' or 'tensor'")
        if smooth:
            p = prepare(w, x_cal, alpha, qtype)
            self.s, self.s_inv, self.wq, self.sw = p["s"], p["s_inv"], p["wq"], p["sw"]
        else:
            self.s = self.s_inv = None
            self.wq, self.sw = quantize_weight(w, None, qtype)
        self.folded_s = None
        self.qtype = qtype
        self.bias = bias
        self.act_scaling = act_scaling
        self.in_features, self.out_features = w.shape
        if act_scaling == "tensor":
            # two floats: the max the next call scales by, and the one it writes
            self._amax = torch.zeros(2, dtype=torch.float32, device=w.device)
            self._cur = 0
            quantize_act_tensor(x_cal, self.s, qtype, amax_out=self._amax[0:1], s_inv=self.s_inv)

    def fold_smoothing_into(self, p: torch.Tensor, axis: str = "column") -> torch.Tensor:
        """Offline: fold this layer's 1/s into the parameters p of the layer
        that produces its input (see fold_smoothing for the axes) and take the
        producer's output as already smoothed from then on, so the runtime
        quantization runs without the division. Returns the folded float32
        parameters for the producer. A layer folds once; any other
        parameter of the producer on the same channels (its bias, say) takes
        fold_smoothing(bias, layer.folded_s)."""
        if self.s is None:
            raise RuntimeError("no smoothing factors to fold (smooth=False, or already folded)")
        out = fold_smoothing(p, self.s, axis)
        self.folded_s, self.s, self.s_inv = self.s, None, None
        return out

    @property
    def last_amax(self) -> torch.Tensor:
        """The activation max the next call will scale by (tensor scaling)."""
        return self._amax[self._cur:self._cur + 1]

    def __call__(self, x: torch.Tensor, out_dtype=torch.bfloat16) -> torch.Tensor:
        if self.act_scaling == "token":
            return linear(x, self.s, self.wq, self.sw, self.bias, self.qtype, out_dtype,
                          s_inv=self.s_inv)
        c = self._cur
        xq, sx, _ = quantize_act_tensor(x, self.s, self.qtype, amax_prev=self._amax[c:c + 1],
                                        amax_out=self._amax[1 - c:2 - c], s_inv=self.s_inv)
        self._cur = 1 - c
        g = gemm_w8a8 if self.qtype == "i8" else gemm_fp8
        return g(xq, sx, self.wq, self.sw, self.bias, out_dtype=out_dtype)


class RMSNormSmoothQuantLinear:
    """A prepared W8A8 linear layer fed by its RMS normalization:
    y = (rmsnorm(h) * gamma) @ W (+ bias), with the smoothing folded into the
    normalization's gain offline, so that one kernel normalizes and quantizes
    each token row of h at run time and the 8-bit GEMM follows.

    h_cal: calibration tokens of the normalization's input (bf16 [T, K]); the
    smoothing factors are calibrated on the normalization's output."""

    def __init__(self, w: torch.Tensor, h_cal: torch.Tensor, gamma: torch.Tensor, eps: float,
                 alpha: float = 0.5, qtype: str = "i8", bias: torch.Tensor | None = None):
        p = prepare_rmsnorm(w, h_cal, gamma, eps, alpha, qtype)
        self.s, self.g, self.wq, self.sw = p["s"], p["g"], p["wq"], p["sw"]
        self.eps, self.qtype, self.bias = float(eps), qtype, bias
        self.in_features, self.out_features = w.shape

    def __call__(self, h: torch.Tensor, out_dtype=torch.bfloat16) -> torch.Tensor:
        xq, sx = rmsnorm_quantize_act(h, self.g, self.eps, self.qtype)
        gm = gemm_w8a8 if self.qtype == "i8" else gemm_fp8
        return gm(xq, sx, self.wq, self.sw, self.bias, out_dtype=out_dtype)
