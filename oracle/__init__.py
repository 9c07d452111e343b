"""Plain CPU oracle for the SmoothQuant W8A8 linear layer (ctypes binding).

TEST INFRASTRUCTURE, NOT PRODUCT CODE: only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline / reference leg of
``bench.py`` may import this package. The arithmetic lives in
``sq_oracle.c`` (plain C, binary32 steps, no FMA contraction); this module only
builds it with gcc and marshals numpy arrays. It never imports the CUDA
package and the CUDA package never imports it.

Sources: "Weight-Activation Quantization" (infra.bea.ai) §2-§4 and the
zenaique flashcard "Define activation quantization ..." -- see the header of
``sq_oracle.c`` for the passage each function follows and the readings taken
where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sq_oracle.c")
_HDR = os.path.join(_HERE, "sq_oracle.h")
_LIB = os.path.join(_HERE, "libsq_oracle.so")
_lock = threading.Lock()
_lib = None

INT8 = 0
E4M3 = 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, no FMA contraction, OpenMP)."""
    stale = (not os.path.exists(_LIB)) or any(
        os.path.getmtime(p) > os.path.getmtime(_LIB) for p in (_SRC, _HDR))
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math",
               "-fopenmp", "-fPIC", "-shared", "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            I = ctypes.c_int
            lib.sqo_bf16_to_f32.argtypes = [ctypes.c_uint16]
            lib.sqo_bf16_to_f32.restype = ctypes.c_float
            lib.sqo_f32_to_bf16_rne.argtypes = [ctypes.c_float]
            lib.sqo_f32_to_bf16_rne.restype = ctypes.c_uint16
            lib.sqo_f32_to_bf16_rne_n.argtypes = [P, P, I64]
            lib.sqo_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.sqo_e4m3_decode.restype = ctypes.c_double
            lib.sqo_e4m3_encode_rn_sat.argtypes = [ctypes.c_float]
            lib.sqo_e4m3_encode_rn_sat.restype = ctypes.c_uint8
            lib.sqo_amax.argtypes = [P, I, I64, I64, I, P]
            lib.sqo_smooth_factors.argtypes = [P, P, I64, ctypes.c_double, P]
            lib.sqo_smooth_act.argtypes = [P, I, I64, I64, P, P]
            lib.sqo_smooth_weight.argtypes = [P, I, I64, I64, P, P]
            lib.sqo_fold_smoothing.argtypes = [P, I, I64, I64, P, I, P]
            lib.sqo_quantize_weight.argtypes = [P, I, I64, I64, P, I, P, P]
            lib.sqo_quantize_act.argtypes = [P, I, I64, I64, P, I, P, P]
            lib.sqo_quantize_act_tensor.argtypes = [P, I, I64, I64, P, I, P, P, P, P]
            lib.sqo_rmsnorm_quantize_act.argtypes = [P, I64, I64, P, ctypes.c_float, I, P, P,
                                                     P, P]
            lib.sqo_gemm_i8.argtypes = [P, P, I64, I64, I64, P]
            lib.sqo_gemm_e4m3.argtypes = [P, P, I64, I64, I64, P]
            lib.sqo_dequant.argtypes = [ctypes.c_float, ctypes.c_float,
                                        ctypes.c_float, I, ctypes.c_uint16]
            lib.sqo_dequant.restype = ctypes.c_float
            lib.sqo_epilogue.argtypes = [P, P, I, P, P, P, I64, I64, P, P]
            lib.sqo_linear_at.argtypes = [P, P, P, P, P, I, I64, P, P, I64,
                                          P, P, P]
            lib.sqo_num_threads.restype = I
            lib.sqo_quantize_weight_i4.argtypes = [P, I, I64, I64, P, P]
            lib.sqo_unpack_i4.argtypes = [P, I64, I64, P]
            lib.sqo_gemm_weight_only.argtypes = [P, P, I, P, P, I64, I64, I64, P]
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _dtype_code(x):
    if x.dtype == np.float32:
        return 0
    if x.dtype == np.uint16:  # raw bf16 bit patterns
        return 1
    raise TypeError(f"oracle input must be float32 or bf16 bits (uint16), got {x.dtype}")


def num_threads() -> int:
    return int(_load().sqo_num_threads())


# ---- number formats --------------------------------------------------------

def bf16_to_f32(h) -> np.ndarray:
    """Widen raw bf16 bit patterns to float32 (exact: the bits move up 16)."""
    lib = _load()
    h = _c(h, np.uint16)
    flat = h.reshape(-1)
    out = np.array([lib.sqo_bf16_to_f32(int(v)) for v in flat], np.float32)
    return out.reshape(h.shape)


def bf16_to_f32_array(h) -> np.ndarray:
    """bf16_to_f32 for whole arrays: the bits move up 16 (exact)."""
    h = _c(h, np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(x) -> np.ndarray:
    """Round float32 to bf16 (nearest-even), returned as raw uint16 bits."""
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    _load().sqo_f32_to_bf16_rne_n(_ptr(x), _ptr(out), x.size)
    return out


def e4m3_decode(codes) -> np.ndarray:
    lib = _load()
    table = np.array([lib.sqo_e4m3_decode(c) for c in range(256)], np.float64)
    return table[_c(codes, np.uint8)]


def e4m3_encode(x) -> np.ndarray:
    lib = _load()
    x = _c(x, np.float32)
    flat = x.reshape(-1)
    out = np.empty(flat.shape, np.uint8)
    f = lib.sqo_e4m3_encode_rn_sat
    for i in range(flat.size):
        out[i] = f(float(flat[i]))
    return out.reshape(x.shape)


# ---- the four stages -------------------------------------------------------

def amax(x: np.ndarray, per_column: bool) -> np.ndarray:
    """a1 (per_column=True: max over rows) / a2 (per_column=False: max over columns)."""
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    out = np.empty(cols if per_column else rows, np.float32)
    _load().sqo_amax(_ptr(x), _dtype_code(x), rows, cols, int(per_column), _ptr(out))
    return out


def smooth_act(x: np.ndarray, s) -> np.ndarray:
    """X~ = X diag(s)^-1 (float32), before any quantization."""
    x = np.ascontiguousarray(x)
    M, K = x.shape
    s = _c(s, np.float32)
    out = np.empty((M, K), np.float32)
    _load().sqo_smooth_act(_ptr(x), _dtype_code(x), M, K, _ptr(s), _ptr(out))
    return out


def smooth_weight(w: np.ndarray, s) -> np.ndarray:
    """W~ = diag(s) W (float32), before any quantization."""
    w = np.ascontiguousarray(w)
    K, N = w.shape
    s = _c(s, np.float32)
    out = np.empty((K, N), np.float32)
    _load().sqo_smooth_weight(_ptr(w), _dtype_code(w), K, N, _ptr(s), _ptr(out))
    return out


def fold_smoothing(p: np.ndarray, s, per_column: bool = True) -> np.ndarray:
    """The producer's per-channel parameters divided by s (float32): channel =
    column (per_column) or row; the producer then emits X~ = X diag(s)^-1."""
    p = np.ascontiguousarray(p)
    if p.ndim == 1:
        p = p.reshape(1, -1) if per_column else p.reshape(-1, 1)
    rows, cols = p.shape
    s = _c(s, np.float32)
    if s.size != (cols if per_column else rows):
        raise ValueError("s must have one entry per channel")
    out = np.empty((rows, cols), np.float32)
    _load().sqo_fold_smoothing(_ptr(p), _dtype_code(p), rows, cols, _ptr(s), int(per_column),
                               _ptr(out))
    return out


def smooth_factors(amax_x, amax_w, alpha: float) -> np.ndarray:
    ax = _c(amax_x, np.float32)
    aw = _c(amax_w, np.float32)
    s = np.empty(ax.shape, np.float32)
    _load().sqo_smooth_factors(_ptr(ax), _ptr(aw), ax.size, float(alpha), _ptr(s))
    return s


def quantize_weight(w: np.ndarray, s, qtype: int = INT8):
    """Returns (wq [N,K] int8 or uint8 E4M3 codes, sw [N] float32)."""
    w = np.ascontiguousarray(w)
    K, N = w.shape
    s = None if s is None else _c(s, np.float32)
    wq = np.empty((N, K), np.uint8 if qtype == E4M3 else np.int8)
    sw = np.empty(N, np.float32)
    _load().sqo_quantize_weight(_ptr(w), _dtype_code(w), K, N, _ptr(s), qtype,
                                _ptr(wq), _ptr(sw))
    return wq, sw


def quantize_act(x: np.ndarray, s, qtype: int = INT8):
    """Returns (xq [M,K] int8 or uint8 E4M3 codes, sx [M] float32)."""
    x = np.ascontiguousarray(x)
    M, K = x.shape
    s = None if s is None else _c(s, np.float32)
    xq = np.empty((M, K), np.uint8 if qtype == E4M3 else np.int8)
    sx = np.empty(M, np.float32)
    _load().sqo_quantize_act(_ptr(x), _dtype_code(x), M, K, _ptr(s), qtype,
                             _ptr(xq), _ptr(sx))
    return xq, sx


def rmsnorm_quantize_act(x_bf16: np.ndarray, g, eps: float, qtype: int = INT8):
    """The producer of X with the smoothing folded in: RMS normalization of
    each row of x (bf16 bits [M,K]) with gain g [K] (= gamma / s), then
    per-token quantization. The sum of squares is exact over the elements
    whose bf16 exponent is within 48 of the row's largest (the rest are below
    2^-94 of the largest square), rounded once to binary64; 1/sqrt(ss/K +
    eps) in binary64 steps, rounded to binary32; xn = (x * r) * g in binary32.
    Returns (xq [M,K] codes, sx [M], r [M] float32, xn [M,K] float32)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    M, K = x.shape
    g = _c(g, np.float32)
    xq = np.empty((M, K), np.uint8 if qtype == E4M3 else np.int8)
    sx = np.empty(M, np.float32)
    r = np.empty(M, np.float32)
    xn = np.empty((M, K), np.float32)
    _load().sqo_rmsnorm_quantize_act(_ptr(x), M, K, _ptr(g), float(eps), qtype, _ptr(xq),
                                     _ptr(sx), _ptr(r), _ptr(xn))
    return xq, sx, r, xn


def quantize_act_tensor(x: np.ndarray, s, qtype: int = INT8, scale=None):
    """Per-tensor scaling: one scale for the whole (smoothed) tensor, the
    online max|x/s|/Q when `scale` is None, else the given (delayed) scale.
    Returns (xq [M,K] codes, scale used as float32, amax = max|x/s|)."""
    x = np.ascontiguousarray(x)
    M, K = x.shape
    s = None if s is None else _c(s, np.float32)
    sc = None if scale is None else np.array([scale], np.float32)
    xq = np.empty((M, K), np.uint8 if qtype == E4M3 else np.int8)
    sx = np.empty(max(M, 1), np.float32)
    amax = np.zeros(1, np.float32)
    _load().sqo_quantize_act_tensor(_ptr(x), _dtype_code(x), M, K, _ptr(s), qtype, _ptr(sc),
                                    _ptr(xq), _ptr(sx), _ptr(amax))
    used = np.float32(scale) if scale is not None else (sx[0] if M else np.float32(0))
    return xq, np.float32(used), np.float32(amax[0])


def gemm_i8(xq, wq) -> np.ndarray:
    xq = _c(xq, np.int8)
    wq = _c(wq, np.int8)
    M, K = xq.shape
    N = wq.shape[0]
    assert wq.shape[1] == K
    acc = np.empty((M, N), np.int32)
    _load().sqo_gemm_i8(_ptr(xq), _ptr(wq), M, N, K, _ptr(acc))
    return acc


def gemm_e4m3(xq, wq) -> np.ndarray:
    xq = _c(xq, np.uint8)
    wq = _c(wq, np.uint8)
    M, K = xq.shape
    N = wq.shape[0]
    assert wq.shape[1] == K
    acc = np.empty((M, N), np.float64)
    _load().sqo_gemm_e4m3(_ptr(xq), _ptr(wq), M, N, K, _ptr(acc))
    return acc


def dequant(acc_f32: float, sx_m: float, sw_n: float, bias_bf16=None) -> np.float32:
    lib = _load()
    return np.float32(lib.sqo_dequant(float(acc_f32), float(sx_m), float(sw_n),
                                      int(bias_bf16 is not None),
                                      0 if bias_bf16 is None else int(bias_bf16)))


def epilogue(acc, sx, sw, bias=None):
    """Returns (y_f32 [M,N] float32, y_bf16 [M,N] uint16)."""
    sx = _c(sx, np.float32)
    sw = _c(sw, np.float32)
    bias = None if bias is None else _c(bias, np.uint16)
    if acc.dtype == np.int32:
        a32, a64, kind = _c(acc, np.int32), None, 0
    else:
        a32, a64, kind = None, _c(acc, np.float64), 1
    M, N = acc.shape
    yf = np.empty((M, N), np.float32)
    yb = np.empty((M, N), np.uint16)
    _load().sqo_epilogue(_ptr(a32), _ptr(a64), kind, _ptr(sx), _ptr(sw), _ptr(bias),
                         M, N, _ptr(yf), _ptr(yb))
    return yf, yb


def linear_at(xq, sx, wq, sw, bias, rows, cols, qtype: int = INT8):
    """Sampled outputs: (acc float64, y_f32, y_bf16) at (rows[i], cols[i])."""
    xq = np.ascontiguousarray(xq)
    wq = np.ascontiguousarray(wq)
    K = xq.shape[1]
    sx = _c(sx, np.float32)
    sw = _c(sw, np.float32)
    bias = None if bias is None else _c(bias, np.uint16)
    rows = _c(rows, np.int64)
    cols = _c(cols, np.int64)
    n = rows.size
    acc = np.empty(n, np.float64)
    yf = np.empty(n, np.float32)
    yb = np.empty(n, np.uint16)
    _load().sqo_linear_at(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), _ptr(bias), qtype,
                          K, _ptr(rows), _ptr(cols), n, _ptr(acc), _ptr(yf), _ptr(yb))
    return acc, yf, yb


def linear(x, s, wq, sw, bias=None, qtype: int = INT8):
    """End-to-end runtime path a5 -> a6/a7 -> epilogue on full matrices."""
    xq, sx = quantize_act(x, s, qtype)
    acc = gemm_e4m3(xq, wq) if qtype == E4M3 else gemm_i8(xq, wq)
    yf, yb = epilogue(acc, sx, sw, bias)
    return dict(xq=xq, sx=sx, acc=acc, y_f32=yf, y_bf16=yb)


# ---- weight-only quantization (W8A16 / W4A16) -------------------------------

def quantize_weight_i4(w: np.ndarray):
    """Per-output-channel symmetric INT4 weights: (wq4 [N, K/2] uint8, sw [N]
    float32 = amax / 7). Each 32-bit little-endian word packs the codes of 8
    consecutive k: the even ones in bits 0,4,8,12, the odd ones in 16,20,24,28."""
    w = np.ascontiguousarray(w)
    K, N = w.shape
    if K % 8:
        raise ValueError("K must be a multiple of 8 for packed INT4 weights")
    wq4 = np.empty((N, K // 2), np.uint8)
    sw = np.empty(N, np.float32)
    _load().sqo_quantize_weight_i4(_ptr(w), _dtype_code(w), K, N, _ptr(wq4), _ptr(sw))
    return wq4, sw


def unpack_i4(wq4: np.ndarray) -> np.ndarray:
    """Codes (int8 [N, K]) of packed INT4 weights [N, K/2]."""
    wq4 = _c(wq4, np.uint8)
    N, half = wq4.shape
    codes = np.empty((N, 2 * half), np.int8)
    _load().sqo_unpack_i4(_ptr(wq4), N, 2 * half, _ptr(codes))
    return codes


def gemm_weight_only(x, wq, sw, bias=None, bits: int = 8) -> np.ndarray:
    """y = x @ (codes * sw).T + bias in binary64 (x: bf16 bits [M,K]; wq: int8
    [N,K] for bits 8, packed uint8 [N,K/2] for bits 4, see quantize_weight_i4)."""
    x = _c(x, np.uint16)
    M, K = x.shape
    wq = np.ascontiguousarray(wq)
    N = wq.shape[0]
    if bits == 8:
        assert wq.dtype == np.int8 and wq.shape[1] == K
    elif bits == 4:
        assert wq.dtype == np.uint8 and 2 * wq.shape[1] == K
    else:
        raise ValueError("bits must be 8 or 4")
    sw = _c(sw, np.float32)
    bias = None if bias is None else _c(bias, np.uint16)
    y = np.empty((M, N), np.float64)
    _load().sqo_gemm_weight_only(_ptr(x), _ptr(wq), bits, _ptr(sw), _ptr(bias), M, N, K, _ptr(y))
    return y
