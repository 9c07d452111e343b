"""Helpers for the GPU parity tests: numpy <-> torch transfers and the error
metric used for the FP8 path (no arithmetic of the layer itself)."""
import numpy as np
import torch

import oracle


def dev(a: np.ndarray) -> torch.Tensor:
    """numpy -> CUDA tensor; uint16 arrays are raw bf16 bit patterns."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    """CUDA tensor -> numpy; bf16 comes back as raw uint16 bit patterns."""
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def ulp_distance(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in binary32 units in the last place (same-sign finite values)."""
    ai = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    bi = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    return np.abs(ai - bi)


def fp8_normalized_error(y, y_ref, xq, wq, sx, sw, bias, rows, cols, chunk=512):
    """|y - y_ref| / (sx*sw*sum_k |a_k b_k| + |bias|) at sampled (rows, cols):
    the accumulated-rounding error measured against the magnitude of the terms
    summed, so that cancellation near y = 0 does not inflate it."""
    table = np.abs(oracle.e4m3_decode(np.arange(256, dtype=np.uint8)))
    out = np.empty(len(rows), np.float64)
    for i in range(0, len(rows), chunk):
        r, c = rows[i:i + chunk], cols[i:i + chunk]
        mag = (table[xq[r]] * table[wq[c]]).sum(axis=1)
        den = sx[r].astype(np.float64) * sw[c].astype(np.float64) * mag
        if bias is not None:
            den = den + np.abs(oracle.bf16_to_f32(bias[c]).astype(np.float64))
        num = np.abs(np.asarray(y[i:i + chunk], np.float64) - np.asarray(y_ref[i:i + chunk], np.float64))
        out[i:i + chunk] = np.where(den > 0, num / np.where(den > 0, den, 1.0), num)
    return out


def sample_points(M, N, seed, n_random=4096, full_rows=4, full_cols=4):
    """(rows, cols) covering a few complete rows and columns (first, last and
    random ones, so every tile edge is hit) plus uniformly random points."""
    g = np.random.default_rng(seed)
    rsel = np.unique(np.concatenate([[0, M - 1], g.integers(0, M, max(0, full_rows - 2))]))
    csel = np.unique(np.concatenate([[0, N - 1], g.integers(0, N, max(0, full_cols - 2))]))
    rows = [np.repeat(rsel, N), np.tile(np.arange(M), csel.size), g.integers(0, M, n_random)]
    cols = [np.tile(np.arange(N), rsel.size), np.repeat(csel, M), g.integers(0, N, n_random)]
    return np.concatenate(rows).astype(np.int64), np.concatenate(cols).astype(np.int64)


def fp8_error_denominator(xq, wq, sx, sw, bias, rows_per_chunk=1024):
    """sx[m]*sw[n]*sum_k |a_mk b_nk| + |bias[n]| for every output element: the
    magnitude sums as one binary64 matrix product per row block."""
    table = np.abs(oracle.e4m3_decode(np.arange(256, dtype=np.uint8)))
    b_mag = table[np.ascontiguousarray(wq)].T.copy()                 # [K,N]
    sw64 = np.asarray(sw, np.float64)
    bias_abs = 0.0 if bias is None else np.abs(oracle.bf16_to_f32_array(bias).astype(np.float64))
    M = xq.shape[0]
    den = np.empty((M, b_mag.shape[1]), np.float64)
    for r0 in range(0, M, rows_per_chunk):
        r1 = min(M, r0 + rows_per_chunk)
        mag = table[np.ascontiguousarray(xq[r0:r1])] @ b_mag
        den[r0:r1] = np.asarray(sx[r0:r1], np.float64)[:, None] * sw64[None, :] * mag + bias_abs
    return den


def fp8_normalized_error_full(y, y_ref, xq=None, wq=None, sx=None, sw=None, bias=None, den=None):
    """The same metric as fp8_normalized_error on whole [M,N] outputs (pass
    `den` from fp8_error_denominator to reuse it across outputs)."""
    if den is None:
        den = fp8_error_denominator(xq, wq, sx, sw, bias)
    num = np.abs(np.asarray(y, np.float64) - np.asarray(y_ref, np.float64))
    return np.where(den > 0, num / np.where(den > 0, den, 1.0), num)


def weight_only_error_denominator(x_bf16, codes, sw, bias):
    """sw[n] * sum_k |x[m,k] q[n,k]| + |bias[n]| for the weight-only GEMM: the
    magnitude its binary32 accumulation error is measured against."""
    xa = np.abs(oracle.bf16_to_f32_array(x_bf16).astype(np.float64))
    mag = xa @ np.abs(codes.astype(np.float64)).T
    den = mag * np.asarray(sw, np.float64)[None, :]
    if bias is not None:
        den = den + np.abs(oracle.bf16_to_f32_array(bias).astype(np.float64))[None, :]
    return np.where(den > 0, den, 1.0)
