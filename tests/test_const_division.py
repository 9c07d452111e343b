"""Exhaustive CPU check of the row-scale division used by the activation
kernel: sx = RN(amax / Q) for Q = 127 (INT8) and Q = 448 (E4M3) computed as
q0 = RN(a*c), e = a - Q*q0 (one fused multiply-add, exact), RN(q0 + e*c)
with the constant c = RN(1/Q) (Markstein's correction step). Every binary32
significand a in [1, 2) is run in exact integer arithmetic; the correctly
rounded quotient is the reference. Scaling a by a power of two scales every
intermediate exactly, so this covers every a whose quotient and residual stay
normal. The uncorrected product q0 must fail somewhere (the check has teeth).
"""
import numpy as np
import pytest


def _bitlen(v):
    """Number of significant bits of each positive int64."""
    b = np.floor(np.log2(v.astype(np.float64))).astype(np.int64) + 1
    b = np.where((v >> np.maximum(b - 1, 0)) == 0, b - 1, b)
    return np.where((v >> b) != 0, b + 1, b)


def _round_sig(v, sticky, nbits=24):
    """Round positive integers v (with a sticky flag for discarded nonzero
    bits below v) to nbits significant bits, ties to even. Returns
    (mantissa, exponent shift)."""
    sh = np.maximum(_bitlen(v) - nbits, 0)
    q = v >> sh
    low = v - (q << sh)
    half = np.where(sh > 0, np.int64(1) << np.maximum(sh - 1, 0), 0)
    above = (low > half) | ((low == half) & sticky)
    tie = (low == half) & ~sticky
    up = (sh > 0) & (above | (tie & (q & 1 == 1)))
    q = q + up
    carry = q >> nbits
    return np.where(carry > 0, q >> 1, q), sh + carry


@pytest.mark.parametrize("Q", [127, 448])
def test_constant_reciprocal_division_is_exact(Q):
    # a = A * 2^-23 in [1, 2), in blocks of 2^20 significands
    naive_fail = 0
    for lo in range(1 << 23, 1 << 24, 1 << 20):
        naive_fail += _check_block(np.arange(lo, lo + (1 << 20), dtype=np.int64), Q)
    # the uncorrected product is not exact on every significand
    assert naive_fail > 1000


def _check_block(A, Q):
    k = int(np.ceil(np.log2(Q)))                           # 2^(k-1) < Q < 2^k
    # c = RN(1/Q) = C * 2^cexp, C a 24-bit integer
    C, r = divmod(1 << (23 + k), Q)
    if 2 * r > Q or (2 * r == Q and C & 1):
        C += 1
    assert (1 << 23) <= C < (1 << 24)
    cexp = -(23 + k)
    assert np.float32(C * 2.0 ** cexp) == np.float32(1.0) / np.float32(Q)
    zero = np.zeros(A.shape, bool)
    # q0 = RN(a * c): the product A*C is exact in int64
    Q0, s0 = _round_sig(A * C, zero)
    e0 = s0 - 23 + cexp                                    # q0 = Q0 * 2^e0
    assert (e0 <= -23).all()
    # e = a - Q*q0 on the grid 2^e0; exactly representable (fits 24 bits)
    E = (A << (-23 - e0)) - Q * Q0
    assert (np.abs(E) < (1 << 24)).all()
    # q1 = RN(q0 + e*c) = RN((Q0 * 2^-cexp + E*C) * 2^(e0 + cexp))
    T = (Q0 << (-cexp)) + E * C
    assert (T > 0).all()
    Q1, s1 = _round_sig(T, zero)
    e1 = s1 + e0 + cexp
    # reference: RN(A / Q * 2^-23) from the integer quotient with a sticky bit
    D, rem = np.divmod(A << 38, Q)
    Qr, sr = _round_sig(D, rem > 0)
    er = sr - 38 - 23
    assert np.array_equal(Q1, Qr) and np.array_equal(e1, er)
    return int((~((Q0 == Qr) & (e0 == er))).sum())
