"""Pins for the oracle's dequantize-then-fp64 GEMM.

The oracle GEMM is checked against exact rational arithmetic (Python
fractions over the decoded codes, with value tables written out in this
file), a closed form, and a C brute-force triple loop.
"""
from fractions import Fraction

import numpy as np
import pytest

E2M1 = [0, Fraction(1, 2), 1, Fraction(3, 2), 2, 3, 4, 6]


def _e4m3_fraction(c):
    e, m = (c >> 3) & 15, c & 7
    if e == 0:
        return Fraction(m, 512)
    return Fraction(8 + m, 8) * (Fraction(2) ** (e - 7))


def _random_quantized(rng, rows, cols, orc, sf_range=(0x20, 0x50)):
    kb = cols // 16
    codes = rng.integers(0, 16, size=(rows, cols)).astype(np.uint8)
    q = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    sf = np.zeros(orc.sf_bytes(rows, cols), dtype=np.uint8)
    sfc = rng.integers(sf_range[0], sf_range[1], size=(rows, kb)).astype(np.uint8)
    for r in range(rows):
        for c in range(kb):
            sf[orc.sf_offset(r, c, kb)] = sfc[r, c]
    return codes, q, sf, sfc


def _exact_value(code, sfc):
    v = E2M1[code & 7] * _e4m3_fraction(int(sfc))
    return -v if code & 8 else v


@pytest.mark.parametrize("n", [16, 32])
def test_gemm_exact_rational(orc, n):
    rng = np.random.default_rng(n)
    M = N = K = n
    ac, aq, asf, asfc = _random_quantized(rng, M, K, orc)
    bc, bq, bsf, bsfc = _random_quantized(rng, N, K, orc)
    a_sdec, b_sdec = np.float32(0.25), np.float32(2.0)   # powers of two: exact
    y = orc.gemm(aq, asf, a_sdec, bq, bsf, b_sdec, M, N, K)
    for m in range(M):
        for nn in range(N):
            s = Fraction(0)
            for k in range(K):
                s += _exact_value(ac[m, k], asfc[m, k // 16]) * _exact_value(bc[nn, k], bsfc[nn, k // 16])
            s *= Fraction(1, 4) * 2
            assert Fraction(y[m, nn]) == s, (m, nn)


def test_gemm_matches_brute_force(orc):
    rng = np.random.default_rng(7)
    M, N, K = 48, 40, 64
    _, aq, asf, _ = _random_quantized(rng, M, K, orc)
    _, bq, bsf, _ = _random_quantized(rng, N, K, orc)
    y = orc.gemm(aq, asf, np.float32(0.5), bq, bsf, np.float32(0.125), M, N, K)
    a = orc.dequantize(aq, asf, np.float32(0.5), M, K)
    b = orc.dequantize(bq, bsf, np.float32(0.125), N, K)
    yn = orc.gemm_naive(a, b)
    assert np.allclose(y, yn, rtol=1e-13, atol=1e-13)
    rows = np.array([3, 0, 47, 10])
    ys = orc.gemm(aq, asf, np.float32(0.5), bq, bsf, np.float32(0.125), M, N, K, rows=rows)
    assert np.array_equal(ys, y[rows])


def test_gemm_closed_form(orc):
    # A = all code 2 (1.0) with scale 1.0 (0x38); B row n = code for value v_n.
    M, N, K = 3, 8, 64
    aq = np.full((M, K // 2), 0x22, dtype=np.uint8)
    asf = np.zeros(orc.sf_bytes(M, K), dtype=np.uint8)
    for r in range(M):
        for c in range(K // 16):
            asf[orc.sf_offset(r, c, K // 16)] = 0x38
    codes = np.arange(N, dtype=np.uint8) | np.array([0, 8] * (N // 2), dtype=np.uint8)
    bq = np.repeat((codes | (codes << 4))[:, None], K // 2, axis=1).astype(np.uint8)
    bsf = asf[: orc.sf_bytes(N, K)].copy()
    bsf[:] = 0
    for r in range(N):
        for c in range(K // 16):
            bsf[orc.sf_offset(r, c, K // 16)] = 0x38
    y = orc.gemm(aq, asf, np.float32(1.0), bq, bsf, np.float32(1.0), M, N, K)
    want = np.array([float(E2M1[c & 7]) * (-1 if c & 8 else 1) * K for c in codes])
    assert np.array_equal(y, np.tile(want, (M, 1)))


def test_tolerance_rule(orc):
    ref = np.array([1.0, -2.0, 0.0, 100.0])
    rms = np.sqrt(np.mean(ref ** 2))
    ok, _ = orc.gemm_tolerance_ok(ref + 0.99e-2 * (np.abs(ref) + rms), ref)
    assert ok
    ok, worst = orc.gemm_tolerance_ok(ref + np.array([0, 0, 1.01e-2 * rms, 0]), ref)
    assert not ok and worst > 1.0
