"""The fused FFN epilogue evaluates erf with Abramowitz & Stegun, Handbook of
Mathematical Functions, formula 7.1.26 (Hastings' rational approximation,
|error| <= 1.5e-7 for x >= 0), the activation of the pages' fused GEMM
kernels ("NVIDIA показала, как сократить генерацию FLUX 3 Image Klein с 22
до 6 секунд", section "Квантование NVFP4 и оптимизация вычислительных
ядер").  This pins the coefficients as the kernel spells them: the same
formula in fp64 must stay within the published bound of scipy's erf over a
dense grid, and a single mistyped coefficient must break the bound."""
import re
from pathlib import Path

import numpy as np
from scipy.special import erf

SRC = Path(__file__).resolve().parents[1] / "nvfp4_block_scaled_19_b200" / "csrc" / "gemm_common.cuh"


def _coefficients():
    text = SRC.read_text()
    vals = dict(re.findall(r"kAs(P|A[1-5]) = (-?[0-9.]+)f", text))
    return {k.lower(): float(v) for k, v in vals.items()}


def _erf_as(x, c):
    t = 1.0 / (1.0 + c["p"] * x)
    poly = t * (c["a1"] + t * (c["a2"] + t * (c["a3"] + t * (c["a4"] + t * c["a5"]))))
    return 1.0 - poly * np.exp(-x * x)


def test_kernel_coefficients_meet_published_bound():
    c = _coefficients()
    assert set(c) == {"p", "a1", "a2", "a3", "a4", "a5"}
    x = np.linspace(0.0, 8.0, 2_000_001)
    assert np.max(np.abs(_erf_as(x, c) - erf(x))) <= 1.5e-7


def test_bound_detects_a_mistyped_coefficient():
    c = _coefficients()
    x = np.linspace(0.0, 8.0, 200_001)
    for k in c:
        bad = dict(c)
        bad[k] *= 1.001
        assert np.max(np.abs(_erf_as(x, bad) - erf(x))) > 1.5e-7, k


def _gelu_folded(h, c):
    """The kernel's arrangement: g = max(h, 0) - |h| erfc(|h|/sqrt 2) / 2, with
    t = 1 / (1 + (p / sqrt 2) |h|), the 1/2 folded into the coefficients and
    exp(-h^2 / 2) written as 2^(h^2 (-log2(e) / 2))."""
    b = {k: 0.5 * c[k] for k in ("a1", "a2", "a3", "a4", "a5")}
    ah = np.abs(h)
    t = 1.0 / (1.0 + c["p"] / np.sqrt(2.0) * ah)
    poly = t * (b["a1"] + t * (b["a2"] + t * (b["a3"] + t * (b["a4"] + t * b["a5"]))))
    half_c = poly * np.exp2(h * h * (-np.log2(np.e) / 2.0))
    return np.maximum(h, 0.0) - ah * half_c


def test_folded_gelu_matches_exact_gelu():
    """Both signs of h through the one expression: within |h| * 1.5e-7 / 2 of
    0.5 h (1 + erf(h / sqrt 2)) (the erf bound carried through), and a sign
    or factor slip in the arrangement breaks that."""
    c = _coefficients()
    h = np.linspace(-12.0, 12.0, 1_200_001)
    exact = 0.5 * h * (1.0 + erf(h / np.sqrt(2.0)))
    bound = np.abs(h) * 0.5 * 1.5e-7 + 1e-300
    assert np.all(np.abs(_gelu_folded(h, c) - exact) <= bound)
    wrong_sign = np.maximum(h, 0.0) + (np.maximum(h, 0.0) - _gelu_folded(h, c))
    assert np.any(np.abs(wrong_sign - exact) > bound)
    no_half = 2.0 * _gelu_folded(h, c) - np.maximum(h, 0.0)
    assert np.any(np.abs(no_half - exact) > bound)
