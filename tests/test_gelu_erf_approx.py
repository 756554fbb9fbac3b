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
    body = text[text.index("__device__ __forceinline__ float gelu_erf"):]
    body = body[:body.index("}")]
    vals = dict(re.findall(r"(p|a[1-5]) = (-?[0-9.]+)f", body))
    return {k: float(v) for k, v in vals.items()}


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
