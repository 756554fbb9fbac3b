"""Pins of the oracle's exact GELU, g(h) = h * Phi(h), against facts of the
standard normal CDF that the oracle does not compute (the activation of the
fused FFN up-projection epilogue; "NVIDIA показала, как сократить генерацию
FLUX 3 Image Klein с 22 до 6 секунд", section "Квантование NVFP4 и
оптимизация вычислительных ядер": fused GEMM kernels)."""
import numpy as np

import oracle

# Phi(1) and Phi(2) from standard normal tables (to 16 digits).
PHI_1 = 0.8413447460685429
PHI_2 = 0.9772498680518208


def test_gelu_table_values():
    g = oracle.gelu(np.array([1.0, -1.0, 2.0, -2.0, 0.0]))
    assert abs(g[0] - PHI_1) < 1e-15
    assert abs(g[1] - (-(1.0 - PHI_1))) < 1e-15
    assert abs(g[2] - 2.0 * PHI_2) < 2e-15
    assert abs(g[3] - (-2.0 * (1.0 - PHI_2))) < 2e-15
    assert g[4] == 0.0


def test_gelu_odd_part_is_identity():
    """Phi(h) + Phi(-h) = 1, so g(h) - g(-h) = h for every h."""
    h = np.random.default_rng(0).normal(0, 3, 100000)
    d = oracle.gelu(h) - oracle.gelu(-h)
    assert np.max(np.abs(d - h) / np.maximum(1.0, np.abs(h))) < 1e-14


def test_gelu_slope_and_limits():
    eps = 1e-6
    slope0 = (oracle.gelu(np.array([eps]))[0] - oracle.gelu(np.array([-eps]))[0]) / (2 * eps)
    assert abs(slope0 - 0.5) < 1e-9                     # g'(0) = Phi(0) = 1/2
    assert oracle.gelu(np.array([40.0]))[0] == 40.0     # Phi(40) rounds to 1
    assert oracle.gelu(np.array([-40.0]))[0] == 0.0 or abs(oracle.gelu(np.array([-40.0]))[0]) < 1e-300


def test_gelu_minimum():
    """g has its single minimum where Phi(h) + h phi(h) = 0, h ~ -0.7518 with
    g ~ -0.16997 (a plausible sign or factor error moves both)."""
    h = np.linspace(-3, 1, 400001)
    g = oracle.gelu(h)
    i = int(np.argmin(g))
    assert abs(h[i] - (-0.75179)) < 2e-4
    assert abs(g[i] - (-0.169971)) < 2e-6
