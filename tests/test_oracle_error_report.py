"""The oracle's quantization-error report (informational figures) pinned to
facts that do not come from it: inputs built from exactly representable
NVFP4 values reproduce the exact product, and on Gaussian-like DiT inputs the
product's error is the two operands' independent errors added in quadrature.
"""
import numpy as np
import torch

from oracle.error_report import layer_error, sample_rows
from workloads import WORKLOADS, layer_inputs

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _representable(rows: int, cols: int, seed: int) -> torch.Tensor:
    """Blocks of 16 whose amax is 6 * 2^e (e in [-6, 0]) and whose elements
    are E2M1 values times 2^e: with the tensor amax 6, S_enc = 448 and every
    block scale 448 * 2^e is an E4M3 value, so the codes reproduce each
    element up to the fp32 rounding of S_dec = 1 / 448."""
    rng = np.random.default_rng(seed)
    v = rng.choice(E2M1, size=(rows, cols)) * rng.choice([-1.0, 1.0], size=(rows, cols))
    v[:, ::16] = 6.0                                   # every block reaches its amax
    e = rng.integers(-6, 1, size=(rows, cols // 16))
    e[0, 0] = 0                                        # tensor amax 6
    v = v * np.repeat(2.0 ** e, 16, axis=1)
    return torch.from_numpy(v).to(torch.bfloat16)


def test_representable_inputs_give_the_exact_product():
    x = _representable(64, 256, 1)
    w = _representable(48, 256, 2)
    e = layer_error(x, w, np.arange(64))
    assert e["x_nvfp4"] < 1e-7
    assert e["nvfp4"] < 1e-6


def test_sample_rows():
    assert np.array_equal(sample_rows(10, 20), np.arange(10))
    r = sample_rows(1000, 64, seed=3)
    assert len(r) == 64 and len(set(r.tolist())) == 64 and np.all(np.diff(r) > 0)


def test_errors_add_in_quadrature_on_dit_inputs():
    wl = WORKLOADS["tiny_linear"]
    x, w = layer_inputs(wl, 0)
    e = layer_error(x, w, np.arange(x.shape[0]))
    # Per-16 E4M3 block scales with E2M1 elements: ~9% relative on a tensor.
    assert 0.07 < e["x_nvfp4"] < 0.12
    # X and W contribute independent errors of about the same size.
    assert abs(e["nvfp4"] / e["x_nvfp4"] - np.sqrt(2.0)) < 0.15
    # Three mantissa bits per element beat one, even with a single scale.
    assert e["fp8"] < 0.5 * e["nvfp4"]
