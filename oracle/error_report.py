"""Quantization error of the NVFP4 linear layer, measured with the oracle.

TEST INFRASTRUCTURE ONLY (as the rest of oracle/): informational, not a
pass/fail bar.  For a layer Y = X . W^T with bf16 X [M, K] and W [N, K], the
NVFP4 product takes X with its dynamic per-tensor scale and W with its static
one (both S_enc = 2688 / amax of the tensor, E4M3 block scales per 16
elements along K, E2M1 elements), dequantizes both and multiplies in fp64.
The error is the relative Frobenius norm of its difference from the exact
product of the bf16 inputs (also fp64), over a seeded sample of rows of Y
(every column).  The FP8 variant (E4M3 elements, one per-tensor scale) is
measured the same way for comparison.

Run as a script to print the table for every single-layer workload:
    python -m oracle.error_report [rows_per_layer]
"""
from __future__ import annotations

import sys

import numpy as np
import torch

from . import dequantize, gemm, gemm_fp8, quantize_dynamic, quantize_fp8


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def layer_error(x: torch.Tensor, w: torch.Tensor, rows: np.ndarray) -> dict:
    """Relative Frobenius errors of the NVFP4 and FP8 products against the
    exact product of the bf16 inputs, on rows `rows` of Y."""
    M, K = x.shape
    N = w.shape[0]
    xb, wb = _bits(x), _bits(w)
    ref = x[torch.from_numpy(rows)].double().numpy() @ w.double().numpy().T
    norm = np.linalg.norm(ref)
    aq, asf, asd, _ = quantize_dynamic(xb, M, K)
    bq, bsf, bsd, _ = quantize_dynamic(wb, N, K)
    y4 = gemm(aq, asf, asd, bq, bsf, bsd, M, N, K, rows=rows)
    fq, fsd, _ = quantize_fp8(xb, M, K)
    gq, gsd, _ = quantize_fp8(wb, N, K)
    y8 = gemm_fp8(fq, fsd, gq, gsd, rows=rows)
    return {"nvfp4": float(np.linalg.norm(y4 - ref) / norm),
            "fp8": float(np.linalg.norm(y8 - ref) / norm),
            "x_nvfp4": float(np.linalg.norm(dequantize(aq, asf, asd, M, K, rows)
                                            - x[torch.from_numpy(rows)].double().numpy())
                             / np.linalg.norm(x[torch.from_numpy(rows)].double().numpy()))}


def sample_rows(M: int, n: int, seed: int = 0) -> np.ndarray:
    """n distinct rows of M (all rows when n >= M), sorted, seeded."""
    if n >= M:
        return np.arange(M)
    return np.sort(np.random.default_rng(seed).choice(M, size=n, replace=False))


def main(n_rows: int = 256) -> None:
    sys.path.insert(0, ".")
    from workloads import WORKLOADS, layer_inputs  # seeded input generators only

    print("| workload | layer | M x K -> N | rows | X error (NVFP4) | Y error NVFP4 | Y error FP8 |")
    print("|---|---|---|---|---|---|---|")
    for name, wl in WORKLOADS.items():
        if len(wl.layers) != 1 and name != "block_chain_2048":
            continue
        for li, spec in enumerate(wl.layers):
            x, w = layer_inputs(wl, li)
            rows = sample_rows(x.shape[0], n_rows)
            e = layer_error(x, w, rows)
            print(f"| {name} | {spec.name} | {x.shape[0]} x {x.shape[1]} -> {w.shape[0]} | "
                  f"{len(rows)} | {e['x_nvfp4']:.4f} | {e['nvfp4']:.4f} | {e['fp8']:.4f} |",
                  flush=True)


if __name__ == "__main__":
    main(int(sys.argv[1]) if len(sys.argv) > 1 else 256)
