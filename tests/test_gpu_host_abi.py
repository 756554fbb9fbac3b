"""GPU parity of the host-memory entry point nvfp4_linear_host (the call the
bench's end-to-end number goes through): pinned host X in, host Y out, the
copies, the activation quantize and the GEMM all enqueued by the library.
Checked against the oracle's dequantize-then-fp64 GEMM, with the single-launch
dynamic quantize (workspace given) and with the two-kernel one (no
workspace)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import TOL, require_cuda
from workloads import WORKLOADS, bf16_bits, draw_w, draw_x, layer_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    return require_cuda()


def _host_linear(nv, x, w, single_launch):
    M, K = x.shape
    N = w.shape[0]
    lin = nv.NVFP4Linear(w.cuda())
    xh = x.contiguous().pin_memory()
    yh = torch.full((M, N), float("nan"), dtype=torch.bfloat16).pin_memory()
    ws = lin.host_workspace(M)
    lin.forward_host(xh, yh, ws, single_launch=single_launch)
    torch.cuda.synchronize()
    code, detail = nv.device_error()
    assert code == 0, f"device wait timed out (tag {detail})"
    return yh.float().numpy()


def _oracle(x, w, rows=None):
    M, K = x.shape
    N = w.shape[0]
    aq, asf, asd, _ = oracle.quantize_dynamic(bf16_bits(x), M, K)
    bq, bsf, bsd, _ = oracle.quantize_dynamic(bf16_bits(w), N, K)
    return oracle.gemm(aq, asf, asd, bq, bsf, bsd, M, N, K, rows=rows)


@pytest.mark.parametrize("single_launch", [True, False])
@pytest.mark.parametrize("M,N,K", [(777, 392, 576), (300, 264, 3072), (1, 8, 64)])
def test_host_linear_shapes(nv, M, N, K, single_launch):
    x = draw_x("lognormal_channels", M, K, seed=7 * M + K, index=0)
    w = draw_w(N, K, None, seed=7 * M + K, index=1)
    y = _host_linear(nv, x, w, single_launch)
    ok, worst = oracle.gemm_tolerance_ok(y, _oracle(x, w), TOL)
    assert np.all(np.isfinite(y)) and ok, f"worst |err|/bound = {worst:.3f}"


@pytest.mark.parametrize("single_launch", [True, False])
def test_host_linear_qkv_sampled(nv, single_launch):
    """The QKV projection at 1024^2 (M=4608, K=3072, N=9216), seeded rows."""
    w = WORKLOADS["qkv_1024"]
    x, wt = layer_inputs(w, 0)
    y = _host_linear(nv, x, wt, single_launch)
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([[0, w.M - 1], rng.choice(w.M, 96, replace=False)]))
    ok, worst = oracle.gemm_tolerance_ok(y[rows], _oracle(x, wt, rows=rows), TOL)
    assert ok, f"worst |err|/bound = {worst:.3f}"
