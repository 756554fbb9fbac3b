"""GPU parity: the tcgen05 block-scaled FP4 GEMM and its fused output
quantization, against the oracle's dequantize-then-fp64 GEMM."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import TOL, bf16_from_fp64, check_fused_blocks, require_cuda
from workloads import OWN_WORKLOADS, WORKLOADS, bf16_bits, draw_w, draw_x, layer_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    return require_cuda()


def _gpu_linear(nv, x, w, fused_s_enc=None):
    lin = nv.NVFP4Linear(w.cuda())
    xd = x.cuda()
    fused = None
    if fused_s_enc is not None:
        M, N = x.shape[0], w.shape[0]
        fused = nv.FusedQuant(torch.tensor([fused_s_enc], dtype=torch.float32, device="cuda"),
                              nv.empty_nvfp4(M, N), torch.empty(1, dtype=torch.float32,
                                                                device="cuda"))
    y = lin(xd, fused=fused)
    torch.cuda.synchronize()
    code, detail = nv.device_error()
    assert code == 0, f"device wait timed out (tag {detail})"
    return y, fused


def _oracle_linear(x, w, rows=None):
    M, K = x.shape
    N = w.shape[0]
    aq, asf, asd, _ = oracle.quantize_dynamic(bf16_bits(x), M, K)
    bq, bsf, bsd, _ = oracle.quantize_dynamic(bf16_bits(w), N, K)
    return oracle.gemm(aq, asf, asd, bq, bsf, bsd, M, N, K, rows=rows)


def _check_tol(y_gpu, ref, what):
    ok, worst = oracle.gemm_tolerance_ok(y_gpu, ref, TOL)
    assert np.all(np.isfinite(y_gpu)), f"{what}: non-finite output"
    assert ok, f"{what}: worst |err|/bound = {worst:.3f}"
    return worst


SHAPES = [(128, 128, 256), (128, 128, 64), (1, 8, 64), (200, 136, 320), (300, 264, 576),
          (256, 512, 512), (129, 128, 1024), (64, 1000, 192), (1000, 256, 768), (777, 392, 3072)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_gemm_shapes(nv, M, N, K):
    x = draw_x("lognormal_channels", M, K, seed=M + N + K, index=0)
    w = draw_w(N, K, None, seed=M + N + K, index=1)
    y, _ = _gpu_linear(nv, x, w)
    _check_tol(y.float().cpu().numpy(), _oracle_linear(x, w), f"{M}x{N}x{K}")


def _representable(rng, rows, cols):
    """E2M1 values with a +-6 in every block of 16: with a static S_enc = 1
    every block scale is 1.0 (E4M3 0x38) and every code is the value itself."""
    mags = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    codes = rng.integers(0, 16, size=(rows, cols))
    v = mags[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    v[:, ::16] = np.where(rng.integers(0, 2, size=(rows, cols // 16)) == 0, 6.0, -6.0)
    return torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16)


def _gpu_static(nv, x, w, fused_s_enc=None):
    one = torch.ones(1, dtype=torch.float32, device="cuda")
    a = nv.quantize_with_scale(x.cuda(), one)
    b = nv.quantize_with_scale(w.cuda(), one)
    fused = None
    if fused_s_enc is not None:
        M, N = x.shape[0], w.shape[0]
        fused = nv.FusedQuant(torch.tensor([fused_s_enc], dtype=torch.float32, device="cuda"),
                              nv.empty_nvfp4(M, N),
                              torch.empty(1, dtype=torch.float32, device="cuda"))
    y = nv.gemm(a, b, fused=fused)
    torch.cuda.synchronize()
    assert nv.device_error()[0] == 0
    return y, fused


def _oracle_static(x, w):
    M, K = x.shape
    N = w.shape[0]
    aq, asf = oracle.quantize(bf16_bits(x), M, K, np.float32(1.0))
    bq, bsf = oracle.quantize(bf16_bits(w), N, K, np.float32(1.0))
    return oracle.gemm(aq, asf, np.float32(1.0), bq, bsf, np.float32(1.0), M, N, K)


@pytest.mark.parametrize("M,N,K", [(256, 256, 64), (130, 200, 128), (384, 384, 256),
                                   (200, 136, 1024)])
def test_gemm_exact_representable(nv, M, N, K):
    # All products are multiples of 1/4 and every partial sum stays below
    # 2^22, so the fp32 accumulation is exact on the GPU; both sides then
    # round the same exact value to bf16 once.
    rng = np.random.default_rng(M + N + K)
    x = _representable(rng, M, K)
    w = _representable(rng, N, K)
    y, _ = _gpu_static(nv, x, w)
    want = bf16_from_fp64(_oracle_static(x, w))
    got = y.float().cpu().numpy()
    assert np.array_equal(got, want), f"{np.sum(got != want)} elements differ"


@pytest.mark.parametrize("name", OWN_WORKLOADS)
def test_gemm_workloads_sampled_rows(nv, name):
    """Full-size GEMMs in the launch configuration the bench times; the
    oracle computes a seeded sample of rows (first, last, random)."""
    w = WORKLOADS[name]
    for li, layer in enumerate(w.layers):
        if layer.x_from_prev:
            continue   # fed by the previous layer's fused output: see test_gpu_ffn_fused.py
        x, wt = layer_inputs(w, li)
        M = x.shape[0]
        rng = np.random.default_rng(li)
        n_s = min(M, 256 if layer.N * layer.K < 40e6 else 96)
        rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, n_s, replace=False)]))
        y, _ = _gpu_linear(nv, x, wt)
        ref = _oracle_linear(x, wt, rows=rows)
        _check_tol(y[torch.from_numpy(rows).cuda()].float().cpu().numpy(), ref,
                   f"{name}/{layer.name}")
        del x, wt, y


@pytest.mark.parametrize("M,N,K", [(256, 256, 64), (130, 208, 128), (300, 512, 256)])
def test_fused_quantize_exact(nv, orc, M, N, K):
    """Exact GEMM -> the fused output quantization must equal the oracle's
    quantization of the same bf16 Y bit for bit (codes, tiled scales with
    padding, amax)."""
    rng = np.random.default_rng(17 + M)
    x = _representable(rng, M, K)
    w = _representable(rng, N, K)
    s_enc_y = np.float32(2688.0) / np.float32(300.0)
    y, fused = _gpu_static(nv, x, w, fused_s_enc=float(s_enc_y))
    ref = bf16_from_fp64(_oracle_static(x, w))
    assert np.array_equal(y.float().cpu().numpy(), ref)
    yb = torch.from_numpy(ref).to(torch.bfloat16)
    oq, osf = orc.quantize(bf16_bits(yb), M, N, s_enc_y)
    assert np.array_equal(fused.out.q.cpu().numpy(), oq)
    assert np.array_equal(fused.out.sf.cpu().numpy(), osf)
    assert np.float32(fused.amax.item()) == np.float32(np.abs(ref).max())


def test_fused_quantize_ffn_down_sampled(nv, orc):
    """FFN-down at 2048^2 with the fused next-layer quantize, on sampled rows:
    Y within the GEMM tolerance; codes and scales by check_fused_blocks
    (blocks equal to the oracle's bf16 outputs bit-exact, the others a valid
    quantization with the oracle's or a neighbouring scale code)."""
    w = WORKLOADS["ffn_down_2048"]
    x, wt = layer_inputs(w, 0)
    M, K = x.shape
    N = wt.shape[0]
    s_enc_y = np.float32(2688.0) / np.float32(8.0)
    y, fused = _gpu_linear(nv, x, wt, fused_s_enc=float(s_enc_y))
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 64, replace=False)]))
    ref = _oracle_linear(x, wt, rows=rows)
    yg = y[torch.from_numpy(rows).cuda()].float().cpu().numpy()
    _check_tol(yg, ref, "ffn_down fused Y")
    check_fused_blocks(orc, yg, bf16_from_fp64(ref), fused.out.q.cpu().numpy(),
                       fused.out.sf.cpu().numpy(), rows, s_enc_y, "ffn_down fused", 0.9)
    assert float(fused.amax.item()) == float(y.float().abs().max().item())
