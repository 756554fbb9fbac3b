"""GPU parity: the FP8 variant (E4M3 elements, one FP32 per-tensor scale; the
pages' "--variant fp8r" mode in "NVIDIA показала, как сократить генерацию
FLUX 3 Image Klein с 22 до 6 секунд", section "2. Запуск генерации
изображения").  Quantization bit-exact against the oracle; the kind::f8f6f4
CTA-pair GEMM within the GEMM tolerance of the oracle's fp64 product."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import TOL, bf16_from_fp64, check_fused_blocks, require_cuda
from workloads import WORKLOADS, bf16_bits, draw_w, draw_x, layer_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    return require_cuda()


def _gpu_fp8(nv, x):
    t = nv.quantize_fp8(x.cuda())
    torch.cuda.synchronize()
    return t.q.cpu().numpy(), np.float32(t.s_dec.item())


@pytest.mark.parametrize("rows,cols", [(1, 16), (3, 48), (130, 272), (257, 512), (64, 3072)])
@pytest.mark.parametrize("dist", ["normal_outliers", "gelu"])
def test_quantize_fp8(nv, rows, cols, dist):
    x = draw_x(dist, rows, cols, seed=rows + cols, index=0)
    q, s_dec = _gpu_fp8(nv, x)
    oq, os_dec, _ = oracle.quantize_fp8(bf16_bits(x), rows, cols)
    assert s_dec == os_dec
    assert np.array_equal(q, oq)


@pytest.mark.parametrize("kind", ["zeros", "negative_zeros", "subnormals", "huge", "midpoints"])
def test_quantize_fp8_edges(nv, kind):
    rows, cols = 40, 64
    g = torch.Generator().manual_seed(8)
    if kind == "zeros":
        x = torch.zeros(rows, cols)
    elif kind == "negative_zeros":
        x = torch.full((rows, cols), -0.0)
    elif kind == "subnormals":
        x = torch.randn(rows, cols, generator=g) * 2.0 ** -130
    elif kind == "huge":
        x = torch.randn(rows, cols, generator=g) * 1e37
    else:   # E4M3 midpoints around 1..2 at S_enc = 1 (amax 448)
        x = torch.tensor([1.0625, 1.1875, 1.3125, -1.4375] * (rows * cols // 4)).view(rows, cols)
        x[0, 0] = 448.0
    x = x.to(torch.bfloat16)
    q, s_dec = _gpu_fp8(nv, x)
    oq, os_dec, _ = oracle.quantize_fp8(bf16_bits(x), rows, cols)
    assert s_dec == os_dec and np.array_equal(q, oq), kind


def _fp8_linear(nv, x, w):
    lin = nv.FP8Linear(w.cuda())
    y = lin(x.cuda())
    torch.cuda.synchronize()
    code, detail = nv.device_error()
    assert code == 0, f"device wait timed out (tag {detail})"
    return y.float().cpu().numpy()


def _oracle_fp8_linear(x, w, rows=None):
    aq, asd, _ = oracle.quantize_fp8(bf16_bits(x), *x.shape)
    bq, bsd, _ = oracle.quantize_fp8(bf16_bits(w), *w.shape)
    return oracle.gemm_fp8(aq, asd, bq, bsd, rows)


@pytest.mark.parametrize("M,N,K", [(256, 256, 32), (300, 512, 96), (129, 264, 160),
                                   (1000, 768, 3072)])
def test_gemm_fp8(nv, M, N, K):
    x = draw_x("lognormal_channels", M, K, seed=M + K, index=0)
    w = draw_w(N, K, None, seed=M + K, index=1)
    ok, worst = oracle.gemm_tolerance_ok(_fp8_linear(nv, x, w), _oracle_fp8_linear(x, w), TOL)
    assert ok, f"{M}x{N}x{K}: worst {worst:.3f}"


def test_gemm_fp8_rejects_small_shapes(nv):
    a = nv.quantize_fp8(torch.ones(128, 64, dtype=torch.bfloat16, device="cuda"))
    b = nv.quantize_fp8(torch.ones(256, 64, dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(nv.NVFP4Error):
        nv.gemm_fp8(a, b)                                   # M <= 128: no FP8 kernel


def test_gemm_fp8_qkv_full_size_sampled(nv):
    w = WORKLOADS["qkv_1024"]
    x, wt = layer_inputs(w, 0)
    M = x.shape[0]
    rng = np.random.default_rng(2)
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 96, replace=False)]))
    y = _fp8_linear(nv, x, wt)
    ok, worst = oracle.gemm_tolerance_ok(y[rows], _oracle_fp8_linear(x, wt, rows), TOL)
    assert ok, f"qkv fp8: worst {worst:.3f}"


def test_quantize_fp8_empty(nv):
    """0 rows: no codes, S_dec = 1 (amax 0), as the oracle gives."""
    x = torch.zeros(0, 64, dtype=torch.bfloat16)
    q, s_dec = _gpu_fp8(nv, x)
    oq, os_dec, _ = oracle.quantize_fp8(bf16_bits(x), 0, 64)
    assert q.size == 0 and oq.size == 0
    assert s_dec == os_dec


@pytest.mark.parametrize("act", ["none", "gelu"])
@pytest.mark.parametrize("M,N,K", [(256, 256, 32), (300, 512, 96), (1000, 768, 3072)])
def test_gemm_fp8_fused_nvfp4_output(nv, orc, M, N, K, act):
    """The FP8 GEMM's fused epilogue, as for the NVFP4 GEMM: bf16 Y (after
    GELU when asked), the next layer's NVFP4 codes and scales with a static
    S_enc, amax of Y and its decode scale.  The oracle computes the FP8 layer
    in fp64, applies its own GELU, rounds to bf16 and quantizes."""
    x = draw_x("lognormal_channels", M, K, seed=3 * M + K, index=0)
    w = draw_w(N, K, None, seed=3 * M + K, index=1)
    ref = _oracle_fp8_linear(x, w)
    out_ref = oracle.gelu(ref) if act == "gelu" else ref
    s_enc_y = float(np.float32(2688.0) / np.float32(1.25 * np.abs(out_ref).max()))
    lin = nv.FP8Linear(w.cuda())
    fq = nv.FusedQuant(torch.tensor([s_enc_y], dtype=torch.float32, device="cuda"),
                       nv.empty_nvfp4(M, N), torch.zeros(1, dtype=torch.float32, device="cuda"),
                       nv.ACT_GELU if act == "gelu" else nv.ACT_NONE)
    y = lin(x.cuda(), fused=fq)
    torch.cuda.synchronize()
    code, detail = nv.device_error()
    assert code == 0, f"device wait timed out (tag {detail})"
    yg = y.float().cpu().numpy()
    rms = float(np.sqrt(np.mean(ref * ref)))
    slope = 1.13 if act == "gelu" else 1.0                  # GELU's slope is at most 1.129
    err = np.abs(yg.astype(np.float64) - out_ref)
    assert np.all(err <= slope * TOL * (np.abs(ref) + rms)), f"{M}x{N}x{K} {act} Y"
    check_fused_blocks(orc, yg, bf16_from_fp64(out_ref), fq.out.q.cpu().numpy(),
                       fq.out.sf.cpu().numpy(), np.arange(M), s_enc_y, f"fp8 {M}x{N}x{K} {act}")
    assert np.float32(fq.amax.item()) == np.float32(np.abs(yg).max())
    assert np.float32(fq.out.s_dec.item()) == np.float32(1.0) / np.float32(s_enc_y)
