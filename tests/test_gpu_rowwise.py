"""GPU parity: per-token (per-row) activation scales, the finer-grained
variant of the pages' per-tensor FP32 scale ("英伟达B200狂飙10.2倍！AI绘图
告别龟速！", section "NVFP4量化"): the quantization is bit-exact against the
oracle (codes, tiled scales with padding, per-row decode scales and amax);
the GEMM with per-row decode scales is within the GEMM tolerance."""
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


def _gpu_rowwise(nv, x):
    rows = x.shape[0]
    amax = torch.full((rows,), -1.0, device="cuda")
    t = nv.quantize_rowwise(x.cuda(), amax_rows=amax)
    torch.cuda.synchronize()
    return t.q.cpu().numpy(), t.sf.cpu().numpy(), t.s_dec.cpu().numpy(), amax.cpu().numpy()


def _assert_equal(g, o, what, rows=None):
    gq, gsf, gsd, gam = g
    oq, osf, osd, oam = o
    sel = slice(None) if rows is None else rows
    assert np.array_equal(gam[sel], oam[sel]), f"{what}: amax"
    assert np.array_equal(gsd[sel], osd[sel]), f"{what}: s_dec"
    assert np.array_equal(gq[sel], oq[sel]), f"{what}: codes"
    if rows is None:
        assert np.array_equal(gsf, osf), f"{what}: scales"


@pytest.mark.parametrize("rows,cols", [(1, 16), (3, 48), (127, 80), (130, 272), (257, 512),
                                       (64, 3072), (5, 4096), (200, 12288)])
def test_quantize_rowwise_shapes(nv, rows, cols):
    x = draw_x("normal_outliers", rows, cols, seed=rows + 3 * cols, index=0)
    _assert_equal(_gpu_rowwise(nv, x), oracle.quantize_rowwise(bf16_bits(x), rows, cols),
                  f"{rows}x{cols}")


def test_quantize_rowwise_edge_rows(nv):
    """Rows of zeros, negative zeros, bf16 subnormals, huge values and an
    exact-midpoint row in one tensor: each row keeps its own scale."""
    rows, cols = 136, 96
    g = torch.Generator().manual_seed(5)
    x = torch.randn(rows, cols, generator=g)
    x[0] = 0.0
    x[1] = -0.0
    x[2] = torch.randn(cols, generator=g) * 2.0 ** -130
    x[3] = torch.randn(cols, generator=g) * 1e37
    x[4] = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * (cols // 8))
    x = x.to(torch.bfloat16)
    _assert_equal(_gpu_rowwise(nv, x), oracle.quantize_rowwise(bf16_bits(x), rows, cols), "edge")


def test_quantize_rowwise_full_size_sampled(nv):
    """FFN-down's input at 2048^2 (16896 x 12288): every row on the GPU, the
    oracle on seeded rows (rows are independent, so they compare exactly)."""
    w = WORKLOADS["ffn_down_2048"]
    x, _ = layer_inputs(w, 0)
    rows, cols = x.shape
    rng = np.random.default_rng(3)
    sel = np.unique(np.concatenate([[0, rows - 1], rng.choice(rows, 40, replace=False)]))
    g = _gpu_rowwise(nv, x)
    o = oracle.quantize_rowwise(bf16_bits(x), rows, cols, row_idx=sel)
    _assert_equal(g, o, "ffn_down X", rows=sel)
    kb = cols // 16
    offs = [oracle.sf_offset(int(r), c, kb) for r in sel for c in range(kb)]
    assert np.array_equal(g[1][offs], o[1][offs])


@pytest.mark.parametrize("M,N,K", [(256, 512, 512), (130, 208, 128), (128, 512, 256),
                                   (777, 392, 3072)])
def test_gemm_rowscale(nv, M, N, K):
    """Per-row decode scales of A through every kernel variant."""
    x = draw_x("lognormal_channels", M, K, seed=M + N, index=0).float()
    x *= torch.exp(torch.linspace(-4.0, 4.0, M))[:, None]       # rows of very different scale
    x = x.to(torch.bfloat16)
    w = draw_w(N, K, None, seed=M + N, index=1)
    lin = nv.NVFP4Linear(w.cuda())
    y = nv.gemm(nv.quantize_rowwise(x.cuda()), lin.w)
    torch.cuda.synchronize()
    aq, asf, asd, _ = oracle.quantize_rowwise(bf16_bits(x), M, K)
    bq, bsf, bsd, _ = oracle.quantize_dynamic(bf16_bits(w), N, K)
    ref = oracle.gemm_rowwise(aq, asf, asd, bq, bsf, bsd, M, N, K)
    # Per-row tolerance: rows differ in scale by e^8, so the rms is per row.
    yg = y.float().cpu().numpy()
    for m in range(M):
        ok, worst = oracle.gemm_tolerance_ok(yg[m], ref[m], TOL)
        assert ok, f"{M}x{N}x{K} row {m}: worst {worst:.3f}"


def test_quantize_rowwise_empty(nv):
    """0 rows: nothing to quantize and no per-row scales; the call succeeds."""
    x = torch.zeros(0, 64, dtype=torch.bfloat16)
    _assert_equal(_gpu_rowwise(nv, x), oracle.quantize_rowwise(bf16_bits(x), 0, 64), "0x64")


@pytest.mark.parametrize("act", ["none", "gelu"])
@pytest.mark.parametrize("M,N,K", [(256, 512, 512), (130, 208, 128), (300, 512, 576)])
def test_gemm_rowscale_fused(nv, orc, M, N, K, act):
    """Per-row decode scales of A with the fused next-layer NVFP4 quantize
    (plain and GELU): the epilogue's alpha is per row; Y, codes, scales, amax
    and decode scale as for the per-tensor GEMM's fused epilogue."""
    x = draw_x("lognormal_channels", M, K, seed=2 * M + N, index=0).float()
    x *= torch.exp(torch.linspace(-1.0, 1.0, M))[:, None]       # rows of different scale
    x = x.to(torch.bfloat16)
    w = draw_w(N, K, None, seed=2 * M + N, index=1)
    aq, asf, asd, _ = oracle.quantize_rowwise(bf16_bits(x), M, K)
    bq, bsf, bsd, _ = oracle.quantize_dynamic(bf16_bits(w), N, K)
    ref = oracle.gemm_rowwise(aq, asf, asd, bq, bsf, bsd, M, N, K)
    out_ref = oracle.gelu(ref) if act == "gelu" else ref
    s_enc_y = float(np.float32(2688.0) / np.float32(1.25 * np.abs(out_ref).max()))
    lin = nv.NVFP4Linear(w.cuda())
    fq = nv.FusedQuant(torch.tensor([s_enc_y], dtype=torch.float32, device="cuda"),
                       nv.empty_nvfp4(M, N), torch.zeros(1, dtype=torch.float32, device="cuda"),
                       nv.ACT_GELU if act == "gelu" else nv.ACT_NONE)
    y = nv.gemm(nv.quantize_rowwise(x.cuda()), lin.w, fused=fq)
    torch.cuda.synchronize()
    code, detail = nv.device_error()
    assert code == 0, f"device wait timed out (tag {detail})"
    yg = y.float().cpu().numpy()
    slope = 1.13 if act == "gelu" else 1.0                  # GELU's slope is at most 1.129
    for m in range(M):
        rms = float(np.sqrt(np.mean(ref[m] * ref[m])))
        err = np.abs(yg[m].astype(np.float64) - out_ref[m])
        assert np.all(err <= slope * TOL * (np.abs(ref[m]) + rms)), f"{M}x{N}x{K} {act} row {m}"
    check_fused_blocks(orc, yg, bf16_from_fp64(out_ref), fq.out.q.cpu().numpy(),
                       fq.out.sf.cpu().numpy(), np.arange(M), s_enc_y,
                       f"rowscale {M}x{N}x{K} {act}")
    assert np.float32(fq.amax.item()) == np.float32(np.abs(yg).max())
    assert np.float32(fq.out.s_dec.item()) == np.float32(1.0) / np.float32(s_enc_y)
