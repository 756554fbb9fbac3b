"""GPU parity: the fused GELU + NVFP4 quantize epilogue and the FFN chain it
feeds (up-projection -> exact GELU -> NVFP4 codes -> down-projection), the
fused GEMM kernels of "NVIDIA показала, как сократить генерацию FLUX 3 Image
Klein с 22 до 6 секунд", section "Квантование NVFP4 и оптимизация
вычислительных ядер".

The oracle never sees a value computed on the GPU: it computes the layer in
fp64, applies its own GELU, rounds to bf16 and quantizes.  The GPU's bf16 Y
must lie within the GEMM tolerance carried through GELU (whose slope is at
most 1.129, at h = sqrt 2); every 16-element block whose bf16 values equal
the oracle's must carry the oracle's codes and scale, and the others (a value
rounded the other way after a different fp32 summation order) must carry the
oracle's scale code or, when their largest magnitude differs, a neighbouring
one, and decode to within one scale unit of the GPU's own values."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import TOL, bf16_from_fp64, check_fused_blocks, require_cuda
from workloads import WORKLOADS, bf16_bits, draw_w, draw_x, layer_inputs

pytestmark = pytest.mark.gpu

GELU_SLOPE = 1.13


@pytest.fixture(scope="module")
def nv():
    return require_cuda()


def _check_device(nv):
    torch.cuda.synchronize()
    code, detail = nv.device_error()
    assert code == 0, f"device wait timed out (tag {detail})"


def _fused_gelu(nv, lin, x, M, N, s_enc_y, want_y=True):
    out = nv.empty_nvfp4(M, N)
    fq = nv.FusedQuant(torch.tensor([s_enc_y], dtype=torch.float32, device="cuda"), out,
                       torch.empty(1, dtype=torch.float32, device="cuda"), nv.ACT_GELU)
    y = lin(x, fused=fq, want_y=want_y)
    _check_device(nv)
    return y, fq


def _oracle_pre(x, w, rows=None):
    """fp64 pre-activation Y of the oracle's quantized linear layer."""
    M, K = x.shape
    N = w.shape[0]
    aq, asf, asd, _ = oracle.quantize_dynamic(bf16_bits(x), M, K)
    bq, bsf, bsd, _ = oracle.quantize_dynamic(bf16_bits(w), N, K)
    return oracle.gemm(aq, asf, asd, bq, bsf, bsd, M, N, K, rows=rows)


def _check_gelu_y(yg, ref_pre, what):
    """|Y_gpu - GELU(ref)| <= 1.13 * TOL * (|ref| + rms(ref)) per element."""
    g = oracle.gelu(ref_pre)
    rms = float(np.sqrt(np.mean(ref_pre * ref_pre)))
    bound = GELU_SLOPE * TOL * (np.abs(ref_pre) + rms)
    err = np.abs(yg.astype(np.float64) - g)
    assert np.all(np.isfinite(yg)), f"{what}: non-finite output"
    assert np.all(err <= bound), f"{what}: worst |err|/bound = {float((err / bound).max()):.3f}"
    return g


SHAPES = [(256, 256, 64), (130, 208, 128), (128, 512, 256), (300, 512, 576), (64, 1024, 3072)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_fused_gelu_quantize(nv, orc, M, N, K):
    """Every kernel variant (CTA pair; 1-CTA with N < 256; 1-CTA with M <= 128)
    with the GELU epilogue: Y, codes, scales (padding rows included), amax of
    Y and the decode scale it writes."""
    x = draw_x("lognormal_channels", M, K, seed=M + N + K, index=0)
    w = draw_w(N, K, None, seed=M + N + K, index=1)
    ref_pre = _oracle_pre(x, w)
    # Static output scale from the oracle's own output, with headroom, so no
    # block saturates (a saturated block is exact on both sides but escapes
    # the error bound used for blocks rounded differently).
    s_enc_y = float(np.float32(2688.0) / np.float32(1.25 * np.abs(oracle.gelu(ref_pre)).max()))
    lin = nv.NVFP4Linear(w.cuda())
    y, fq = _fused_gelu(nv, lin, x.cuda(), M, N, s_enc_y)
    yg = y.float().cpu().numpy()
    g = _check_gelu_y(yg, ref_pre, f"{M}x{N}x{K} Y")
    gq = fq.out.q.cpu().numpy()
    gsf = fq.out.sf.cpu().numpy()
    _, osf = check_fused_blocks(orc, yg, bf16_from_fp64(g), gq, gsf, np.arange(M), s_enc_y,
                                 f"{M}x{N}x{K}")
    kb = N // 16
    pad = [orc.sf_offset(r, c, kb) for r in range(M, (M + 127) // 128 * 128) for c in range(kb)]
    assert np.all(gsf[pad] == 0) and np.all(osf[pad] == 0)
    assert np.float32(fq.amax.item()) == np.float32(np.abs(yg).max())
    assert np.float32(fq.out.s_dec.item()) == np.float32(1.0) / np.float32(s_enc_y)


def test_fused_gelu_without_y(nv):
    """Fused-only call (no bf16 Y written): the same codes and scales as with Y."""
    M, N, K = 384, 512, 512
    x = draw_x("lognormal_channels", M, K, seed=9, index=0).cuda()
    w = draw_w(N, K, None, seed=9, index=1).cuda()
    lin = nv.NVFP4Linear(w)
    s = float(np.float32(2688.0) / np.float32(6.0))
    _, a = _fused_gelu(nv, lin, x, M, N, s, want_y=True)
    none, b = _fused_gelu(nv, lin, x, M, N, s, want_y=False)
    assert none is None
    assert torch.equal(a.out.q, b.out.q) and torch.equal(a.out.sf, b.out.sf)
    assert a.amax.item() == b.amax.item()


def test_ffn_block_chain_sampled(nv, orc):
    """The FFN block at 2048^2 as bench.py runs it (M = 16896): X quantized on
    the GPU, up-projection with the fused GELU + quantize, its codes fed
    straight into the down-projection.  On seeded rows the oracle runs the
    same chain from X in fp64 (its own GELU, bf16 rounding and quantization,
    with the same static output scale)."""
    w = WORKLOADS["ffn_block_2048"]
    x, w_up = layer_inputs(w, 0)
    _, w_down = layer_inputs(w, 1)
    M, K = x.shape
    N_up, N_down = w_up.shape[0], w_down.shape[0]
    # Static scale with headroom: |GELU(h)| stays well below 12 here (h has a
    # standard deviation of about 1.3 over 2e8 values).
    s_enc_h = float(np.float32(2688.0) / np.float32(12.0))
    up = nv.NVFP4Linear(w_up.cuda())
    down = nv.NVFP4Linear(w_down.cuda())
    h, fq = _fused_gelu(nv, up, x.cuda(), M, N_up, s_enc_h, want_y=True)
    y = nv.gemm(fq.out, down.w)
    _check_device(nv)

    rng = np.random.default_rng(11)
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 48, replace=False)]))
    rows_t = torch.from_numpy(rows).cuda()
    ref_up = _oracle_pre(x, w_up, rows=rows)
    hg = h[rows_t].float().cpu().numpy()
    g = _check_gelu_y(hg, ref_up, "ffn_block up Y")
    oq, osf = check_fused_blocks(orc, hg, bf16_from_fp64(g), fq.out.q.cpu().numpy(),
                                  fq.out.sf.cpu().numpy(), rows, s_enc_h, "ffn_block H")
    # The oracle's own chain: its quantized H (rows only) through the down GEMM.
    s_dec_h = np.float32(1.0) / np.float32(s_enc_h)
    bq, bsf, bsd, _ = oracle.quantize_dynamic(bf16_bits(w_down), N_down, N_up)
    ref = oracle.gemm(oq, osf, s_dec_h, bq, bsf, bsd, len(rows), N_down, N_up)
    ok, worst = oracle.gemm_tolerance_ok(y[rows_t].float().cpu().numpy(), ref, TOL)
    assert ok, f"ffn_block down Y: worst |err|/bound = {worst:.3f}"
