"""GPU parity: amax and NVFP4 quantization (bit-exact against the oracle)."""
import numpy as np
import pytest
import torch

from gpu_common import (assert_quant_equal, gpu_quantize_dynamic, oracle_quantize_dynamic,
                        require_cuda)
from workloads import OWN_WORKLOADS, WORKLOADS, bf16_bits, draw_x, layer_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    return require_cuda()


@pytest.mark.parametrize("numel", [0, 1, 7, 8, 9, 1000, 4096 * 3 + 5, 1 << 22, (1 << 24) + 3])
def test_amax(nv, orc, numel):
    g = torch.Generator().manual_seed(numel)
    x = (torch.randn(max(numel, 1), generator=g) * 3).to(torch.bfloat16)[:numel]
    if numel > 5:
        x[numel // 3] = -17.5   # the max sits at a negative value
    xd = x.cuda()
    amax = nv.tensor_amax(xd)
    torch.cuda.synchronize()
    want = orc.tensor_amax(bf16_bits(x)) if numel else np.float32(0)
    assert np.float32(amax.item()) == want


# Widths that are multiples of 64 take the flat single-launch kernel, the
# others the row-stream one; both appear, with ragged row counts.
SMALL_SHAPES = [(1, 16), (3, 48), (127, 80), (128, 64), (130, 272), (257, 512), (64, 3072),
                (1000, 16), (5, 4096), (1, 64), (129, 192)]


PATHS = ["two_kernel", "fused"]


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("rows,cols", SMALL_SHAPES)
def test_quantize_small_shapes(nv, rows, cols, path):
    x = draw_x("normal_outliers", rows, cols, seed=rows * 7 + cols, index=0)
    assert_quant_equal(gpu_quantize_dynamic(nv, x, path), oracle_quantize_dynamic(x),
                       f"{rows}x{cols}/{path}")


def _edge_tensor(kind, rows=130, cols=80):
    g = torch.Generator().manual_seed(11)
    if kind == "zeros":
        return torch.zeros(rows, cols, dtype=torch.bfloat16)
    if kind == "negative_zeros":
        return torch.full((rows, cols), -0.0, dtype=torch.bfloat16)
    if kind == "mixed_zero_blocks":
        x = torch.randn(rows, cols, generator=g)
        x[:, 16:32] = 0.0
        x[::3, 48:64] = -0.0
        return x.to(torch.bfloat16)
    if kind == "bf16_subnormals":
        x = torch.randn(rows, cols, generator=g) * 2.0 ** -128
        return x.to(torch.bfloat16)
    if kind == "subnormals_with_zeros":
        x = torch.randn(rows, cols, generator=g) * 2.0 ** -130
        x[:, ::5] = 0.0
        return x.to(torch.bfloat16)
    if kind == "huge":
        x = torch.randn(rows, cols, generator=g) * 1e37
        x[0, 0] = 3.0e38
        return x.to(torch.bfloat16)
    if kind == "underflow_blocks":
        x = torch.randn(rows, cols, generator=g) * 1e-6
        x[:, :16] = torch.randn(rows, 16, generator=g) * 1e4
        return x.to(torch.bfloat16)
    if kind == "one_hot":
        x = torch.zeros(rows, cols)
        x[torch.arange(rows), torch.arange(rows) % cols] = torch.linspace(-5, 5, rows)
        return x.to(torch.bfloat16)
    if kind == "ties":
        # Values that land exactly on E2M1 midpoints after scaling by inv=1:
        # blocks with amax 6 and S_enc = 2688/6 give sf = 448 and inv = 1.
        mids = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0])
        x = mids.repeat(rows, cols // 8)
        x = x * torch.where(torch.rand(rows, cols, generator=g) < 0.5, -1.0, 1.0)
        return x.to(torch.bfloat16)
    raise ValueError(kind)


@pytest.mark.parametrize("cols", [80, 128])
@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("kind", ["zeros", "negative_zeros", "mixed_zero_blocks",
                                  "bf16_subnormals", "subnormals_with_zeros", "huge",
                                  "underflow_blocks", "one_hot", "ties"])
def test_quantize_edge_cases(nv, kind, path, cols):
    x = _edge_tensor(kind, cols=cols)
    assert_quant_equal(gpu_quantize_dynamic(nv, x, path), oracle_quantize_dynamic(x),
                       f"{kind}/{path}/{cols}")


def test_quantize_dynamic_back_to_back(nv):
    """Consecutive single-launch quantizations of different shapes (different
    cooperative grid sizes) share one workspace: every result must be exact,
    so the grid barrier and the per-launch amax words reset correctly."""
    shapes = [(257, 512), (64, 3072), (1, 16), (4608, 3072), (130, 272), (1000, 12288),
              (3, 48), (257, 512)]
    for i, (rows, cols) in enumerate(shapes):
        x = draw_x("lognormal_channels", rows, cols, seed=100 + i, index=0)
        x = (x * (10.0 ** (i % 5 - 2))).to(torch.bfloat16)   # amax changes every call
        assert_quant_equal(gpu_quantize_dynamic(nv, x, "fused"), oracle_quantize_dynamic(x),
                           f"call {i} {rows}x{cols}")


def test_quantize_static_scale(nv, orc):
    g = torch.Generator().manual_seed(3)
    x = (torch.randn(200, 96, generator=g) * 4).to(torch.bfloat16)
    for s in (1.0, 0.37, 448.0, 2.0 ** -20):
        s_enc = torch.tensor([s], dtype=torch.float32, device="cuda")
        t = nv.quantize_with_scale(x.cuda(), s_enc)
        torch.cuda.synchronize()
        oq, osf = orc.quantize(bf16_bits(x), 200, 96, np.float32(s))
        assert np.array_equal(t.q.cpu().numpy(), oq)
        assert np.array_equal(t.sf.cpu().numpy(), osf)
        assert np.float32(t.s_dec.item()) == orc.decode_scale(np.float32(s))


@pytest.mark.parametrize("name", OWN_WORKLOADS)
def test_quantize_workloads_full_size(nv, name):
    """Activations (per-call, single-launch path) and weights (load-time,
    two-kernel path) of every workload, at full size, bit-exact."""
    w = WORKLOADS[name]
    for li in range(len(w.layers)):
        x, wt = layer_inputs(w, li)
        if x is not None:   # None: the layer's input is the previous layer's fused output
            assert_quant_equal(gpu_quantize_dynamic(nv, x, "fused"), oracle_quantize_dynamic(x),
                               f"{name}/{w.layers[li].name}/X")
        assert_quant_equal(gpu_quantize_dynamic(nv, wt, "two_kernel"),
                           oracle_quantize_dynamic(wt), f"{name}/{w.layers[li].name}/W")
        del x, wt


@pytest.mark.parametrize("cols", [272, 320])
@pytest.mark.parametrize("path", PATHS)
def test_quantize_input_16_byte_aligned(nv, path, cols):
    """An input that is 16-byte but not 32-byte aligned (a view 8 elements
    into a buffer) takes the two-load path and gives the same codes."""
    rows = 130
    x = draw_x("normal_outliers", rows, cols, seed=77, index=0)
    buf = torch.zeros(rows * cols + 16, dtype=torch.bfloat16, device="cuda")
    view = buf[8:8 + rows * cols].view(rows, cols)
    assert view.data_ptr() % 32 == 16
    view.copy_(x.cuda())
    if path == "two_kernel":
        amax = nv.tensor_amax(view)
        t = nv.quantize(view, amax)
    else:
        amax = torch.empty(1, device="cuda")
        t = nv.quantize_dynamic(view, amax=amax)
    torch.cuda.synchronize()
    got = (t.q.cpu().numpy(), t.sf.cpu().numpy(), np.float32(t.s_dec.item()),
           np.float32(amax.item()))
    assert_quant_equal(got, oracle_quantize_dynamic(x), f"16B-aligned/{path}")


@pytest.mark.parametrize("extra_rows", [0, 1])
def test_quantize_dynamic_resident_limit(nv, extra_rows):
    """The single-launch quantize keeps a slice of the input per SM in shared
    memory when one fits (216 KB of 32-byte blocks, a multiple of 4 blocks);
    at the largest such input for this GPU and one row past it (the
    re-reading form) the codes and scales are the oracle's."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    cols = 3072
    kb = cols // 16
    rows = (sms * (216 * 1024 // 32)) // kb + extra_rows
    x = draw_x("normal_outliers", rows, cols, seed=rows, index=0)
    assert_quant_equal(gpu_quantize_dynamic(nv, x, "fused"), oracle_quantize_dynamic(x),
                       f"{rows}x{cols}")


@pytest.mark.parametrize("cols", [64, 80])
@pytest.mark.parametrize("path", PATHS)
def test_quantize_empty(nv, orc, cols, path):
    """An empty tensor (0 rows; its arrays have no storage): no codes, no
    scales, amax 0 and S_dec = 1 / S_enc(0) = 1 on every path, as the oracle
    gives; the static-scale call writes 1 / S_enc from its given scale."""
    x = torch.zeros(0, cols, dtype=torch.bfloat16)
    assert_quant_equal(gpu_quantize_dynamic(nv, x, path), oracle_quantize_dynamic(x),
                       f"0x{cols}/{path}")
    s_enc = torch.tensor([0.37], dtype=torch.float32, device="cuda")
    t = nv.quantize_with_scale(x.cuda(), s_enc)
    torch.cuda.synchronize()
    assert t.q.numel() == 0 and t.sf.numel() == 0
    assert np.float32(t.s_dec.item()) == orc.decode_scale(np.float32(0.37))


@pytest.mark.parametrize("rows,cols", [(1, 16), (130, 272), (257, 512), (64, 3072), (4608, 3072)])
@pytest.mark.parametrize("prev", [0.5, 1.0, 1.3])
def test_quantize_one_pass(nv, orc, rows, cols, prev):
    """One pass with the scale from an earlier amax (prev x this tensor's:
    saturating, exact, with headroom): codes, scales and S_dec are the
    oracle's for that amax, and the amax written for the next call is this
    tensor's."""
    x = draw_x("normal_outliers", rows, cols, seed=rows + cols, index=0)
    xb = bf16_bits(x)
    amax_prev = np.float32(orc.tensor_amax(xb) * np.float32(prev))
    a_prev = torch.tensor([float(amax_prev)], dtype=torch.float32, device="cuda")
    a_out = torch.full((1,), -1.0, device="cuda")
    t = nv.quantize_one_pass(x.cuda(), a_prev, a_out)
    torch.cuda.synchronize()
    oq, osf, osd, oamax = orc.quantize_one_pass(xb, rows, cols, amax_prev)
    assert np.array_equal(t.q.cpu().numpy(), oq)
    assert np.array_equal(t.sf.cpu().numpy(), osf)
    assert np.float32(t.s_dec.item()) == osd
    assert np.float32(a_out.item()) == oamax


def test_quantize_one_pass_rejects_aliased_amax(nv):
    x = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    a = torch.ones(1, device="cuda")
    with pytest.raises(nv.NVFP4Error):
        nv.quantize_one_pass(x, a, a)
