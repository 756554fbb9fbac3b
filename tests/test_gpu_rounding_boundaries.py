"""GPU parity at the conversions' rounding boundaries: E4M3 block-scale
midpoints (normal and subnormal range) and their fp32 neighbours, the 448
saturation band, and E2M1 element midpoints with block scales other than 1,
through every quantize path, bit-exact against the oracle.  Random inputs
almost never hit these cases; tests/rounding_cases.py builds them and
tests/test_rounding_cases.py checks that they land where they should."""
import numpy as np
import pytest
import torch

import rounding_cases as rc
from gpu_common import assert_quant_equal, gpu_quantize_dynamic, oracle_quantize_dynamic, \
    require_cuda
from workloads import bf16_bits

pytestmark = pytest.mark.gpu

# 64 blocks per row take the flat kernels (rows a multiple of 64 elements),
# 65 the row-stream ones.
WIDTHS = [64, 65]


@pytest.fixture(scope="module")
def nv():
    return require_cuda()


def _all_blocks():
    return rc.scale_midpoint_blocks() + rc.element_midpoint_blocks() + rc.saturation_blocks()


@pytest.mark.parametrize("blocks_per_row", WIDTHS)
@pytest.mark.parametrize("s_enc", rc.STATIC_SCALES)
def test_static_scale(nv, orc, s_enc, blocks_per_row):
    x = rc.as_tensor(_all_blocks(), blocks_per_row)
    rows, cols = x.shape
    t = nv.quantize_with_scale(x.cuda(), torch.tensor([s_enc], dtype=torch.float32,
                                                       device="cuda"))
    torch.cuda.synchronize()
    oq, osf = orc.quantize(bf16_bits(x), rows, cols, np.float32(s_enc))
    bad = np.flatnonzero(t.sf.cpu().numpy() != osf)
    assert bad.size == 0, f"{bad.size} scale bytes differ, first at {bad[:8]}"
    assert np.array_equal(t.q.cpu().numpy(), oq)
    assert np.float32(t.s_dec.item()) == orc.decode_scale(np.float32(s_enc))


def _with_unit_scale(blocks_per_row):
    """Every row starts with a block whose largest magnitude is 2688, so the
    tensor's (and every row's) amax is 2688 and S_enc = 2688 / 2688 = 1; the
    saturation band (larger magnitudes) is left out."""
    first = np.array([2688.0] + [0.0] * 15)
    blocks = rc.scale_midpoint_blocks() + rc.element_midpoint_blocks()
    return rc.as_tensor(blocks, blocks_per_row, first=first)


@pytest.mark.parametrize("path", ["fused", "two_kernel"])
@pytest.mark.parametrize("blocks_per_row", WIDTHS)
def test_dynamic(nv, path, blocks_per_row):
    x = _with_unit_scale(blocks_per_row)
    g = gpu_quantize_dynamic(nv, x, path)
    o = oracle_quantize_dynamic(x)
    assert o[2] == np.float32(1.0)          # S_dec = 1 / S_enc = 1
    assert_quant_equal(g, o, f"{path}/{blocks_per_row}")


@pytest.mark.parametrize("blocks_per_row", WIDTHS)
def test_one_pass(nv, orc, blocks_per_row):
    x = _with_unit_scale(blocks_per_row)
    rows, cols = x.shape
    prev = torch.tensor([2688.0], device="cuda")
    amax = torch.empty(1, device="cuda")
    t = nv.quantize_one_pass(x.cuda(), prev, amax)
    torch.cuda.synchronize()
    oq, osf, osd, oamax = orc.quantize_one_pass(bf16_bits(x), rows, cols, np.float32(2688.0))
    assert np.array_equal(t.sf.cpu().numpy(), osf)
    assert np.array_equal(t.q.cpu().numpy(), oq)
    assert np.float32(t.s_dec.item()) == osd and np.float32(amax.item()) == oamax


@pytest.mark.parametrize("blocks_per_row", WIDTHS)
def test_rowwise(nv, orc, blocks_per_row):
    x = _with_unit_scale(blocks_per_row)
    rows, cols = x.shape
    t = nv.quantize_rowwise(x.cuda())
    torch.cuda.synchronize()
    oq, osf, osd, _ = orc.quantize_rowwise(bf16_bits(x), rows, cols)
    assert np.all(osd == np.float32(1.0))
    assert np.array_equal(t.sf.cpu().numpy(), osf)
    assert np.array_equal(t.q.cpu().numpy(), oq)
    assert np.array_equal(t.s_dec.cpu().numpy(), osd)
