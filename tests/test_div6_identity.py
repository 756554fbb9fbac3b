"""The GPU computes the block-scale quotient a_b / 6 (a_b the bf16 amax of a
16-element block; "英伟达B200狂飙10.2倍！AI绘图告别龟速！", section "NVFP4量化")
as the double product a_b * RN64(1/6) rounded once to fp32, instead of an
fp32 division.  The two agree for every bf16 value: a_b = M * 2^k with
k >= -133, so a_b / 6 measured in units of the fp32 result spacing is an
integer multiple of 1/3 and never within 1/6 unit of a rounding midpoint.
Checked here exhaustively over every non-negative finite bf16 value, in IEEE
arithmetic on the host (numpy's float64 product and float64 -> float32
rounding are the operations the kernel issues)."""
import numpy as np


def _div6_pair(a: np.ndarray):
    with np.errstate(all="ignore"):
        want = a / np.float32(6.0)                                    # IEEE fp32 RN division
        got = (a.astype(np.float64) * np.float64(1.0 / 6.0)).astype(np.float32)
    return got.view(np.uint32), want.view(np.uint32)


def test_div6_double_product_equals_fp32_division_for_all_bf16():
    bits = np.arange(0, 0x7F80, dtype=np.uint32)  # +0 .. largest finite, subnormals included
    a = (bits << 16).view(np.float32)
    got, want = _div6_pair(a)
    assert np.array_equal(got, want)


def test_fp32_reciprocal_product_is_not_enough():
    """Negative control: the same exhaustive comparison rejects the cheaper
    fp32 product a_b * RN32(1/6) (thousands of bf16 values round
    differently), so the check above is sensitive to the method."""
    bits = np.arange(0, 0x7F80, dtype=np.uint32)
    a = (bits << 16).view(np.float32)
    with np.errstate(all="ignore"):
        want = (a / np.float32(6.0)).view(np.uint32)
        got = (a * np.float32(1.0 / 6.0)).view(np.uint32)
    assert np.count_nonzero(got != want) > 1000
