"""The rounding-boundary inputs (tests/rounding_cases.py) do what they claim,
checked against the oracle's format tables, and the oracle rounds them by the
formats' definitions: round to nearest, ties to the even code, saturating at
448 (block scales, E4M3) and 6 (elements, E2M1).  The GPU side of the same
inputs is tests/test_gpu_rounding_boundaries.py."""
import numpy as np
import pytest
import torch

import rounding_cases as rc
from workloads import bf16_bits


def _grid(orc):
    """(value, code) of every finite non-negative E4M3 code, from the oracle."""
    return sorted((orc.e4m3_value(c), c) for c in range(0x7F))


def test_grid_matches_oracle_table(orc):
    assert np.array_equal(rc.e4m3_grid(), np.array([v for v, _ in _grid(orc)]))


@pytest.mark.parametrize("s_enc", rc.STATIC_SCALES[:3])
def test_scale_midpoints_round_as_defined(orc, s_enc):
    """Each block's scale s = (a_b / 6) * S_enc sits on an E4M3 midpoint
    (S_enc = 1), one fp32 step above it or one below; the oracle picks the
    even neighbour, the upper, the lower."""
    g = _grid(orc)
    vals = np.array([v for v, _ in g])
    for blk, m in zip(rc.scale_midpoint_blocks(), rc.e4m3_midpoints()):
        a_b = np.float32(np.abs(blk).max())
        s = np.float32(np.float32(a_b / np.float32(6.0)) * np.float32(s_enc))
        i = int(np.searchsorted(vals, m)) - 1           # lower neighbour of m
        (lo, c_lo), (hi, c_hi) = g[i], g[i + 1]
        assert lo < m < hi and m == (lo + hi) / 2
        if s_enc == 1.0:
            assert s == np.float32(m)
            want = c_lo if c_lo % 2 == 0 else c_hi
        elif s_enc > 1.0:
            assert m < s < hi
            want = c_hi
        else:
            assert lo < s < m
            want = c_lo
        x = torch.from_numpy(blk.astype(np.float32)).bfloat16()
        _, sf = orc.quantize(bf16_bits(x), 1, 16, np.float32(s_enc))
        assert int(sf[0]) == want, (m, s_enc)


def test_saturation_band(orc):
    """Block scales from 448 to 501.3 all encode to 448 (0x7E)."""
    for blk in rc.saturation_blocks():
        x = torch.from_numpy(blk.astype(np.float32)).bfloat16()
        _, sf = orc.quantize(bf16_bits(x), 1, 16, np.float32(1.0))
        assert int(sf[0]) == 0x7E


def test_element_midpoints(orc):
    """With S_enc = 1 and a power-of-two scale v, x * (1 / v) lands exactly on
    the E2M1 midpoints, which go to the even code; the bf16 neighbours go up
    and down."""
    mids = np.array(rc.E2M1_MIDPOINTS)
    even = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    blocks = rc.element_midpoint_blocks()
    vs = [2.0 ** e for e in range(-9, 9)]
    for bi, v in enumerate(vs):
        for variant in range(3):
            blk = blocks[3 * bi + variant]
            x = torch.from_numpy(blk.astype(np.float32)).bfloat16()
            q, sf = orc.quantize(bf16_bits(x), 1, 16, np.float32(1.0))
            assert orc.e4m3_value(int(sf[0])) == v
            codes = np.stack([q[0] & 0xF, q[0] >> 4], -1).reshape(-1)
            got = np.array([orc.e2m1_value(int(c)) for c in codes])
            assert got[0] == 6.0
            for k, mid in enumerate(mids):
                if variant == 0:
                    assert got[1 + k] == even[mid] and got[8 + k] == -even[mid], (v, mid)
                elif variant == 1:
                    assert got[1 + k] == min(
                        (e for e in (0.5, 1, 1.5, 2, 3, 4, 6) if e > mid), default=6), (v, mid)
                else:
                    assert got[1 + k] < mid and got[1 + k] == max(
                        (e for e in (0, 0.5, 1, 1.5, 2, 3, 4) if e < mid)), (v, mid)
