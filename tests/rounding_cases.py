"""Inputs that put NVFP4's two conversions exactly on their rounding
boundaries.  Nothing here quantizes: the module builds bf16 tensors from the
definitions of the two formats, and the tests hand the same tensors to the
kernels and to the oracle.

With a per-tensor scale S_enc = 1 the block scale is s = a_b / 6 (a_b the
block's largest magnitude), so a block whose largest magnitude is 6 m puts s
exactly on m.  E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits,
largest finite 448, smallest subnormal 2^-9) has the values (1 + j/8) 2^e
for e in -6..8 and k 2^-9 for k in 1..7; a midpoint of two neighbours has at
most five significant bits, so 6 m has at most eight and is a bf16 value.
S_enc = 1 + 2^-23 and 1 - 2^-24 then move every s one fp32 step above or
below its midpoint.

The elements of a block whose scale is itself an E4M3 value v (a_b = 6 v)
land, after the multiplication by S_enc / v, on the E2M1 midpoints 0.25,
0.75, 1.25, 1.75, 2.5, 3.5 and 5 (exactly when v is a power of two), and on
their bf16 neighbours."""
from __future__ import annotations

import numpy as np
import torch

E2M1_MIDPOINTS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


def e4m3_grid() -> np.ndarray:
    """All finite non-negative E4M3 values, ascending (0 and 2^-9 .. 448)."""
    sub = [k * 2.0 ** -9 for k in range(1, 8)]
    normal = [(1 + j / 8) * 2.0 ** e for e in range(-6, 9) for j in range(8)]
    normal = [v for v in normal if v <= 448.0]
    return np.array([0.0] + sub + normal)


def e4m3_midpoints() -> np.ndarray:
    g = e4m3_grid()
    return (g[:-1] + g[1:]) / 2


def _bf16(v: np.ndarray) -> np.ndarray:
    """fp64 values that must already be bf16 values, checked and returned."""
    t = torch.from_numpy(np.asarray(v, dtype=np.float32)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(t, np.asarray(v, dtype=np.float64)), "not a bf16 value"
    return t


def _bf16_round(v: np.ndarray) -> np.ndarray:
    """fp64 values rounded to bf16 (filler elements whose exact value does
    not matter, only that they stay below the block's largest magnitude)."""
    return torch.from_numpy(np.asarray(v, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def _bf16_step(x: np.ndarray, up: bool) -> np.ndarray:
    """The bf16 neighbour of each (positive, bf16) value, above or below."""
    bits = torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16)
    bits = bits + (1 if up else -1)
    return bits.view(torch.bfloat16).double().numpy()


def scale_midpoint_blocks() -> list[np.ndarray]:
    """One block per E4M3 midpoint m (subnormal range included): largest
    magnitude 6 m, the rest spread over the block's range with mixed signs."""
    fr = np.array([1.0, -0.5, 0.25, -0.75, 0.125, 0.9375, -0.0625, 0.375, -1.0, 0.625,
                   -0.3125, 0.0, 0.5, -0.875, 0.1875, 0.8125])
    out = []
    for m in e4m3_midpoints():
        a_b = _bf16(np.array([6.0 * m]))[0]
        blk = _bf16_round(a_b * fr)
        assert np.abs(blk).max() == a_b
        out.append(blk)
    return out


def element_midpoint_blocks() -> list[np.ndarray]:
    """Blocks whose scale is an E4M3 value v (largest magnitude 6 v) and whose
    other elements are v times the E2M1 midpoints, and their bf16 neighbours
    above and below, with both signs."""
    out = []
    vs = [2.0 ** e for e in range(-9, 9)] + [0.75, 1.25, 3.5, 13.0, 0.01171875, 288.0]
    for v in vs:
        mids = _bf16(v * np.array(E2M1_MIDPOINTS))
        for variant in range(3):
            x = mids if variant == 0 else _bf16_step(mids, up=variant == 1)
            blk = np.zeros(16)
            blk[0] = 6.0 * v
            blk[1:8] = x
            blk[8:15] = -x
            blk[15] = -0.0 if variant == 2 else v * 0.125
            out.append(_bf16(blk))
    return out


def saturation_blocks() -> list[np.ndarray]:
    """Largest magnitudes 2688 .. 3008 (every bf16 value there, spacing 16):
    block scales 448 .. 501.3, across the E4M3 saturation at 448 and the
    448 | 480 midpoint 464."""
    out = []
    for a_b in np.arange(2688.0, 3009.0, 16.0):
        out.append(_bf16_round(a_b * np.array([1.0, -0.5, 0.25, 0.75] * 4)))
    return out


def as_tensor(blocks: list[np.ndarray], blocks_per_row: int, first: np.ndarray | None = None):
    """Rows of `blocks_per_row` blocks (zero blocks fill the last row); with
    `first`, every row starts with that block."""
    per = blocks_per_row - (1 if first is not None else 0)
    rows = []
    for i in range(0, len(blocks), per):
        row = list(blocks[i:i + per])
        row += [np.zeros(16)] * (per - len(row))
        if first is not None:
            row = [first] + row
        rows.append(np.concatenate(row))
    return torch.from_numpy(np.stack(rows).astype(np.float32)).to(torch.bfloat16)


# S_enc values: exactly 1, one fp32 step above 1, one below, and an exact
# power of two that moves every scale down three binades.
STATIC_SCALES = (1.0, 1.0 + 2.0 ** -23, 1.0 - 2.0 ** -24, 0.125)
