"""Pins for the oracle's E2M1 / E4M3 encoders and decoders.

Expected values are written out from the format definitions (E2M1: sign,
2 exponent bits with bias 1, 1 mantissa bit; E4M3 "fn": sign, 4 exponent
bits with bias 7, 3 mantissa bits, no infinities, S.1111.111 = NaN) and
cross-checked against torch's own float8_e4m3fn cast, which shares no code
with the oracle.
"""
import math

import numpy as np
import pytest
import torch

E2M1_MAGS = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_value_set(orc):
    for c in range(16):
        mag = E2M1_MAGS[c & 7]
        v = orc.e2m1_value(c)
        assert abs(v) == mag
        assert math.copysign(1.0, v) == (-1.0 if c & 8 else 1.0)


def test_e2m1_round_trip(orc):
    for c in range(16):
        assert orc.e2m1_encode(orc.e2m1_value(c)) == c


# (input, expected code), derived by hand: nearest of the value set,
# ties to the even code, saturation at 6, sign bit kept.
E2M1_CASES = [
    (0.0, 0), (0.24, 0), (0.25, 0), (0.2500001, 1), (0.5, 1), (0.74, 1),
    (0.75, 2), (1.0, 2), (1.2499, 2), (1.25, 2), (1.2501, 3), (1.5, 3),
    (1.7499, 3), (1.75, 4), (2.0, 4), (2.5, 4), (2.5001, 5), (3.0, 5),
    (3.4999, 5), (3.5, 6), (4.0, 6), (4.9999, 6), (5.0, 6), (5.0001, 7),
    (6.0, 7), (6.5, 7), (7.0, 7), (1e30, 7), (float("inf"), 7),
    (-0.0, 8), (-0.1, 8), (-0.25, 8), (-0.26, 9), (-0.75, 10), (-1.75, 12),
    (-2.5, 12), (-3.5, 14), (-5.0, 14), (-5.5, 15), (-100.0, 15),
    (1e-45, 0), (-1e-45, 8),
]


@pytest.mark.parametrize("v,code", E2M1_CASES)
def test_e2m1_hand_derived(orc, v, code):
    assert orc.e2m1_encode(v) == code


def test_e2m1_nearest_and_sign_symmetry(orc):
    rng = np.random.default_rng(11)
    vals = np.concatenate([rng.uniform(0, 7, 4000), np.linspace(0, 6.5, 2601)]).astype(np.float32)
    for v in vals:
        c = orc.e2m1_encode(float(v))
        got = E2M1_MAGS[c & 7]
        best = min(abs(m - float(v)) for m in E2M1_MAGS[:7] + [6.0])
        if float(v) <= 6.0:
            assert abs(got - float(v)) == best
        else:
            assert got == 6.0
        if float(v) != 0.0:
            assert orc.e2m1_encode(-float(v)) == (c | 8)


def _e4m3_literal(c):
    s = -1.0 if c & 0x80 else 1.0
    e = (c >> 3) & 15
    m = c & 7
    if e == 15 and m == 7:
        return float("nan")
    if e == 0:
        return s * m / 512.0
    return s * (1 + m / 8) * 2.0 ** (e - 7)


def test_e4m3_literals(orc):
    assert orc.e4m3_value(0x7E) == 448.0
    assert orc.e4m3_value(0x01) == 2.0 ** -9
    assert orc.e4m3_value(0x07) == 7 * 2.0 ** -9
    assert orc.e4m3_value(0x08) == 2.0 ** -6
    assert orc.e4m3_value(0x38) == 1.0
    assert orc.e4m3_value(0x30) == 0.5
    assert orc.e4m3_value(0x35) == 0.8125
    assert math.isnan(orc.e4m3_value(0x7F)) and math.isnan(orc.e4m3_value(0xFF))
    for c in range(256):
        a, b = orc.e4m3_value(c), _e4m3_literal(c)
        assert (math.isnan(a) and math.isnan(b)) or a == b


def test_e4m3_round_trip(orc):
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue
        assert orc.e4m3_encode(orc.e4m3_value(c)) == c


def test_e4m3_against_torch_cast(orc):
    # torch's float8_e4m3fn cast rounds to nearest-even and is independent of
    # the oracle; it turns values >= 464 into NaN, so compare below that.
    rng = np.random.default_rng(5)
    vals = [orc.e4m3_value(c) for c in range(127)]
    mids = [(vals[i] + vals[i + 1]) / 2 for i in range(126)]
    near = [m * f for m in mids for f in (1 - 2**-20, 1.0, 1 + 2**-20)]
    rand = list(np.exp(rng.uniform(np.log(1e-4), np.log(463.0), 20000)))
    tiny = [2.0 ** -10, 2.0 ** -10 * 1.0001, 2.0 ** -11, 1e-30, 0.0]
    xs = np.array(near + rand + tiny + vals, dtype=np.float32)
    xs = xs[xs < 464.0]
    t = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for x, tc in zip(xs, t):
        assert orc.e4m3_encode(float(x)) == int(tc), float(x)


def test_e4m3_saturates(orc):
    for v in (448.0, 449.0, 463.9, 464.0, 480.0, 1e6, float("inf")):
        assert orc.e4m3_encode(v) == 0x7E
    # tie between 416 (0x7D) and 448 (0x7E): even code wins
    assert orc.e4m3_encode(432.0) == 0x7E
    # below half the smallest subnormal -> 0; the tie 2^-10 goes to even 0
    assert orc.e4m3_encode(2.0 ** -10) == 0x00
    assert orc.e4m3_encode(2.0 ** -10 * 1.0001) == 0x01
