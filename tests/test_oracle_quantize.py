"""Pins for the oracle's tensor scale, block quantizer and scale layout.

Each test checks the oracle against something it does not compute itself:
hand-derived worked examples (tests/golden/), lossless round trips of
exactly representable inputs, the block-amax-to-6 invariant, sign symmetry,
the dequantization error bound and brute-force layout properties.
"""
import os

import numpy as np
import pytest
import torch

from workloads import WORKLOADS, bf16_bits, layer_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
FLT_MAX = np.float32(3.4028234663852886e38)


def _bits(values):
    return bf16_bits(torch.tensor(values, dtype=torch.float32).to(torch.bfloat16))


def test_tensor_scale_cases(orc):
    assert orc.tensor_scale(0.0) == np.float32(1.0)
    assert orc.tensor_scale(2688.0) == np.float32(1.0)
    assert orc.tensor_scale(6.0) == np.float32(448.0)
    assert orc.tensor_scale(1e-40) == FLT_MAX          # 2688/amax overflows
    assert orc.tensor_scale(5.0) == np.float32(537.6)  # one fp32 division
    assert orc.decode_scale(np.float32(448.0)) == np.float32(1.0) / np.float32(448.0)


def test_tensor_amax(orc):
    x = _bits([0.5, -7.25, 3.0, -0.0, 7.0])
    assert orc.tensor_amax(x) == np.float32(7.25)
    assert orc.tensor_amax(_bits([0.0, -0.0])) == np.float32(0.0)


def _read_golden(name):
    d = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, _, v = line.partition(" ")
            d[k] = v.split()
    return d


def test_worked_example(orc):
    g = _read_golden("quantize_worked_example.txt")
    rows, cols = int(g["rows"][0]), int(g["cols"][0])
    x = _bits([float(v) for v in g["x"]])
    q, sf = orc.quantize(x, rows, cols, np.float32(float(g["s_enc"][0])))
    assert [f"{b:02x}" for b in q.reshape(-1)] == g["q"]
    assert sf.size == int(g["sf_bytes"][0])
    want = np.zeros_like(sf)
    for item in g["sf_nonzero"]:
        off, val = item.split(":")
        want[int(off)] = int(val, 16)
    assert np.array_equal(sf, want)


def test_sf_offsets_golden(orc):
    with open(os.path.join(GOLDEN, "sf_layout_offsets.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            r, c, kb, off = map(int, line.split())
            assert orc.sf_offset(r, c, kb) == off, (r, c, kb)


@pytest.mark.parametrize("rows,kb", [(1, 1), (130, 5), (256, 8), (77, 12)])
def test_sf_layout_is_bijection(orc, rows, kb):
    total = orc.sf_bytes(rows, kb * 16)
    assert total == ((rows + 127) // 128 * 128) * ((kb + 3) // 4 * 4)
    seen = np.zeros(total, dtype=np.int32)
    for r in range((rows + 127) // 128 * 128):
        for c in range((kb + 3) // 4 * 4):
            seen[orc.sf_offset(r, c, kb)] += 1
    assert np.all(seen == 1)


def _representable_tensor(rng, rows, kb, exps):
    """Blocks of 2^e * (E2M1 value) with one element per block at +-6*2^e."""
    mags = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    codes = rng.integers(0, 16, size=(rows, kb, 16))
    lead = rng.integers(0, 16, size=(rows, kb))
    for r in range(rows):
        for c in range(kb):
            codes[r, c, lead[r, c]] = 7 | (rng.integers(0, 2) << 3)
    e = rng.choice(exps, size=(rows, kb))
    vals = mags[codes & 7] * np.where(codes & 8, -1.0, 1.0) * (2.0 ** e)[..., None]
    return vals.reshape(rows, kb * 16), codes, e


def test_lossless_round_trip(orc):
    # With S_enc = 1 each block scale is 2^e exactly (an E4M3 value for
    # e in [-9, 8]), so every element is encoded exactly and dequantizes to
    # the input bit for bit.
    rng = np.random.default_rng(3)
    rows, kb = 37, 6
    vals, codes, e = _representable_tensor(rng, rows, kb, np.arange(-9, 9))
    x = _bits(vals.astype(np.float32))
    q, sf = orc.quantize(x, rows, kb * 16, np.float32(1.0))
    xhat = orc.dequantize(q, sf, np.float32(1.0), rows, kb * 16)
    assert np.array_equal(xhat, vals)
    for r in range(rows):
        for c in range(kb):
            assert orc.e4m3_value(sf[orc.sf_offset(r, c, kb)]) == 2.0 ** e[r, c]
    # the codes themselves (zeros may carry either sign)
    lo = q & 0xF
    hi = q >> 4
    got = np.stack([lo, hi], -1).reshape(rows, kb, 16)
    nz = (codes & 7) != 0
    assert np.array_equal(got[nz], codes[nz])


def test_block_amax_maps_to_six(orc):
    # For every block whose scale is a normal E4M3 value, the element with
    # |x| = a_b encodes to magnitude code 7 (value 6): the E4M3 relative
    # rounding error is at most 2^-4 and 6/(1+2^-4) > 5, the 4|6 midpoint.
    w = WORKLOADS["tiny_linear"]
    x, _ = layer_inputs(w, 0)
    rows, cols = x.shape
    xb = bf16_bits(x)
    q, sf, _, _ = orc.quantize_dynamic(xb, rows, cols)
    xf = x.float().numpy().reshape(rows, cols // 16, 16)
    codes = np.stack([q & 0xF, q >> 4], -1).reshape(rows, cols // 16, 16)
    kb = cols // 16
    checked = 0
    for r in range(rows):
        for c in range(kb):
            s = sf[orc.sf_offset(r, c, kb)]
            if (s >> 3) == 0:      # subnormal or zero scale: invariant not claimed
                continue
            i = int(np.argmax(np.abs(xf[r, c])))
            assert (codes[r, c, i] & 7) == 7
            checked += 1
    assert checked > 0.9 * rows * kb


def test_sign_symmetry(orc):
    w = WORKLOADS["tiny_linear"]
    x, _ = layer_inputs(w, 0, M=64)
    rows, cols = x.shape
    s_enc = orc.tensor_scale(orc.tensor_amax(bf16_bits(x)))
    q1, sf1 = orc.quantize(bf16_bits(x), rows, cols, s_enc)
    q2, sf2 = orc.quantize(bf16_bits(-x), rows, cols, s_enc)
    assert np.array_equal(sf1, sf2)
    assert np.array_equal(q2, q1 ^ 0x88)


def test_dequantization_error_bound(orc):
    # |x - x_hat| <= sf * S_dec * (1 + 2^-20): in code space the E2M1 rounding
    # error is at most 1 (half the widest gap, 4..6) and saturation above 6
    # costs at most 6 * 2^-4 < 1.
    w = WORKLOADS["qkv_1024"]
    x, _ = layer_inputs(w, 0, M=96)
    rows, cols = x.shape
    q, sf, s_dec, _ = orc.quantize_dynamic(bf16_bits(x), rows, cols)
    xhat = orc.dequantize(q, sf, s_dec, rows, cols)
    kb = cols // 16
    sfv = np.array([[orc.e4m3_value(sf[orc.sf_offset(r, c, kb)]) for c in range(kb)]
                    for r in range(rows)])
    bound = np.repeat(sfv, 16, axis=1) * float(s_dec) * (1 + 2**-20)
    err = np.abs(x.double().numpy() - xhat)
    assert np.all(err <= bound + 1e-300)


def test_zero_and_underflow_blocks(orc):
    rows, cols = 2, 48
    vals = np.zeros((rows, cols), dtype=np.float32)
    vals[0, 16:32] = -0.0             # block of negative zeros
    vals[1, :16] = 1000.0             # sets the tensor amax
    vals[1, 16:32] = 1e-4             # far below 2^-10 of the block scale
    vals[1, 32] = -1e-4
    vals = vals.copy()
    vals[0, 16:32] = np.float32(-0.0)
    x = _bits(vals)
    s_enc = orc.tensor_scale(orc.tensor_amax(x))
    q, sf = orc.quantize(x, rows, cols, s_enc)
    kb = 3
    assert sf[orc.sf_offset(0, 0, kb)] == 0
    assert sf[orc.sf_offset(0, 1, kb)] == 0
    assert sf[orc.sf_offset(1, 1, kb)] == 0     # scale underflows to 0
    assert np.all(q[0, :8] == 0)
    assert np.all(q[0, 8:16] == 0x88)           # -0 keeps its sign bit
    assert np.all(q[1, 8:16] == 0)
    assert q[1, 16] & 0x0F == 0x8               # -1e-4 * 0 = -0 -> code 8
    # padding of the scale layout stays zero
    used = {orc.sf_offset(r, c, kb) for r in range(rows) for c in range(kb)}
    pad = np.array([sf[i] for i in range(sf.size) if i not in used])
    assert np.all(pad == 0)


def test_bf16_subnormal_tensor(orc):
    # amax of a subnormal-only tensor makes 2688/amax overflow: S_enc=FLT_MAX.
    tiny = np.float32(2.0 ** -130)
    x = _bits(np.array([tiny, -tiny] * 8, dtype=np.float32))
    amax = orc.tensor_amax(x)
    assert amax == tiny
    s_enc = orc.tensor_scale(amax)
    assert s_enc == FLT_MAX
    q, sf = orc.quantize(x, 1, 16, s_enc)
    # a_b/6 = 2^-130/6 is the fp32 subnormal 87381 * 2^-149; times FLT_MAX
    # that is ~0.041666 = 1.333 * 2^-5, between 1.25 and 1.375 (midpoint
    # 1.3125) -> mantissa 3, exponent field 2 -> code 0x13.
    assert sf[0] == 0x13
    # inv = FLT_MAX / 0.04296875 overflows and is clamped to FLT_MAX, so
    # x * inv = 2^-130 * FLT_MAX = 0.25 * (1 - 2^-24) -> below the 0|0.5 tie -> 0
    # (with the sign kept); a zero element stays 0 instead of becoming NaN.
    assert np.all(q == 0x80)
    z = _bits(np.array([tiny, 0.0] * 8, dtype=np.float32))
    qz, _ = orc.quantize(z, 1, 16, s_enc)
    assert np.all(qz == 0)
