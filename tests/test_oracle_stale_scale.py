"""The per-tensor scale one call stale (one-pass quantize): S_enc from an
earlier tensor's amax instead of this tensor's ("static or dynamic" FP32
scale, "英伟达B200狂飙10.2倍！AI绘图告别龟速！", section "NVFP4量化").

Pins of the oracle's one-pass form, and its error measured against the
oracle's dynamic quantization of the same tensor (relative RMS error of the
fp64 dequantized tensor), on the seeded DiT-shaped inputs scaled by a
growth factor between the two calls."""
import numpy as np
import pytest
import torch

import oracle
from workloads import bf16_bits, draw_x

ROWS, COLS = 256, 3072


def _rel_err(q, sf, s_dec, x):
    ref = x.double().numpy()
    deq = oracle.dequantize(q, sf, s_dec, ROWS, COLS)
    return float(np.linalg.norm(deq - ref) / np.linalg.norm(ref)), deq


def test_one_pass_with_own_amax_is_dynamic(orc):
    x = draw_x("lognormal_channels", ROWS, COLS, seed=21, index=0)
    xb = bf16_bits(x)
    q, sf, sd, amax = oracle.quantize_one_pass(xb, ROWS, COLS, oracle.tensor_amax(xb))
    dq, dsf, dsd, damax = oracle.quantize_dynamic(xb, ROWS, COLS)
    assert np.array_equal(q, dq) and np.array_equal(sf, dsf)
    assert sd == dsd and amax == damax


@pytest.mark.parametrize("dist", ["lognormal_channels", "normal_outliers", "gelu"])
def test_stale_scale_error(orc, dist):
    """Growth up to 1.1x between calls costs nothing measurable (the E4M3
    block scales are floating point); growth beyond the stale amax saturates
    the largest blocks: nothing dequantizes above the stale amax, and at 4x
    the error is well above the dynamic one."""
    x1 = draw_x(dist, ROWS, COLS, seed=22, index=0)
    a1 = oracle.tensor_amax(bf16_bits(x1))
    for growth in (0.9, 1.1, 4.0):
        x2 = (x1.float() * growth).to(torch.bfloat16)
        xb = bf16_bits(x2)
        e_dyn, _ = _rel_err(*oracle.quantize_dynamic(xb, ROWS, COLS)[:3], x2)
        q, sf, sd, a2 = oracle.quantize_one_pass(xb, ROWS, COLS, a1)
        assert a2 == oracle.tensor_amax(xb)
        e_stale, deq = _rel_err(q, sf, sd, x2)
        if growth <= 1.1:
            assert abs(e_stale - e_dyn) <= 0.01 * e_dyn, (growth, e_dyn, e_stale)
        else:
            assert np.abs(deq).max() <= float(a1) * (1 + 1e-6)
            assert e_stale > 1.5 * e_dyn, (growth, e_dyn, e_stale)
