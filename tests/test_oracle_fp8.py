"""Pins of the oracle's FP8 variant (E4M3 elements, one FP32 per-tensor scale
S_enc = 448 / amax; the pages' "--variant fp8r" mode in "NVIDIA показала, как
сократить генерацию FLUX 3 Image Klein с 22 до 6 секунд", section "2. Запуск
генерации изображения"), against facts the oracle does not compute: torch's
own float8_e4m3fn conversion, the amax-to-448 property, exactly
representable round trips and a closed-form GEMM."""
import numpy as np
import torch

import oracle
from workloads import bf16_bits, draw_x


def test_codes_match_torch_float8_cast():
    for dist, seed in (("normal_outliers", 1), ("lognormal_channels", 2), ("gelu", 3)):
        x = draw_x(dist, 64, 512, seed=seed, index=0)
        q, s_dec, amax = oracle.quantize_fp8(bf16_bits(x), 64, 512)
        s_enc = oracle.fp8_tensor_scale(amax)
        prod = x.float() * torch.tensor(float(s_enc), dtype=torch.float32)   # fp32 RN product
        want = prod.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(q, want), dist
        assert s_dec == np.float32(1.0) / s_enc


def test_amax_element_maps_to_448():
    x = draw_x("normal_outliers", 32, 256, seed=4, index=0).float()
    x[5, 7] = -500.0
    x[9, 3] = 500.0
    q, _, amax = oracle.quantize_fp8(bf16_bits(x.to(torch.bfloat16)), 32, 256)
    assert amax == np.float32(500.0)
    assert q[9, 3] == 0x7E and q[5, 7] == 0xFE          # +448, -448


def test_scale_special_cases():
    assert oracle.fp8_tensor_scale(0.0) == np.float32(1.0)
    assert oracle.fp8_tensor_scale(2.0 ** -133) == np.float32(np.finfo(np.float32).max)
    assert oracle.fp8_tensor_scale(448.0) == np.float32(1.0)
    z = torch.zeros(4, 32, dtype=torch.bfloat16)
    q, s_dec, amax = oracle.quantize_fp8(bf16_bits(z), 4, 32)
    assert amax == 0 and s_dec == 1 and np.all(q == 0)


def test_representable_round_trip_and_exact_gemm():
    rng = np.random.default_rng(0)
    vals = np.array([oracle.e4m3_value(c) for c in range(0x7F)])   # non-negative E4M3 set
    M, N, K = 24, 16, 64
    a = rng.choice(vals[vals <= 16], (M, K)) * rng.choice([-1.0, 1.0], (M, K))
    b = rng.choice(vals[vals <= 16], (N, K)) * rng.choice([-1.0, 1.0], (N, K))
    a[0, 0], b[0, 0] = 448.0, 448.0                      # amax 448 -> S_enc = 1
    ab = torch.from_numpy(a).to(torch.bfloat16)
    bb = torch.from_numpy(b).to(torch.bfloat16)
    aq, asd, _ = oracle.quantize_fp8(bf16_bits(ab), M, K)
    bq, bsd, _ = oracle.quantize_fp8(bf16_bits(bb), N, K)
    assert asd == 1 and bsd == 1
    assert np.array_equal(oracle.dequantize_fp8(aq, asd), a)
    assert np.array_equal(oracle.gemm_fp8(aq, asd, bq, bsd), a @ b.T)
