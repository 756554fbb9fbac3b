"""Pins of the oracle's per-token (per-row) quantization: the per-tensor FP32
scale of the two-level scheme ("英伟达B200狂飙10.2倍！AI绘图告别龟速！",
section "NVFP4量化") taken per row.  Each pin reduces the per-row oracle to
the already pinned per-tensor one, or checks a property that a plausible
mistake (the global amax, a misplaced row of scales) would break."""
import numpy as np
import torch

import oracle
from workloads import bf16_bits, draw_x


def _x(rows, cols, seed):
    return draw_x("normal_outliers", rows, cols, seed=seed, index=0)


def test_rows_with_equal_amax_match_per_tensor():
    rows, cols = 130, 80
    x = _x(rows, cols, 1).float()
    x[torch.arange(rows), torch.arange(rows) % cols] = 100.0   # every row's max is 100
    xb = bf16_bits(x.to(torch.bfloat16))
    q, sf, sdec, amax = oracle.quantize_rowwise(xb, rows, cols)
    tq, tsf, tsdec, tamax = oracle.quantize_dynamic(xb, rows, cols)
    assert np.array_equal(q, tq) and np.array_equal(sf, tsf)
    assert np.all(sdec == tsdec) and np.all(amax == tamax)


def test_power_of_two_row_scaling_keeps_codes():
    rows, cols = 64, 96
    x = _x(rows, cols, 2)
    scaled = x.float().clone()
    k = np.array([(r % 9) - 4 for r in range(rows)], dtype=np.float32)
    scaled *= torch.from_numpy(2.0 ** k)[:, None]
    q1, sf1, sd1, _ = oracle.quantize_rowwise(bf16_bits(x), rows, cols)
    q2, sf2, sd2, _ = oracle.quantize_rowwise(bf16_bits(scaled.to(torch.bfloat16)), rows, cols)
    assert np.array_equal(q1, q2) and np.array_equal(sf1, sf2)
    assert np.array_equal(sd2, (sd1 * (2.0 ** k)).astype(np.float32))


def test_one_row_does_not_change_the_others():
    rows, cols = 128, 64
    x = _x(rows, cols, 3).float()
    y = x.clone()
    y[17] *= 1000.0                                  # an outlier token
    q1, sf1, _, _ = oracle.quantize_rowwise(bf16_bits(x.to(torch.bfloat16)), rows, cols)
    q2, sf2, _, _ = oracle.quantize_rowwise(bf16_bits(y.to(torch.bfloat16)), rows, cols)
    other = [r for r in range(rows) if r != 17]
    assert np.array_equal(q1[other], q2[other])
    kb = cols // 16
    offs = [oracle.sf_offset(r, c, kb) for r in other for c in range(kb)]
    assert np.array_equal(sf1[offs], sf2[offs])
    # ... whereas with one per-tensor scale the outlier changes other rows.
    t1, _, _, _ = oracle.quantize_dynamic(bf16_bits(x.to(torch.bfloat16)), rows, cols)
    t2, _, _, _ = oracle.quantize_dynamic(bf16_bits(y.to(torch.bfloat16)), rows, cols)
    assert not np.array_equal(t1[other], t2[other])


def test_row_subset_and_padding():
    rows, cols = 70, 48
    xb = bf16_bits(_x(rows, cols, 4))
    q, sf, sd, am = oracle.quantize_rowwise(xb, rows, cols)
    sel = np.array([0, 5, 69])
    qs, sfs, sds, ams = oracle.quantize_rowwise(xb, rows, cols, row_idx=sel)
    assert np.array_equal(qs[sel], q[sel]) and np.array_equal(sds[sel], sd[sel])
    kb = cols // 16
    for r in sel:
        for c in range((kb + 3) // 4 * 4):
            assert sfs[oracle.sf_offset(int(r), c, kb)] == sf[oracle.sf_offset(int(r), c, kb)]
    pad = [oracle.sf_offset(r, c, kb) for r in range(rows, 128) for c in range(4)]
    assert np.all(sf[pad] == 0)


def test_gemm_rowwise_reduces_to_per_tensor():
    M, N, K = 40, 24, 64
    x = _x(M, K, 5).float()
    x[torch.arange(M), torch.arange(M) % K] = 50.0           # equal row amax
    xb = bf16_bits(x.to(torch.bfloat16))
    wb = bf16_bits(_x(N, K, 6))
    aq, asf, asd, _ = oracle.quantize_rowwise(xb, M, K)
    tq, tsf, tsd, _ = oracle.quantize_dynamic(xb, M, K)
    bq, bsf, bsd, _ = oracle.quantize_dynamic(wb, N, K)
    assert np.array_equal(oracle.gemm_rowwise(aq, asf, asd, bq, bsf, bsd, M, N, K),
                          oracle.gemm(tq, tsf, tsd, bq, bsf, bsd, M, N, K))


def test_rowwise_error_against_per_tensor_with_outlier_tokens():
    """Where per-token scales matter, measured on the oracle.  The E4M3 block
    scales span about 17 binades, so with one tensor scale an outlier token
    costs the other tokens nothing until it is ~1e4 x larger; beyond that
    their block scales fall into E4M3 subnormals and then to zero, while the
    per-row error stays put (relative Frobenius error of the other tokens:
    0.092 for both at x300, 0.180 against 0.092 at x1e5, 0.999 against 0.092
    at x1e6)."""
    rows, cols = 256, 512
    base = draw_x("lognormal_channels", rows, cols, seed=7, index=0).float()
    normal = np.ones(rows, bool)
    normal[::64] = False
    errs = {}
    for f in (300.0, 1e5, 1e6):
        x = base.clone()
        x[::64] *= f                                      # 4 outlier tokens
        xb16 = x.to(torch.bfloat16)
        xb = bf16_bits(xb16)
        xf = xb16.double().numpy()
        tq, tsf, tsd, _ = oracle.quantize_dynamic(xb, rows, cols)
        rq, rsf, rsd, _ = oracle.quantize_rowwise(xb, rows, cols)
        t_hat = oracle.dequantize(tq, tsf, tsd, rows, cols)
        r_hat = oracle.dequantize(rq, rsf, 1.0, rows, cols) * rsd.astype(np.float64)[:, None]
        err = lambda h: np.linalg.norm(h[normal] - xf[normal]) / np.linalg.norm(xf[normal])
        errs[f] = (err(r_hat), err(t_hat))
    assert abs(errs[300.0][0] - errs[300.0][1]) < 1e-3          # no difference yet
    assert errs[1e5][1] > 1.5 * errs[1e5][0]                     # subnormal block scales
    assert errs[1e6][1] > 0.99 and errs[1e6][0] < 0.1            # zeroed blocks vs per-row
