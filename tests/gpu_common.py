"""Helpers shared by the GPU parity tests: run the CUDA path (through the
C ABI) and the CPU oracle on the same seeded inputs.  The two sides share
only the inputs; no value computed by the CUDA path is given to the oracle."""
import numpy as np
import torch

import oracle
from workloads import bf16_bits

TOL = 1e-2  # |gpu - ref| <= TOL * (|ref| + rms(ref)), per element


def require_cuda():
    assert torch.cuda.is_available(), "GPU test run without a CUDA device"
    import nvfp4_block_scaled_19_b200 as nv
    nv.lib()
    return nv


def gpu_quantize_dynamic(nv, x_cpu, path="fused"):
    """Dynamic quantize on the GPU -> numpy (q, sf, s_dec, amax).
    path "two_kernel": nvfp4_tensor_amax + nvfp4_quantize;
    path "fused": nvfp4_quantize_dynamic (one cooperative launch)."""
    x = x_cpu.cuda()
    if path == "two_kernel":
        amax = nv.tensor_amax(x)
        t = nv.quantize(x, amax)
    else:
        amax = torch.full((1,), -1.0, device="cuda")
        t = nv.quantize_dynamic(x, amax=amax)
    torch.cuda.synchronize()
    code, tag = nv.device_error()
    assert code == 0, f"device wait timed out (tag {tag})"
    return (t.q.cpu().numpy(), t.sf.cpu().numpy(), np.float32(t.s_dec.item()),
            np.float32(amax.item()))


def oracle_quantize_dynamic(x_cpu):
    rows, cols = x_cpu.shape
    return oracle.quantize_dynamic(bf16_bits(x_cpu), rows, cols)


def assert_quant_equal(g, o, what=""):
    gq, gsf, gsdec, gamax = g
    oq, osf, osdec, oamax = o
    assert gamax == oamax, f"{what}: amax {gamax} != {oamax}"
    assert gsdec == osdec, f"{what}: s_dec {gsdec} != {osdec}"
    assert gsf.shape == osf.shape
    bad_sf = np.flatnonzero(gsf != osf)
    assert bad_sf.size == 0, f"{what}: {bad_sf.size} scale bytes differ, first at {bad_sf[:8]}"
    bad_q = np.argwhere(gq.reshape(oq.shape) != oq)
    assert bad_q.size == 0, f"{what}: {len(bad_q)} packed bytes differ, first {bad_q[:4].tolist()}"


def bf16_from_fp64(a: np.ndarray) -> np.ndarray:
    """Round fp64 values to bfloat16 (via fp32; exact for values already
    representable in fp32) and return fp32 copies of the bf16 values."""
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def decode_block(orc, sf_code, qbytes, s_dec) -> np.ndarray:
    """fp64 values of one 16-element block from its 8 code bytes and scale."""
    codes = np.stack([qbytes & 0xF, qbytes >> 4], -1).reshape(-1)
    return np.array([orc.e2m1_value(int(c)) for c in codes]) * orc.e4m3_value(int(sf_code)) * s_dec


def check_fused_blocks(orc, yg, refb, gq, gsf, g_rows, s_enc_y, what, min_equal=0.8):
    """Fused next-layer quantization of a GEMM's output, on sampled rows.

    yg, refb: [R, N] the GPU's bf16 Y and the oracle's bf16-rounded fp64 Y of
    rows g_rows; gq, gsf: the GPU's full fused codes and tiled scales.  A
    block whose 16 bf16 values equal the oracle's must carry the oracle's
    codes and scale.  Any other block (an output rounded the other way after
    a different fp32 summation order) must carry the oracle's scale code when
    its largest magnitude is the oracle's, else one of the two neighbouring
    codes, and its codes must decode to within one scale unit of the GPU's own
    bf16 values: the largest E2M1 rounding step is one unit (between 4 and 6),
    saturation above 6 costs less.  Returns the oracle's (q, sf)."""
    import torch
    R, N = refb.shape
    kb = N // 16
    oq, osf = orc.quantize(bf16_bits(torch.from_numpy(refb).to(torch.bfloat16)), R, N,
                           np.float32(s_enc_y))
    s_dec = float(np.float32(1.0) / np.float32(s_enc_y))
    same = other = 0
    for i, r in enumerate(g_rows):
        eq = (yg[i] == refb[i]).reshape(kb, 16).all(axis=1)
        for c in range(kb):
            gs = int(gsf[orc.sf_offset(int(r), c, kb)])
            os_ = int(osf[orc.sf_offset(i, c, kb)])
            gqb = gq[r, c * 8:(c + 1) * 8]
            if eq[c]:
                same += 1
                assert gs == os_, (what, r, c)
                assert np.array_equal(gqb, oq[i, c * 8:(c + 1) * 8]), (what, r, c)
                continue
            other += 1
            yb = yg[i, c * 16:(c + 1) * 16].astype(np.float64)
            rb = refb[i, c * 16:(c + 1) * 16]
            if np.abs(yb).max() == np.abs(rb).max():
                assert gs == os_, (what, r, c, gs, os_)
            else:
                assert abs(gs - os_) <= 1, (what, r, c, gs, os_)
            unit = orc.e4m3_value(gs) if gs else 6.0 * 2.0 ** -10
            deq = decode_block(orc, gs, gqb, s_dec)
            assert np.all(np.abs(deq - yb) <= unit * s_dec * (1 + 2.0 ** -10)), (what, r, c)
    assert same > min_equal * (same + other), f"{what}: only {same} of {same + other} blocks equal"
    return oq, osf
