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
