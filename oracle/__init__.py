"""CPU oracle for NVFP4 quantization and the block-scaled FP4 GEMM.

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
cpu_baseline / reference legs of bench.py may import this package; the
product path (nvfp4_block_scaled_19_b200) never does, and the two share no
code.  The scalar steps live in nvfp4_oracle.c (see its header for the
pages followed and every reading taken); this module marshals numpy arrays
and does the one library step: the fp64 matrix product of the dequantized
operands (numpy.matmul), after which nothing is reordered or fused.

Parity status: every function here is pinned by tests/test_oracle_*.py
against facts that do not come from the oracle itself (format value sets,
hand-derived rounding ties, torch's float8_e4m3fn conversion, exact rational
GEMMs, lossless round trips, the amax-to-6 invariant, and for gelu the
normal-CDF identities and table values).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        c_u8p = ctypes.POINTER(ctypes.c_uint8)
        c_u16p = ctypes.POINTER(ctypes.c_uint16)
        c_dp = ctypes.POINTER(ctypes.c_double)
        c_i64p = ctypes.POINTER(ctypes.c_int64)
        i64 = ctypes.c_int64
        L.ref_e2m1_value.restype = ctypes.c_double
        L.ref_e2m1_value.argtypes = [ctypes.c_uint8]
        L.ref_e4m3_value.restype = ctypes.c_double
        L.ref_e4m3_value.argtypes = [ctypes.c_uint8]
        L.ref_e2m1_encode.restype = ctypes.c_uint8
        L.ref_e2m1_encode.argtypes = [ctypes.c_float]
        L.ref_e4m3_encode.restype = ctypes.c_uint8
        L.ref_e4m3_encode.argtypes = [ctypes.c_float]
        L.ref_tensor_amax.restype = ctypes.c_float
        L.ref_tensor_amax.argtypes = [c_u16p, i64]
        L.ref_tensor_scale.restype = ctypes.c_float
        L.ref_tensor_scale.argtypes = [ctypes.c_float]
        L.ref_decode_scale.restype = ctypes.c_float
        L.ref_decode_scale.argtypes = [ctypes.c_float]
        L.ref_sf_bytes.restype = i64
        L.ref_sf_bytes.argtypes = [i64, i64]
        L.ref_sf_offset.restype = i64
        L.ref_sf_offset.argtypes = [i64, i64, i64]
        L.ref_fp8_tensor_scale.restype = ctypes.c_float
        L.ref_fp8_tensor_scale.argtypes = [ctypes.c_float]
        L.ref_quantize_fp8.restype = None
        L.ref_quantize_fp8.argtypes = [c_u16p, i64, ctypes.c_float, c_u8p]
        L.ref_quantize.restype = None
        L.ref_quantize.argtypes = [c_u16p, i64, i64, ctypes.c_float, c_u8p, c_u8p]
        L.ref_dequantize.restype = None
        L.ref_dequantize.argtypes = [c_u8p, c_u8p, ctypes.c_float, i64, i64, c_i64p, i64, c_dp]
        L.ref_gemm_naive.restype = None
        L.ref_gemm_naive.argtypes = [c_dp, c_dp, i64, i64, i64, c_dp]
        L.ref_num_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a: np.ndarray, ctype):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctype))


# ---------------------------------------------------------------- formats

def e2m1_value(code: int) -> float:
    return lib().ref_e2m1_value(code)


def e4m3_value(code: int) -> float:
    return lib().ref_e4m3_value(code)


def e2m1_encode(v: float) -> int:
    return lib().ref_e2m1_encode(float(np.float32(v)))


def e4m3_encode(v: float) -> int:
    return lib().ref_e4m3_encode(float(np.float32(v)))


# ---------------------------------------------------------------- scales

def tensor_amax(x_bits: np.ndarray) -> np.float32:
    """max |x| over a bfloat16 tensor given as uint16 bit patterns."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16).reshape(-1)
    return np.float32(lib().ref_tensor_amax(_ptr(x, ctypes.c_uint16), x.size))


def tensor_scale(amax) -> np.float32:
    """S_enc = 2688 / amax (1 if amax == 0, FLT_MAX if not finite)."""
    return np.float32(lib().ref_tensor_scale(float(np.float32(amax))))


def decode_scale(s_enc) -> np.float32:
    return np.float32(lib().ref_decode_scale(float(np.float32(s_enc))))


# ---------------------------------------------------------------- layout

def sf_bytes(rows: int, cols: int) -> int:
    return int(lib().ref_sf_bytes(rows, cols))


def sf_offset(r: int, c: int, kb: int) -> int:
    return int(lib().ref_sf_offset(r, c, kb))


def packed_bytes(rows: int, cols: int) -> int:
    return rows * cols // 2


# ---------------------------------------------------------------- quantize

def quantize(x_bits: np.ndarray, rows: int, cols: int, s_enc) -> tuple[np.ndarray, np.ndarray]:
    """NVFP4 quantize with a given S_enc -> (q [rows, cols/2] u8, sf tiled u8)."""
    assert cols % 16 == 0
    x = np.ascontiguousarray(x_bits, dtype=np.uint16).reshape(-1)
    assert x.size == rows * cols
    q = np.empty(rows * cols // 2, dtype=np.uint8)
    sf = np.empty(sf_bytes(rows, cols), dtype=np.uint8)
    lib().ref_quantize(_ptr(x, ctypes.c_uint16), rows, cols, float(np.float32(s_enc)),
                       _ptr(q, ctypes.c_uint8), _ptr(sf, ctypes.c_uint8))
    return q.reshape(rows, cols // 2), sf


def quantize_dynamic(x_bits: np.ndarray, rows: int, cols: int):
    """amax -> S_enc -> quantize; returns (q, sf, s_dec, amax)."""
    amax = tensor_amax(x_bits)
    s_enc = tensor_scale(amax)
    q, sf = quantize(x_bits, rows, cols, s_enc)
    return q, sf, decode_scale(s_enc), amax


def quantize_one_pass(x_bits: np.ndarray, rows: int, cols: int, amax_prev):
    """The per-tensor scale one call stale: S_enc from an earlier tensor's
    amax (the "static or dynamic" FP32 scale of the NVFP4 section of the
    nmedialink page, read as dynamic with the previous call's amax), then the
    same block quantize; returns (q, sf, s_dec, amax of this tensor for the
    next call)."""
    s_enc = tensor_scale(amax_prev)
    q, sf = quantize(x_bits, rows, cols, s_enc)
    return q, sf, decode_scale(s_enc), tensor_amax(x_bits)


def dequantize(q: np.ndarray, sf: np.ndarray, s_dec, rows: int, cols: int,
               row_idx: np.ndarray | None = None) -> np.ndarray:
    """fp64 x_hat = e2m1(q) * e4m3(sf) * s_dec for all rows or the listed ones."""
    qq = np.ascontiguousarray(q, dtype=np.uint8).reshape(-1)
    ss = np.ascontiguousarray(sf, dtype=np.uint8).reshape(-1)
    assert qq.size == rows * cols // 2 and ss.size == sf_bytes(rows, cols)
    if row_idx is not None:
        idx = np.ascontiguousarray(row_idx, dtype=np.int64)
        n = idx.size
        ip = _ptr(idx, ctypes.c_int64)
    else:
        idx, n, ip = None, rows, None
    out = np.empty((n, cols), dtype=np.float64)
    lib().ref_dequantize(_ptr(qq, ctypes.c_uint8), _ptr(ss, ctypes.c_uint8),
                         float(np.float32(s_dec)), rows, cols, ip, n if idx is not None else 0,
                         _ptr(out, ctypes.c_double))
    return out


def quantize_rowwise(x_bits: np.ndarray, rows: int, cols: int,
                     row_idx: np.ndarray | None = None):
    """Per-token (per-row) tensor scales: row r is quantized exactly as the
    1-row tensor X[r] with its own dynamic scale (amax, S_enc = 2688/amax,
    the per-16 block scales of quantize()), its scales placed at row r of the
    tiled layout.  The pages' per-tensor FP32 scale ("英伟达B200狂飙10.2倍！
    AI绘图告别龟速！", section "NVFP4量化") taken per row; padding is zero.
    Returns (q [rows, cols/2], sf tiled, s_dec [rows], amax [rows]); with
    row_idx only those rows are computed (the others stay zero)."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16).reshape(rows, cols)
    kb = cols // 16
    kbp = (kb + 3) // 4 * 4
    q = np.zeros((rows, cols // 2), dtype=np.uint8)
    sf = np.zeros(sf_bytes(rows, cols), dtype=np.uint8)
    s_dec = np.zeros(rows, dtype=np.float32)
    amax = np.zeros(rows, dtype=np.float32)
    for r in (range(rows) if row_idx is None else row_idx):
        a = tensor_amax(x[r])
        s_enc = tensor_scale(a)
        qr, sfr = quantize(x[r], 1, cols, s_enc)
        q[r] = qr[0]
        for c in range(kbp):
            sf[sf_offset(int(r), c, kb)] = sfr[sf_offset(0, c, kb)]
        s_dec[r] = decode_scale(s_enc)
        amax[r] = a
    return q, sf, s_dec, amax


def gemm_rowwise(aq, asf, a_sdec_rows, bq, bsf, b_sdec, M: int, N: int, K: int,
                 rows: np.ndarray | None = None) -> np.ndarray:
    """ref[m,n] = sum_k x_hat[m,k] w_hat[n,k] in fp64 with per-row decode
    scales of A: x_hat[m,k] = e2m1 * sf * s_dec[m]."""
    idx = np.arange(M) if rows is None else np.asarray(rows)
    a = dequantize(aq, asf, 1.0, M, K, None if rows is None else idx)
    a = a * np.asarray(a_sdec_rows, dtype=np.float64)[idx][:, None]
    b = dequantize(bq, bsf, b_sdec, N, K)
    return np.matmul(a, b.T)


def fp8_tensor_scale(amax) -> np.float32:
    """FP8 variant: S_enc = 448 / amax (1 if 0, FLT_MAX if not finite)."""
    return np.float32(lib().ref_fp8_tensor_scale(float(np.float32(amax))))


def quantize_fp8(x_bits: np.ndarray, rows: int, cols: int):
    """FP8 (E4M3) with one dynamic FP32 per-tensor scale: returns
    (q [rows, cols] E4M3 codes, s_dec, amax); see nvfp4_oracle.c for the
    pages' passage and the reading taken."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16).reshape(-1)
    amax = tensor_amax(x)
    s_enc = fp8_tensor_scale(amax)
    q = np.empty(x.size, dtype=np.uint8)
    lib().ref_quantize_fp8(_ptr(x, ctypes.c_uint16), x.size, float(s_enc), _ptr(q, ctypes.c_uint8))
    return q.reshape(rows, cols), decode_scale(s_enc), amax


def dequantize_fp8(q: np.ndarray, s_dec, rows: np.ndarray | None = None) -> np.ndarray:
    """fp64 x_hat = e4m3(q) * s_dec (all rows or the listed ones)."""
    table = np.array([e4m3_value(c) if (c & 0x7F) != 0x7F else np.nan for c in range(256)])
    qq = np.asarray(q) if rows is None else np.asarray(q)[rows]
    return table[qq] * np.float64(np.float32(s_dec))


def gemm_fp8(aq, a_sdec, bq, b_sdec, rows: np.ndarray | None = None) -> np.ndarray:
    """ref[m,n] = sum_k x_hat[m,k] w_hat[n,k] in fp64 for the FP8 variant."""
    return np.matmul(dequantize_fp8(aq, a_sdec, rows), dequantize_fp8(bq, b_sdec).T)


# ---------------------------------------------------------------- GEMM

def gemm(aq, asf, a_sdec, bq, bsf, b_sdec, M: int, N: int, K: int,
         rows: np.ndarray | None = None) -> np.ndarray:
    """ref[m,n] = sum_k x_hat[m,k] * w_hat[n,k] in fp64 (all rows or `rows`)."""
    a = dequantize(aq, asf, a_sdec, M, K, rows)
    b = dequantize(bq, bsf, b_sdec, N, K)
    return np.matmul(a, b.T)


def gemm_naive(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Brute-force fp64 triple loop (small sizes): y = a . b^T."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    b = np.ascontiguousarray(b, dtype=np.float64)
    M, K = a.shape
    N = b.shape[0]
    y = np.empty((M, N), dtype=np.float64)
    lib().ref_gemm_naive(_ptr(a, ctypes.c_double), _ptr(b, ctypes.c_double), M, N, K,
                         _ptr(y, ctypes.c_double))
    return y


def gemm_tolerance_ok(gpu: np.ndarray, ref: np.ndarray, rel: float = 1e-2):
    """|gpu - ref| <= rel * (|ref| + rms(ref)) elementwise; returns (ok, worst ratio)."""
    ref = np.asarray(ref, dtype=np.float64)
    g = np.asarray(gpu, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    bound = rel * (np.abs(ref) + rms)
    err = np.abs(g - ref)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(bound > 0, err / bound, np.where(err > 0, np.inf, 0.0))
    worst = float(ratio.max()) if ratio.size else 0.0
    return bool(np.all(err <= bound)), worst


def gelu(h: np.ndarray) -> np.ndarray:
    """Exact GELU in fp64, g(h) = h * Phi(h) = 0.5 h (1 + erf(h / sqrt 2)): the
    activation a fused FFN up-projection epilogue applies before rounding to
    bf16.  The pages fuse consecutive operations into their GEMM kernels
    ("NVIDIA показала, как сократить генерацию FLUX 3 Image Klein с 22 до 6
    секунд", section "Квантование NVFP4 и оптимизация вычислительных ядер")
    without naming the activation; exact GELU is the reading taken.  One
    library step: scipy's fp64 erf."""
    from scipy.special import erf
    h = np.asarray(h, dtype=np.float64)
    return 0.5 * h * (1.0 + erf(h / np.sqrt(2.0)))


def num_threads() -> int:
    return int(lib().ref_num_threads())
