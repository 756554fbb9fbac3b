"""NVFP4 linear layers for B200 (sm_100a): Python binding of libnvfp4.so.

NVFP4 two-level microblock quantization (FP32 per-tensor scale + E4M3 scale
per 16 elements, E2M1 elements) and the tcgen05 block-scaled FP4 GEMM, as
used for the linear layers of FLUX diffusion transformers ("英伟达B200狂飙
10.2倍！AI绘图告别龟速！", section "NVFP4量化"; "Scaling NVFP4 Inference for
FLUX.2 on NVIDIA Blackwell Data Center GPUs", section "Key Questions
Answered").

This module only marshals arguments: every step runs in the CUDA kernels of
libnvfp4.so through its C ABI (include/nvfp4.h).  PyTorch supplies device
memory and the current stream.  There is no CPU fallback: if the library is
missing or the device is not sm_100, calls raise.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnvfp4.so")

STATUS = {0: "ok", 1: "invalid argument", 2: "misaligned", 3: "unsupported device",
          4: "launch error", 5: "device wait timed out"}


class NVFP4Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {STATUS.get(status, status)} (status {status})")
        self.status = status


class FusedOut(ctypes.Structure):
    _fields_ = [("s_enc_y", ctypes.c_void_p), ("yq", ctypes.c_void_p),
                ("ysf", ctypes.c_void_p), ("amax_y", ctypes.c_void_p),
                ("s_dec_y", ctypes.c_void_p), ("activation", ctypes.c_int)]


ACT_NONE = 0   # nvfp4_activation values
ACT_GELU = 1


class LinearWorkspace(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("xq", ctypes.c_void_p), ("xsf", ctypes.c_void_p),
                ("amax", ctypes.c_void_p), ("s_dec", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("dyn_ws", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C-ABI library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m nvfp4_block_scaled_19_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, st = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.nvfp4_packed_bytes.restype = ctypes.c_size_t
        L.nvfp4_packed_bytes.argtypes = [i64, i64]
        L.nvfp4_sf_bytes.restype = ctypes.c_size_t
        L.nvfp4_sf_bytes.argtypes = [i64, i64]
        L.nvfp4_status_string.restype = ctypes.c_char_p
        L.nvfp4_status_string.argtypes = [st]
        L.nvfp4_tensor_amax.restype = st
        L.nvfp4_tensor_amax.argtypes = [vp, i64, vp, vp]
        L.nvfp4_quantize.restype = st
        L.nvfp4_quantize.argtypes = [vp, i64, i64, vp, vp, vp, vp, vp]
        L.nvfp4_quantize_with_scale.restype = st
        L.nvfp4_quantize_with_scale.argtypes = [vp, i64, i64, vp, vp, vp, vp, vp]
        L.nvfp4_quantize_one_pass.restype = st
        L.nvfp4_quantize_one_pass.argtypes = [vp, i64, i64, vp, vp, vp, vp, vp, vp]
        L.nvfp4_quantize_dynamic_workspace_bytes.restype = ctypes.c_size_t
        L.nvfp4_quantize_dynamic_workspace_bytes.argtypes = []
        L.nvfp4_quantize_dynamic.restype = st
        L.nvfp4_quantize_dynamic.argtypes = [vp, i64, i64, vp, vp, vp, vp, vp, vp]
        L.nvfp4_quantize_dynamic_noalloc.restype = st
        L.nvfp4_quantize_dynamic_noalloc.argtypes = [vp, i64, i64, vp, vp, vp, vp, vp]
        L.nvfp4_gemm.restype = st
        L.nvfp4_gemm.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp,
                                 ctypes.POINTER(FusedOut), vp]
        L.nvfp4_gemm_rowscale.restype = st
        L.nvfp4_gemm_rowscale.argtypes = list(L.nvfp4_gemm.argtypes)
        L.nvfp4_quantize_rowwise.restype = st
        L.nvfp4_quantize_rowwise.argtypes = [vp, i64, i64, vp, vp, vp, vp, vp]
        L.nvfp4_fp8_quantize.restype = st
        L.nvfp4_fp8_quantize.argtypes = [vp, i64, i64, vp, vp, vp, vp]
        L.nvfp4_fp8_gemm.restype = st
        L.nvfp4_fp8_gemm.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, vp, vp]
        L.nvfp4_selftest_wait_timeout.restype = st
        L.nvfp4_selftest_wait_timeout.argtypes = [i64, vp]
        L.nvfp4_linear_host.restype = st
        L.nvfp4_linear_host.argtypes = [vp, i64, i64, vp, vp, vp, i64, vp,
                                        ctypes.POINTER(LinearWorkspace), vp]
        L.nvfp4_device_error.restype = st
        L.nvfp4_device_error.argtypes = [ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
        _lib = L
    return _lib


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise NVFP4Error(fn, status)


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def packed_bytes(rows: int, cols: int) -> int:
    return int(lib().nvfp4_packed_bytes(rows, cols))


def sf_bytes(rows: int, cols: int) -> int:
    return int(lib().nvfp4_sf_bytes(rows, cols))


def _require(x: torch.Tensor, dtype, name: str) -> None:
    if not x.is_cuda or x.dtype != dtype or not x.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor")


@dataclass
class NVFP4Tensor:
    """A quantized [rows, cols] tensor: packed codes, tiled scales, decode scale."""
    q: torch.Tensor       # uint8 [rows, cols/2]
    sf: torch.Tensor      # uint8 [sf_bytes(rows, cols)]
    s_dec: torch.Tensor   # float32 [1] = 1 / S_enc, or [rows] with per-row scales
    rows: int
    cols: int


def empty_nvfp4(rows: int, cols: int, device=None, row_scales: bool = False) -> NVFP4Tensor:
    dev = torch.device("cuda") if device is None else device
    return NVFP4Tensor(torch.empty(rows, cols // 2, dtype=torch.uint8, device=dev),
                       torch.empty(sf_bytes(rows, cols), dtype=torch.uint8, device=dev),
                       torch.empty(rows if row_scales else 1, dtype=torch.float32, device=dev),
                       rows, cols)


def tensor_amax(x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """max |x| of a bf16 CUDA tensor into a 1-element fp32 CUDA tensor."""
    _require(x, torch.bfloat16, "x")
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=x.device)
    _check("nvfp4_tensor_amax", lib().nvfp4_tensor_amax(x.data_ptr(), x.numel(), out.data_ptr(),
                                                        _stream(stream)))
    return out


def quantize(x: torch.Tensor, amax: torch.Tensor, out: NVFP4Tensor | None = None,
             stream=None) -> NVFP4Tensor:
    """Dynamic NVFP4 quantization of bf16 x[rows, cols] given its amax (device)."""
    _require(x, torch.bfloat16, "x")
    rows, cols = x.shape
    out = empty_nvfp4(rows, cols, x.device) if out is None else out
    _check("nvfp4_quantize", lib().nvfp4_quantize(
        x.data_ptr(), rows, cols, amax.data_ptr(), out.q.data_ptr(), out.sf.data_ptr(),
        out.s_dec.data_ptr(), _stream(stream)))
    return out


def quantize_with_scale(x: torch.Tensor, s_enc: torch.Tensor, out: NVFP4Tensor | None = None,
                        stream=None) -> NVFP4Tensor:
    """NVFP4 quantization with a static per-tensor scale S_enc (device fp32)."""
    _require(x, torch.bfloat16, "x")
    rows, cols = x.shape
    out = empty_nvfp4(rows, cols, x.device) if out is None else out
    _check("nvfp4_quantize_with_scale", lib().nvfp4_quantize_with_scale(
        x.data_ptr(), rows, cols, s_enc.data_ptr(), out.q.data_ptr(), out.sf.data_ptr(),
        out.s_dec.data_ptr(), _stream(stream)))
    return out


def quantize_one_pass(x: torch.Tensor, amax_prev: torch.Tensor, amax_out: torch.Tensor,
                      out: NVFP4Tensor | None = None, stream=None) -> NVFP4Tensor:
    """One pass over x with the tensor scale derived from an earlier amax
    (amax_prev, device fp32); writes this tensor's amax into amax_out (a
    different device fp32) for the next call."""
    _require(x, torch.bfloat16, "x")
    rows, cols = x.shape
    out = empty_nvfp4(rows, cols, x.device) if out is None else out
    _check("nvfp4_quantize_one_pass", lib().nvfp4_quantize_one_pass(
        x.data_ptr(), rows, cols, amax_prev.data_ptr(), out.q.data_ptr(), out.sf.data_ptr(),
        out.s_dec.data_ptr(), amax_out.data_ptr(), _stream(stream)))
    return out


_dyn_workspaces: dict = {}


def dynamic_workspace(device=None) -> torch.Tensor:
    """A zero-filled workspace for nvfp4_quantize_dynamic (one per device,
    shared by calls on one stream; give concurrent streams their own)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    ws = _dyn_workspaces.get(dev)
    if ws is None:
        n = int(lib().nvfp4_quantize_dynamic_workspace_bytes())
        ws = torch.zeros((n + 15) // 16 * 16, dtype=torch.uint8, device=dev)
        _dyn_workspaces[dev] = ws
    return ws


def quantize_dynamic(x: torch.Tensor, out: NVFP4Tensor | None = None,
                     amax: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                     stream=None) -> NVFP4Tensor:
    """Per-call activation path in one launch: amax, S_enc, block quantize."""
    _require(x, torch.bfloat16, "x")
    rows, cols = x.shape
    out = empty_nvfp4(rows, cols, x.device) if out is None else out
    ws = dynamic_workspace(x.device) if workspace is None else workspace
    _check("nvfp4_quantize_dynamic", lib().nvfp4_quantize_dynamic(
        x.data_ptr(), rows, cols, out.q.data_ptr(), out.sf.data_ptr(), out.s_dec.data_ptr(),
        _ptr(amax), ws.data_ptr(), _stream(stream)))
    return out


def quantize_rowwise(x: torch.Tensor, out: NVFP4Tensor | None = None,
                     amax_rows: torch.Tensor | None = None, stream=None) -> NVFP4Tensor:
    """Per-token activation scales: each row quantized with its own tensor
    scale 2688 / amax(row); out.s_dec holds one decode scale per row."""
    _require(x, torch.bfloat16, "x")
    rows, cols = x.shape
    out = empty_nvfp4(rows, cols, x.device, row_scales=True) if out is None else out
    if out.s_dec.numel() != rows:
        raise ValueError("out.s_dec must hold one scale per row")
    _check("nvfp4_quantize_rowwise", lib().nvfp4_quantize_rowwise(
        x.data_ptr(), rows, cols, out.q.data_ptr(), out.sf.data_ptr(), out.s_dec.data_ptr(),
        _ptr(amax_rows), _stream(stream)))
    return out


@dataclass
class FusedQuant:
    """Fused next-layer quantization outputs of a GEMM.  out is a complete
    NVFP4Tensor afterwards (out.s_dec = 1/s_enc is written by the GEMM), so it
    can feed the next GEMM directly."""
    s_enc: torch.Tensor           # fp32 [1], read
    out: NVFP4Tensor              # q [M, N/2], sf tiled, s_dec written
    amax: torch.Tensor | None     # fp32 [1], written with max|Y|
    activation: int = ACT_NONE    # ACT_GELU: Y = bf16(GELU(alpha * acc))


def gemm(a: NVFP4Tensor, b: NVFP4Tensor, y: torch.Tensor | None = None,
         fused: FusedQuant | None = None, want_y: bool = True, stream=None) -> torch.Tensor | None:
    """Y[M,N] = A[M,K] . B[N,K]^T on tcgen05 block-scaled FP4 tensor cores."""
    M, K = a.rows, a.cols
    N = b.rows
    if b.cols != K:
        raise ValueError("K mismatch")
    if y is None and want_y:
        y = torch.empty(M, N, dtype=torch.bfloat16, device=a.q.device)
    fo = None
    if fused is not None:
        fo = FusedOut(fused.s_enc.data_ptr(), fused.out.q.data_ptr(), fused.out.sf.data_ptr(),
                      _ptr(fused.amax), fused.out.s_dec.data_ptr(), int(fused.activation))
    if b.s_dec.numel() != 1:
        raise ValueError("per-row scales are supported for A (activations) only")
    row_scaled = a.s_dec.numel() != 1
    if row_scaled and a.s_dec.numel() != M:
        raise ValueError("a.s_dec must hold 1 or M decode scales")
    fn = lib().nvfp4_gemm_rowscale if row_scaled else lib().nvfp4_gemm
    _check("nvfp4_gemm", fn(
        a.q.data_ptr(), a.sf.data_ptr(), a.s_dec.data_ptr(), b.q.data_ptr(), b.sf.data_ptr(),
        b.s_dec.data_ptr(), M, N, K, _ptr(y), ctypes.byref(fo) if fo is not None else None,
        _stream(stream)))
    return y


@dataclass
class FP8Tensor:
    """The FP8 variant's quantized [rows, cols] tensor: E4M3 codes and one
    decode scale."""
    q: torch.Tensor       # uint8 [rows, cols]
    s_dec: torch.Tensor   # float32 [1] = 1 / S_enc = amax / 448
    rows: int
    cols: int


def quantize_fp8(x: torch.Tensor, amax: torch.Tensor | None = None,
                 out: FP8Tensor | None = None, stream=None) -> FP8Tensor:
    """FP8 (E4M3) with one FP32 per-tensor scale 448 / amax; amax computed
    here (dynamic) unless given (static)."""
    _require(x, torch.bfloat16, "x")
    rows, cols = x.shape
    amax = tensor_amax(x, stream=stream) if amax is None else amax
    if out is None:
        out = FP8Tensor(torch.empty(rows, cols, dtype=torch.uint8, device=x.device),
                        torch.empty(1, dtype=torch.float32, device=x.device), rows, cols)
    _check("nvfp4_fp8_quantize", lib().nvfp4_fp8_quantize(
        x.data_ptr(), rows, cols, amax.data_ptr(), out.q.data_ptr(), out.s_dec.data_ptr(),
        _stream(stream)))
    return out


def gemm_fp8(a: FP8Tensor, b: FP8Tensor, y: torch.Tensor | None = None,
             fused: FusedQuant | None = None, want_y: bool = True, stream=None):
    """Y[M,N] = A[M,K] . B[N,K]^T on tcgen05 FP8 (E4M3) tensor cores."""
    M, K, N = a.rows, a.cols, b.rows
    if b.cols != K:
        raise ValueError("K mismatch")
    if y is None and want_y:
        y = torch.empty(M, N, dtype=torch.bfloat16, device=a.q.device)
    fo = None
    if fused is not None:
        fo = FusedOut(fused.s_enc.data_ptr(), fused.out.q.data_ptr(), fused.out.sf.data_ptr(),
                      _ptr(fused.amax), fused.out.s_dec.data_ptr(), int(fused.activation))
    _check("nvfp4_fp8_gemm", lib().nvfp4_fp8_gemm(
        a.q.data_ptr(), a.s_dec.data_ptr(), b.q.data_ptr(), b.s_dec.data_ptr(), M, N, K, _ptr(y),
        ctypes.byref(fo) if fo is not None else None, _stream(stream)))
    return y


class FP8Linear:
    """nn.Linear-shaped FP8 variant: weights quantized once (static scale),
    activations with a dynamic per-tensor scale on every call."""

    def __init__(self, weight: torch.Tensor):
        _require(weight, torch.bfloat16, "weight")
        self.N, self.K = weight.shape
        self.w = quantize_fp8(weight)

    def __call__(self, x: torch.Tensor, y: torch.Tensor | None = None,
                 fused: FusedQuant | None = None, want_y: bool = True):
        return gemm_fp8(quantize_fp8(x), self.w, y, fused, want_y)


SELFTEST_TAG = 90


def selftest_wait_timeout(timeout_us: int = 50_000, stream=None) -> None:
    """Failure-detection self-test: a kernel whose bounded wait can never be
    satisfied gives up after timeout_us; read the result with device_error()."""
    _check("nvfp4_selftest_wait_timeout",
           lib().nvfp4_selftest_wait_timeout(int(timeout_us), _stream(stream)))


class NVFP4Linear:
    """An nn.Linear-shaped NVFP4 layer: weights quantized once with a static
    per-tensor scale (from the weight amax, or a given one), activations
    quantized dynamically on every call."""

    def __init__(self, weight: torch.Tensor, w_amax: torch.Tensor | None = None):
        _require(weight, torch.bfloat16, "weight")
        self.N, self.K = weight.shape
        amax = tensor_amax(weight) if w_amax is None else w_amax
        self.w = quantize(weight, amax)
        self._x = None

    def _xbuf(self, M: int, device) -> tuple[NVFP4Tensor, torch.Tensor]:
        if self._x is None or self._x[0].rows != M:
            self._x = (empty_nvfp4(M, self.K, device),
                       torch.empty(1, dtype=torch.float32, device=device))
        return self._x

    def __call__(self, x: torch.Tensor, y: torch.Tensor | None = None,
                 fused: FusedQuant | None = None, want_y: bool = True) -> torch.Tensor | None:
        xq, amax = self._xbuf(x.shape[0], x.device)
        quantize_dynamic(x, xq, amax)
        return gemm(xq, self.w, y, fused, want_y)

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor, ws: dict,
                     stream=None, single_launch: bool = True) -> None:
        """Host bf16 X -> host bf16 Y through nvfp4_linear_host (copies included).
        single_launch=False passes no dynamic-quantize workspace, so the call
        quantizes X with nvfp4_tensor_amax + nvfp4_quantize."""
        M = x_host.shape[0]
        dyn = ws.get("dyn")
        if dyn is None:
            dyn = dynamic_workspace(ws["x"].device)
        w = LinearWorkspace(ws["x"].data_ptr(), ws["xq"].data_ptr(), ws["xsf"].data_ptr(),
                            ws["amax"].data_ptr(), ws["s_dec"].data_ptr(), ws["y"].data_ptr(),
                            dyn.data_ptr() if single_launch else None)
        _check("nvfp4_linear_host", lib().nvfp4_linear_host(
            x_host.data_ptr(), M, self.K, self.w.q.data_ptr(), self.w.sf.data_ptr(),
            self.w.s_dec.data_ptr(), self.N, y_host.data_ptr(), ctypes.byref(w),
            _stream(stream)))

    def host_workspace(self, M: int, device=None) -> dict:
        """Device buffers for forward_host, including a dynamic-quantize
        workspace of its own, so calls with different workspaces may run on
        different streams at the same time."""
        dev = torch.device("cuda") if device is None else device
        n = int(lib().nvfp4_quantize_dynamic_workspace_bytes())
        return {"dyn": torch.zeros((n + 15) // 16 * 16, dtype=torch.uint8, device=dev),
                "x": torch.empty(M, self.K, dtype=torch.bfloat16, device=dev),
                "xq": torch.empty(M, self.K // 2, dtype=torch.uint8, device=dev),
                "xsf": torch.empty(sf_bytes(M, self.K), dtype=torch.uint8, device=dev),
                "amax": torch.empty(1, dtype=torch.float32, device=dev),
                "s_dec": torch.empty(1, dtype=torch.float32, device=dev),
                "y": torch.empty(M, self.N, dtype=torch.bfloat16, device=dev)}


def device_error() -> tuple[int, int]:
    """(code, detail) of the device error word, cleared on read (synchronises)."""
    c, d = ctypes.c_int(0), ctypes.c_int(0)
    _check("nvfp4_device_error", lib().nvfp4_device_error(ctypes.byref(c), ctypes.byref(d)))
    return c.value, d.value


def status_string(status: int) -> str:
    return lib().nvfp4_status_string(status).decode()
