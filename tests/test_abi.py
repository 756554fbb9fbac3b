"""The C-ABI library loads, exports every function include/nvfp4.h declares,
and rejects bad arguments before touching a device (runs without a GPU)."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4.h")


@pytest.fixture(scope="module")
def L():
    from nvfp4_block_scaled_19_b200 import build
    build.build()
    import nvfp4_block_scaled_19_b200 as nv
    return nv.lib()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(nvfp4_[a-z0-9_]+)\s*\(",
                       text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ("nvfp4_tensor_amax", "nvfp4_quantize", "nvfp4_quantize_with_scale", "nvfp4_gemm",
              "nvfp4_packed_bytes", "nvfp4_sf_bytes", "nvfp4_status_string",
              "nvfp4_linear_host", "nvfp4_device_error", "nvfp4_quantize_dynamic",
              "nvfp4_quantize_dynamic_workspace_bytes", "nvfp4_quantize_dynamic_noalloc",
              "nvfp4_quantize_rowwise", "nvfp4_gemm_rowscale"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for n in _declared_functions():
        assert hasattr(L, n), n


def test_sizes_and_strings(L, orc):
    for rows, cols in [(1, 16), (128, 512), (130, 48), (4608, 3072), (7, 80)]:
        assert L.nvfp4_packed_bytes(rows, cols) == rows * cols // 2
        assert L.nvfp4_sf_bytes(rows, cols) == orc.sf_bytes(rows, cols)
    for s in range(6):
        assert L.nvfp4_status_string(s)
    assert L.nvfp4_status_string(99) == b"unknown status"


def _dev_buf(n=4096):
    # Any 16-byte aligned host address stands in for a device pointer: these
    # calls must fail on their arguments before anything reaches a device.
    return ctypes.create_string_buffer(n + 16)


def _aligned(buf, off=0):
    a = ctypes.addressof(buf)
    return (a + 15) // 16 * 16 + off


def test_invalid_arguments_rejected_first(L):
    b = _dev_buf()
    p = _aligned(b)
    # quantize: cols % 16 != 0, negative rows, null outputs, misaligned input
    assert L.nvfp4_quantize(p, 4, 24, p, p, p, None, None) == 1
    assert L.nvfp4_quantize(p, -1, 32, p, p, p, None, None) == 1
    assert L.nvfp4_quantize(p, 4, 32, p, None, p, None, None) == 1
    assert L.nvfp4_quantize(p + 2, 4, 32, p, p, p, None, None) == 2
    assert L.nvfp4_quantize_with_scale(p, 4, 0, p, p, p, None, None) == 1
    # an empty tensor's arrays may be NULL (not an argument error); its scale may not
    assert L.nvfp4_quantize(None, 0, 32, p, None, None, None, None) != 1
    assert L.nvfp4_quantize(None, 0, 32, None, None, None, None, None) == 1
    assert L.nvfp4_quantize(None, 4, 32, p, p, p, None, None) == 1
    # amax
    assert L.nvfp4_tensor_amax(p, -5, p, None) == 1
    assert L.nvfp4_tensor_amax(p, 8, None, None) == 1
    assert L.nvfp4_tensor_amax(p + 8, 8, p, None) == 2
    # gemm: K % 64, N % 8, M < 1, no output at all, misaligned operand
    g = L.nvfp4_gemm
    assert g(p, p, p, p, p, p, 128, 128, 96, p, None, None) == 1
    assert g(p, p, p, p, p, p, 128, 12, 128, p, None, None) == 1
    assert g(p, p, p, p, p, p, 0, 128, 128, p, None, None) == 1
    assert g(p, p, p, p, p, p, 128, 128, 128, None, None, None) == 1
    assert g(p + 4, p, p, p, p, p, 128, 128, 128, p, None, None) == 2
    import nvfp4_block_scaled_19_b200 as nv
    bad = nv.FusedOut(p, None, p, None)       # fused output without yq
    assert g(p, p, p, p, p, p, 128, 128, 128, p, ctypes.byref(bad), None) == 1
    ok = nv.FusedOut(p, p, p, None)
    assert g(p, p, p, p, p, p, 128, 120, 128, p, ctypes.byref(ok), None) == 1  # N % 16
    act = nv.FusedOut(p, p, p, None, None, 2)  # no such activation
    assert g(p, p, p, p, p, p, 128, 128, 128, p, ctypes.byref(act), None) == 1
    assert ctypes.sizeof(nv.FusedOut) == 48   # five pointers + int, padded (header layout)
    assert L.nvfp4_device_error(None, None) == 1
    qd = L.nvfp4_quantize_dynamic
    assert qd(p, 4, 24, p, p, None, None, p, None) == 1         # cols % 16
    assert qd(p, 4, 32, p, p, None, None, None, None) == 1      # no workspace
    assert qd(p, 4, 32, p, p, None, None, p + 4, None) == 2     # misaligned workspace
    assert L.nvfp4_quantize_dynamic_workspace_bytes() == 32
    qr = L.nvfp4_quantize_rowwise
    assert qr(p, 4, 24, p, p, p, None, None) == 1              # cols % 16
    assert qr(p, 4, 32, p, p, None, None, None) == 1           # no per-row scales
    assert qr(p, 4, 32, p, p, p + 2, None, None) == 2          # misaligned scales
    gr = L.nvfp4_gemm_rowscale
    assert gr(p, p, p, p, p, p, 128, 128, 96, p, None, None) == 1     # K % 64
    assert gr(p, p, p, p, p, p, 128, 128, 128, None, None, None) == 1


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device answer")
def test_valid_call_without_device_reports_unsupported(L):
    b = _dev_buf()
    p = _aligned(b)
    assert L.nvfp4_quantize(p, 4, 32, p, p, p, None, None) == 3
    assert L.nvfp4_gemm(p, p, p, p, p, p, 128, 128, 128, p, None, None) == 3


def test_noalloc_refuses_exactly_what_quantize_dynamic_refuses(L):
    """The no-allocation entry point answers every call that the entry point
    with a caller workspace answers with an argument error the same way, and
    before anything is enqueued (no device is touched here)."""
    b = _dev_buf()
    p = _aligned(b)
    ws = _aligned(b, 2048)
    qd, na = L.nvfp4_quantize_dynamic, L.nvfp4_quantize_dynamic_noalloc
    cases = [
        (None, 0, 32, None, None),           # empty tensor, NULL arrays: allowed
        (p, 0, 32, p, p),                    # empty tensor
        (p, 4, 24, p, p),                    # cols % 16 != 0
        (p, -1, 32, p, p),                   # negative rows
        (p, 4, 0, p, p),                     # no columns
        (p, (1 << 40) // 32 + 1, 32, p, p),  # rows * cols above 2^40
        (None, 4, 32, p, p),                 # NULL input with rows
        (p, 4, 32, None, p),                 # NULL codes
        (p, 4, 32, p, None),                 # NULL scales
        (p + 2, 4, 32, p, p),                # misaligned input
        (p, 4, 32, p + 8, p),                # misaligned codes
        (p, 4, 32, p, p + 4),                # misaligned scales
        (p, 4, 32, p, p),                    # valid
    ]
    for x, rows, cols, q, sf in cases:
        a = qd(x, rows, cols, q, sf, None, None, ws, None)
        n = na(x, rows, cols, q, sf, None, None, None)
        assert a == n, (rows, cols, a, n)
    assert qd(p, (1 << 40) // 32 + 1, 32, p, p, None, None, ws, None) == 1
    assert na(p + 2, 4, 32, p, p, None, None, None) == 2
