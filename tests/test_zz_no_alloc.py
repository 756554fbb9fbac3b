"""nvfp4_quantize_dynamic_noalloc: the quantize entry point for callers that
cannot allocate device memory (its workspace lives in a static array inside
the library).  Called through the C ABI twice in a row, its outputs must
equal those of nvfp4_quantize_dynamic with a caller workspace, bit for bit
(the tolerance of every quantization test here).  Kept in a file collected
last so that a failure here leaves the rest of the suite already run."""
import ctypes

import numpy as np
import pytest
import torch

from gpu_common import require_cuda
from workloads import draw_x

pytestmark = pytest.mark.gpu


def _noalloc(nv):
    f = nv.lib().nvfp4_quantize_dynamic_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    return f


def test_noalloc_matches_workspace_entry_point_twice():
    nv = require_cuda()
    f = _noalloc(nv)
    stream = torch.cuda.current_stream().cuda_stream
    # Two calls in a row, different shapes and scales: the second must not see
    # anything the first left in the shared scratch.
    for call, (rows, cols, scale) in enumerate([(4608, 3072, 1.0), (130, 272, 1e-3)]):
        x = (draw_x("lognormal_channels", rows, cols, seed=500 + call, index=0).float() *
             scale).to(torch.bfloat16).cuda()
        # Existing entry point with its own zero-filled workspace.
        ws = torch.zeros(nv.lib().nvfp4_quantize_dynamic_workspace_bytes(), dtype=torch.uint8,
                         device="cuda")
        ref_amax = torch.empty(1, device="cuda")
        ref = nv.quantize_dynamic(x, amax=ref_amax, workspace=ws)
        # The no-allocation entry point into fresh output buffers.
        out = nv.empty_nvfp4(rows, cols)
        amax = torch.full((1,), -1.0, device="cuda")
        status = f(x.data_ptr(), rows, cols, out.q.data_ptr(), out.sf.data_ptr(),
                   out.s_dec.data_ptr(), amax.data_ptr(), stream)
        assert status == 0, nv.status_string(status)
        torch.cuda.synchronize()
        code, tag = nv.device_error()
        assert code == 0, f"device wait timed out (tag {tag})"
        assert np.array_equal(out.q.cpu().numpy(), ref.q.cpu().numpy()), f"call {call}: codes"
        assert np.array_equal(out.sf.cpu().numpy(), ref.sf.cpu().numpy()), f"call {call}: scales"
        assert out.s_dec.item() == ref.s_dec.item(), f"call {call}: decode scale"
        assert amax.item() == ref_amax.item(), f"call {call}: amax"
