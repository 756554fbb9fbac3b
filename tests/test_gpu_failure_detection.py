"""Failure detection on the GPU without a fault: a wait that nothing will
satisfy (a barrier whose phase never completes) runs out through the
library's own bounded wait; the kernel records NVFP4_ERR_TIMEOUT with its
tag, returns normally, the host reads the status through
nvfp4_device_error, and the context keeps working."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import TOL, require_cuda
from workloads import bf16_bits, draw_w, draw_x

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    return require_cuda()


def test_wait_timeout_is_reported_and_context_survives(nv):
    assert nv.device_error() == (0, 0)
    nv.selftest_wait_timeout(50_000)          # 50 ms
    torch.cuda.synchronize()
    assert nv.device_error() == (5, nv.SELFTEST_TAG)
    assert nv.device_error() == (0, 0)        # reading clears it
    # The context still runs the real path correctly.
    x = draw_x("lognormal_channels", 300, 512, seed=31, index=0)
    w = draw_w(512, 512, None, seed=31, index=1)
    y = nv.NVFP4Linear(w.cuda())(x.cuda())
    torch.cuda.synchronize()
    assert nv.device_error() == (0, 0)
    aq, asf, asd, _ = oracle.quantize_dynamic(bf16_bits(x), 300, 512)
    bq, bsf, bsd, _ = oracle.quantize_dynamic(bf16_bits(w), 512, 512)
    ok, worst = oracle.gemm_tolerance_ok(y.float().cpu().numpy(),
                                         oracle.gemm(aq, asf, asd, bq, bsf, bsd, 300, 512, 512),
                                         TOL)
    assert ok, worst


def test_selftest_rejects_bad_timeouts(nv):
    for bad in (0, -5, 3_000_000):
        with pytest.raises(nv.NVFP4Error):
            nv.selftest_wait_timeout(bad)
