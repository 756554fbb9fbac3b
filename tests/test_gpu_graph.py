"""A whole step of the path captured in a CUDA graph replays bit for bit like
eager execution: dynamic quantize (whose grid barrier keeps its generation
word in device memory across replays), the FFN up-projection with the fused
GELU + quantize epilogue, and the down-projection on its codes."""
import pytest
import torch

from gpu_common import require_cuda
from workloads import draw_w, draw_x

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    return require_cuda()


def test_graph_replay_matches_eager(nv):
    M, K, H = 640, 512, 1024
    x = draw_x("lognormal_channels", M, K, seed=21, index=0).cuda()
    up = nv.NVFP4Linear(draw_w(H, K, None, seed=21, index=1).cuda())
    down = nv.NVFP4Linear(draw_w(K, H, None, seed=21, index=2).cuda())
    xq = nv.empty_nvfp4(M, K)
    amax = torch.empty(1, device="cuda")
    fq = nv.FusedQuant(torch.tensor([2688.0 / 12.0], device="cuda"), nv.empty_nvfp4(M, H),
                       torch.empty(1, device="cuda"), nv.ACT_GELU)
    y = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    ws = nv.dynamic_workspace(x.device)

    def step():
        nv.quantize_dynamic(x, xq, amax, ws)
        nv.gemm(xq, up.w, None, fq, want_y=False)
        nv.gemm(fq.out, down.w, y)

    step()
    torch.cuda.synchronize()
    want = [t.clone() for t in (xq.q, xq.sf, xq.s_dec, amax, fq.out.q, fq.out.sf, fq.out.s_dec,
                                fq.amax, y)]
    for t in (xq.q, xq.sf, fq.out.q, fq.out.sf, y):
        t.zero_()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        step()                       # warm-up on the capture stream
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            step()
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        for t in (xq.q, xq.sf, fq.out.q, fq.out.sf, y):
            t.zero_()
        g.replay()
        torch.cuda.synchronize()
        code, detail = nv.device_error()
        assert code == 0, f"device wait timed out (tag {detail})"
        got = (xq.q, xq.sf, xq.s_dec, amax, fq.out.q, fq.out.sf, fq.out.s_dec, fq.amax, y)
        for a, b in zip(got, want):
            assert torch.equal(a, b)
    del g
