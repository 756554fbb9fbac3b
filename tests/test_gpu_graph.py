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


def test_block_chain_graph_vs_oracle(nv, orc):
    """The 2048^2 DiT block linear chain with guidance batch 2 (M = 33792:
    QKV, attn-out, FFN up, FFN down with the fused next-layer quantize), each
    layer's input quantized on the GPU inside the step, captured once in a
    CUDA graph and replayed twice with every output cleared before each
    replay.  After the last replay, seeded rows of every layer's Y and of the
    fused codes are checked against the oracle, which computes each layer from
    its bf16 X in fp64 and never sees a GPU value."""
    import numpy as np

    import oracle
    from gpu_common import TOL, bf16_from_fp64, check_fused_blocks
    from workloads import WORKLOADS, bf16_bits, layer_inputs

    w = WORKLOADS["block_chain_2048"]
    M = w.M
    s_enc_y = np.float32(2688.0) / np.float32(8.0)
    ws = nv.dynamic_workspace(torch.device("cuda"))
    state = []
    for li, l in enumerate(w.layers):
        x, wt = layer_inputs(w, li)
        fq = None
        if l.fused_out:
            fq = nv.FusedQuant(torch.tensor([float(s_enc_y)], device="cuda"),
                               nv.empty_nvfp4(M, l.N), torch.empty(1, device="cuda"))
        state.append(dict(x_cpu=x, w_cpu=wt, x=x.cuda(), lin=nv.NVFP4Linear(wt.cuda()),
                          xq=nv.empty_nvfp4(M, l.K), amax=torch.empty(1, device="cuda"),
                          y=torch.empty(M, l.N, dtype=torch.bfloat16, device="cuda"), fq=fq))

    def step():
        for s in state:
            nv.quantize_dynamic(s["x"], s["xq"], s["amax"], ws)
            nv.gemm(s["xq"], s["lin"].w, s["y"], s["fq"])

    def outputs():
        out = []
        for s in state:
            out += [s["xq"].q, s["xq"].sf, s["y"]]
            if s["fq"] is not None:
                out += [s["fq"].out.q, s["fq"].out.sf]
        return out

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        step()
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=side):
            step()
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(2):
        for t in outputs():
            t.zero_()
        g.replay()
        torch.cuda.synchronize()
        code, detail = nv.device_error()
        assert code == 0, f"device wait timed out (tag {detail})"
    del g

    rng = np.random.default_rng(45)
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 40, replace=False)]))
    rows_t = torch.from_numpy(rows).cuda()
    for l, s in zip(w.layers, state):
        x, wt = s["x_cpu"], s["w_cpu"]
        aq, asf, asd, amax = oracle.quantize_dynamic(bf16_bits(x), M, l.K)
        assert np.float32(s["amax"].item()) == amax, l.name
        bq, bsf, bsd, _ = oracle.quantize_dynamic(bf16_bits(wt), l.N, l.K)
        ref = oracle.gemm(aq, asf, asd, bq, bsf, bsd, M, l.N, l.K, rows=rows)
        yg = s["y"][rows_t].float().cpu().numpy()
        ok, worst = oracle.gemm_tolerance_ok(yg, ref, TOL)
        assert ok, f"{l.name}: worst |err|/bound = {worst:.3f}"
        # the step's own quantized X on the sampled rows: bit-exact
        kb = l.K // 16
        sf_idx = [orc.sf_offset(int(r), c, kb) for r in rows for c in range(kb)]
        assert np.array_equal(s["xq"].q[rows_t].cpu().numpy(), aq[rows]), l.name
        assert np.array_equal(s["xq"].sf.cpu().numpy()[sf_idx], asf[sf_idx]), l.name
        if s["fq"] is not None:
            check_fused_blocks(orc, yg, bf16_from_fp64(ref), s["fq"].out.q.cpu().numpy(),
                               s["fq"].out.sf.cpu().numpy(), rows, s_enc_y,
                               f"{l.name} fused", 0.9)
        s.clear()
        torch.cuda.empty_cache()
