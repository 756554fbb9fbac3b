"""GPU: token-sharded quantization (one exchange: the amax all-reduce) gives
every row the codes and block scales of the whole tensor's single-GPU
quantization; the sharded linear layer on one rank is the plain one."""
import socket

import numpy as np
import pytest
import torch

from gpu_common import require_cuda
from workloads import draw_w, draw_x

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    return require_cuda()


def _sf_rows(orc, sf, rows, kb, r0=0):
    return np.array([[sf[orc.sf_offset(r - r0, c, kb)] for c in range(kb)] for r in rows])


@pytest.mark.parametrize("world", [2, 3])
def test_shards_on_one_gpu(nv, orc, world):
    """The shards of one GPU, with torch.maximum standing in for the
    all-reduce: codes, scales and S_dec of every shard match the whole
    tensor's dynamic quantization."""
    from nvfp4_block_scaled_19_b200.sharded import shard_rows
    M, K = 1001, 3072
    kb = K // 16
    x = draw_x("lognormal_channels", M, K, seed=31, index=0).cuda()
    whole = nv.quantize_dynamic(x)
    spans = [shard_rows(M, world, r) for r in range(world)]
    amaxes = [nv.tensor_amax(x[s:e].contiguous()) for s, e in spans]
    g = torch.stack(amaxes).max().reshape(1)
    wq, wsf = whole.q.cpu().numpy(), whole.sf.cpu().numpy()
    rows = np.array([0, 1, 127, 128, 500, 999, 1000])
    for s, e in spans:
        t = nv.quantize(x[s:e].contiguous(), g)
        torch.cuda.synchronize()
        assert np.array_equal(t.q.cpu().numpy(), wq[s:e])
        assert t.s_dec.item() == whole.s_dec.item()
        mine = rows[(rows >= s) & (rows < e)]
        assert np.array_equal(_sf_rows(orc, t.sf.cpu().numpy(), mine, kb, s),
                              _sf_rows(orc, wsf, mine, kb))


def test_sharded_linear_single_rank_group(nv):
    """A one-rank NCCL group: the all-reduce is a real collective call, and
    the sharded layer's quantization and output equal the plain layer's."""
    import torch.distributed as dist

    from nvfp4_block_scaled_19_b200.sharded import ShardedNVFP4Linear, quantize_sharded
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        M, K, N = 640, 1024, 512
        x = draw_x("normal_outliers", M, K, seed=3, index=0).cuda()
        w = draw_w(N, K, None, seed=3, index=1).cuda()
        a = quantize_sharded(x)
        b = nv.quantize_dynamic(x)
        torch.cuda.synchronize()
        assert torch.equal(a.q, b.q) and torch.equal(a.sf, b.sf) and torch.equal(a.s_dec, b.s_dec)
        ys = ShardedNVFP4Linear(w)(x)
        yp = nv.NVFP4Linear(w)(x)
        torch.cuda.synchronize()
        assert torch.equal(ys, yp)
    finally:
        dist.destroy_process_group()
