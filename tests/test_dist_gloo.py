"""The multi-process (N > 1) bench plumbing on CPU with gloo, world size 2:
max-over-ranks timing, whole-job aggregation of replicas, and rank-0-only
output of the reference arm."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist = bench.init_dist(world, "gloo")
    dev = torch.device("cpu")
    t = bench.max_over_ranks(1.5 + rank, dist, dev)       # rank 1 is the slow one
    bench.barrier(dist, dev)
    v = bench.aggregate(per_rank_units=10.0, world=world, max_seconds=t)
    out[rank] = (t, v, bench.dist_env())
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_timing_and_aggregation():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        t, v, env = out[r]
        assert t == 2.5                 # the max over ranks, on every rank
        assert v == pytest.approx(10.0 * 2 / 2.5)
        assert env == (r, world, r)


def test_single_process_defaults(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    import bench
    assert bench.dist_env() == (0, 1, 0)
    assert bench.init_dist(1, "gloo") is None
    assert bench.max_over_ranks(3.0, None, torch.device("cpu")) == 3.0
    assert bench.aggregate(5.0, 1, 2.0) == 2.5


def test_reference_arm_only_rank0_prints(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    import bench
    assert bench.reference_arm(bench.argparse.Namespace(
        workload="tiny_linear", warmup=1, steps=1, cpu_seconds=0.1)) is None


def test_reference_arm_rank0_line(monkeypatch):
    """Rank 0 of the reference arm times the oracle and fills the contract's
    keys (impl, cpu_baseline, e2e with zero copy bytes)."""
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    import bench
    line = bench.reference_arm(bench.argparse.Namespace(
        workload="tiny_linear", warmup=1, steps=2, cpu_seconds=0.2))
    assert line["impl"] == "reference" and line["steps"] == 2
    assert line["value"] > 0 and line["unit"] == bench.UNIT
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["e2e"]["value"] == line["value"]


def test_cpu_baseline_sample_is_bounded():
    import bench
    from workloads import WORKLOADS
    t0 = bench.time.perf_counter()
    cb = bench.cpu_baseline(WORKLOADS["tiny_linear"], 0.3)
    assert bench.time.perf_counter() - t0 < 30
    assert cb["seconds"] >= 0.3 and cb["value"] > 0 and "passes of" in cb["sample"]


def _shard_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import numpy as np
    import torch.distributed as dist

    import oracle
    from nvfp4_block_scaled_19_b200.sharded import all_reduce_max, shard_rows
    from workloads import bf16_bits, draw_x
    dist.init_process_group("gloo", rank=rank, world_size=world)
    M, K = 301, 256
    x = draw_x("lognormal_channels", M, K, seed=7, index=0)
    s, e = shard_rows(M, world, rank)
    xb = bf16_bits(x[s:e])
    amax = torch.tensor([float(oracle.tensor_amax(xb))], dtype=torch.float32)
    all_reduce_max(amax)
    q, sf = oracle.quantize(xb, e - s, K, oracle.tensor_scale(np.float32(amax.item())))
    out[rank] = (s, e, float(amax.item()), q, sf)
    dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_token_shards_quantize_like_one_tensor():
    """Two gloo ranks each take a slice of the tokens, reduce their amax with
    the package's all-reduce(MAX) and quantize their rows (with the oracle):
    every row's codes and block scales are those of the whole tensor's
    quantization, and the reduced amax is the whole tensor's."""
    import numpy as np

    import oracle
    from workloads import bf16_bits, draw_x
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_shard_worker, args=(world, port, out), nprocs=world, join=True)
    M, K = 301, 256
    kb = K // 16
    x = draw_x("lognormal_channels", M, K, seed=7, index=0)
    fq, fsf, _, famax = oracle.quantize_dynamic(bf16_bits(x), M, K)
    covered = 0
    for r in range(world):
        s, e, amax, q, sf = out[r]
        assert np.float32(amax) == famax
        assert np.array_equal(q, fq[s:e])
        for row in range(s, e):
            for c in range(kb):
                assert sf[oracle.sf_offset(row - s, c, kb)] == fsf[oracle.sf_offset(row, c, kb)]
        covered += e - s
    assert covered == M


def test_shard_rows_partition():
    from nvfp4_block_scaled_19_b200.sharded import shard_rows
    for rows in (0, 1, 7, 4608, 16897):
        for world in (1, 2, 3, 8):
            spans = [shard_rows(rows, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == rows
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [e - s for s, e in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_rows(10, 2, 2)
