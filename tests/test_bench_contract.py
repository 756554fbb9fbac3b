"""bench.py's JSON line keeps the contract: the keys and their meaning on
both arms (the oracle's reference arm runs here, the GPU arm on a B200)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BASE_KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
             "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"}


def _run(args, timeout):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                       capture_output=True, text=True, timeout=timeout)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


def test_reference_arm_line():
    d = _run(["--impl", "reference", "--steps", "2", "--warmup", "1", "--cpu-seconds", "0.5"], 300)
    assert BASE_KEYS <= set(d)
    assert d["impl"] == "reference" and d["steps"] == 2 and d["n_gpus"] == 1
    assert d["config"]["workload"] == "ffn_2048" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


@pytest.mark.gpu
def test_gpu_arm_line():
    d = _run(["--steps", "20", "--warmup", "3", "--no-cpu-baseline", "--e2e-steps", "2"], 600)
    assert BASE_KEYS <= set(d)
    assert d["n_gpus"] == 1 and d["steps"] == 20 and d["warmup"] == 3
    assert d["higher_is_better"] is True and d["scaling"] == "weak"
    # The default step: the 2048^2 FFN GEMMs (up, then down with the fused
    # next-layer quantize), each with the dynamic quantize of its input.
    assert d["config"]["workload"] == "ffn_2048"
    M, H, F = 16896, 3072, 12288
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert 0 < r["frac"] < 1.5 and abs(r["achieved"] / r["peak"] - r["frac"]) < 1e-3
    assert r["traffic"] is None or r["traffic"] > 0
    # 20 steps of ~0.8 ms: a short run, measured against the burst figure.
    assert d["pct_fp4_peak"]["regime"] == "burst" and "burst (" in r["peak_source"]
    assert abs(d["pct_fp4_peak"]["of_4x_measured_bf16_burst"] * r["peak"] - d["value"]) < 1.0
    e = d["e2e"]
    assert e["h2d_bytes_per_step"] == 2 * M * (H + F)
    assert e["d2h_bytes_per_step"] == 2 * M * (F + H)
    assert 0 < e["value"] < d["value"]
    assert d["gpu_launches"] == 4 * 20
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(d["clocks"])
    # ms_per_step is the evented step; value is the work of the step over it
    flops = 2 * M * F * H * 2
    assert abs(flops / (d["ms_per_step"] * 1e-3) / 1e12 - d["value"]) < 0.01 * d["value"]
    pl = d["per_layer"]
    assert [p["layer"] for p in pl] == ["ffn_up", "ffn_down"]
    assert abs(sum(p["quantize_us"] + p["gemm_us"] for p in pl) - d["ms_per_step"] * 1e3) \
        < 0.01 * d["ms_per_step"] * 1e3
    for p in pl:
        assert 0 < p["gemm_frac"] < 1.5 and p["tflops_incl_quantize"] < p["gemm_tflops"]
    m = d["ffn_down_modes"]
    assert {"dynamic", "stale_scale", "fused_producer"} <= set(m)
    assert m["stale_scale"]["quantize_us"] < m["dynamic"]["quantize_us"]
    assert m["fused_producer"]["block_tflops_incl_quantize"] > 0


class _L:
    def __init__(self, M, N, K, m_global=None, sharded=False):
        self.M, self.N, self.K = M, N, K
        self.m_global = M if m_global is None else m_global
        self.sharded = sharded
        self.flops = 2 * M * N * K


def test_job_flops_replicas_and_shards():
    import bench
    rep = [_L(4608, 9216, 3072)]
    assert bench.job_flops(rep, 4) == 4 * 2 * 4608 * 9216 * 3072
    shards = [_L(1152, 9216, 3072, m_global=4608, sharded=True)]
    assert bench.job_flops(shards, 4) == 2 * 4608 * 9216 * 3072
    one = [_L(4608, 9216, 3072, m_global=4608, sharded=True)]
    assert bench.job_flops(one, 1) == 2 * 4608 * 9216 * 3072


def test_tensor_peak_follows_the_timed_length():
    # Pool measurements: bf16 1627.8 burst, 1395 sustained; FP4 = 4 x bf16.
    import bench
    short = bench.tensor_peak(4.0, 1627.8, 1395.0, 0.016)
    long = bench.tensor_peak(4.0, 1627.8, 1395.0, 1.6)
    assert short[:2] == (4.0 * 1627.8, "burst")
    assert long[:2] == (4.0 * 1395.0, "sustained")
    edge = bench.tensor_peak(2.0, 1627.8, 1395.0, bench.SUSTAINED_AFTER_S)
    assert edge[:2] == (2.0 * 1395.0, "sustained")
    assert "burst would be" in long[2] and "sustained would be" in short[2]


@pytest.mark.gpu
def test_gpu_arm_token_shards_one_rank():
    d = _run(["--workload", "qkv_1024", "--shard", "tokens", "--steps", "10", "--warmup", "3",
              "--no-cpu-baseline", "--e2e-steps", "2"], 600)
    assert d["scaling"] == "strong" and d["config"]["parallelism"].startswith("tokens x1")
    assert d["gpu_launches"] == 3 * 10      # amax + quantize + GEMM per step
    assert d["value"] > 0 and d["e2e"]["value"] > 0


@pytest.mark.gpu
@pytest.mark.parametrize("mode,launches", [(["--act-scale", "stale"], 2), (["--act-scale", "row"], 2),
                                           (["--variant", "fp8"], 3)])
def test_gpu_arm_variants(mode, launches):
    """The one-pass stale-scale, per-token and FP8 modes print the same line
    (launches per step: quantize kernels + GEMM)."""
    d = _run(mode + ["--workload", "qkv_1024", "--steps", "5", "--warmup", "3",
                     "--no-cpu-baseline", "--e2e-steps", "2"], 600)
    assert BASE_KEYS <= set(d)
    assert d["value"] > 0 and d["gpu_launches"] == launches * 5
    assert d["roofline"]["frac"] > 0 and d["e2e"]["value"] > 0
