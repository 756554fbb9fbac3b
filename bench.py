"""Benchmark of the NVFP4 linear-layer hot path on B200.

One step = one pass of the whole per-call path over one batch of synthetic
DiT activations: for every layer of the workload, the single-launch dynamic
NVFP4 quantize of its input (amax, tensor scale, block quantize) and the
block-scaled FP4 GEMM, with the fused next-layer quantize (and activation)
in the GEMM epilogue where the layer feeds one; a layer whose input is the
previous layer's fused output skips the quantize.  Weights are quantized
once, before timing (static scale); a fused output's static tensor scale is
calibrated once from an untimed pass.  The headline metric is NVFP4 GEMM
TFLOP/s including the activation quantize, i.e. 2*M*N*K / (t_quantize +
t_gemm) summed over layers.

Multi-GPU: one process per GPU (torchrun).  By default each rank runs an
independent replica of the workload (the linear layer needs no exchange), so
scaling is weak and the value is the work of all ranks over the max-over-
ranks time.  --shard tokens splits the workload's tokens across the ranks
instead (strong scaling); the one exchange is an all-reduce(MAX) of each
layer input's amax, so every row is quantized as on one GPU.

--impl reference times the CPU oracle (test infrastructure, the only
reference for this path) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from workloads import WORKLOADS, layer_inputs  # noqa: E402

METRIC = "NVFP4 GEMM TFLOPS incl. act quantize (% FP4 peak); quantize GB/s (% HBM)"
UNIT = "TFLOP/s"
DEFAULT_WORKLOAD = "ffn_2048"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Device time of back-to-back steps from which the timed region counts as
# sustained load: the GPU has settled at its power cap (B200, FP4 GEMMs: 20
# steps of the FFN step, ~16 ms, run at the burst clock; 2000 steps, ~1.6 s,
# 12-15% slower), so the roofline takes the sustained bf16 figure there.
SUSTAINED_AFTER_S = 0.5
FP4_PER_BF16 = 4.0      # nominal dense FP4 / dense BF16 (9 / 2.25 PFLOP/s)
FP8_PER_BF16 = 2.0      # nominal dense FP8 / dense BF16 (4.5 / 2.25 PFLOP/s)
NOMINAL_FP4_TFLOPS = 9000.0
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, vendor figure


GEMM_SOURCES = ["gemm.h", "gemm.cu", "gemm_pair.cuh", "gemm_common.cuh", "ptx.cuh",
                "nvfp4_math.cuh"]


def strip_c_comments(text: str) -> str:
    """C/C++ source without its comments, whitespace runs collapsed to one
    space (string and character literals kept as written)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            out.append(" ")
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def gemm_source_hash() -> str:
    """sha256 over the GEMM kernel sources without their comments, in a fixed
    order: ties a profile's counters to the kernel code they were taken on."""
    import hashlib
    h = hashlib.sha256()
    for name in GEMM_SOURCES:
        with open(os.path.join(ROOT, "nvfp4_block_scaled_19_b200", "csrc", name)) as f:
            h.update(strip_c_comments(f.read()).encode())
    return h.hexdigest()


def profile_name(w, layer) -> str:
    """Name under which a layer's GEMM capture is filed in profiles/: the
    single-layer workload the layer's tensors come from, else the workload
    (with the layer's name when the workload has several layers)."""
    if layer.source is not None:
        return layer.source[0]
    return w.name if len(w.layers) == 1 else f"{w.name}_{layer.name}"


def profiled_traffic(name: str) -> tuple[float | None, str]:
    """DRAM bytes per launch of a GEMM from the committed ncu summary
    profiles/gemm_pair_<name>.md, or None when there is none or the kernel
    sources changed after the capture."""
    path = os.path.join(ROOT, "profiles", f"gemm_pair_{name}.md")
    try:
        with open(path) as f:
            kv = dict(l.split(":", 1) for l in f.read().splitlines()
                      if l.startswith(("traffic_bytes_per_launch:", "source_sha256:")))
    except OSError:
        return None, "no ncu summary"
    if kv.get("source_sha256", "").strip() != gemm_source_hash():
        return None, "kernel changed since the ncu capture"
    try:
        return float(kv["traffic_bytes_per_launch"]), os.path.relpath(path, ROOT)
    except (KeyError, ValueError):
        return None, "no traffic line"


def gemm_kernel_name(M: int, N: int) -> str:
    """Which kernel nvfp4_gemm dispatches to (mirrors gemm_kind in csrc/gemm.cu)."""
    if N >= 256 and M > 128:
        return "gemm_pair_kernel (tcgen05.mma cta_group::2 kind::mxf4nvf4, 256x256 tiles)"
    if N >= 256:
        return "gemm_kernel 128x256 (tcgen05.mma kind::mxf4nvf4)"
    return "gemm_kernel 128x128 (tcgen05.mma kind::mxf4nvf4)"


def load_peaks() -> tuple[dict, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------- distributed plumbing

def dist_env() -> tuple[int, int, int]:
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def init_dist(world: int, backend: str):
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value: float, dist, device) -> float:
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist, device) -> None:
    if dist is not None:
        t = torch.zeros(1, device=device)
        dist.all_reduce(t)


def aggregate(per_rank_units: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: units processed by all ranks / max-over-ranks time."""
    return per_rank_units * world / max_seconds


# ----------------------------------------------------------------- clocks

CLOCK_FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
                "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
                "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons (read-only)."""

    def __init__(self, index: int, period_ms: int = 50):
        self.samples: list[tuple[float, list[str]]] = []
        self.proc = None
        self.index = index
        self.period_ms = period_ms
        self.window: tuple[float, float] | None = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={','.join(CLOCK_FIELDS)}",
                 "--format=csv,noheader,nounits", f"-lms={self.period_ms}"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == len(CLOCK_FIELDS):
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        rows = self.samples
        if self.window is not None:
            lo, hi = self.window
            inside = [r for r in rows if lo - 0.06 <= r[0] <= hi + 0.06]
            rows = inside if inside else rows
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1][0]) for r in rows if r[1][0].replace(".", "").isdigit()]
        mx = [float(r[1][1]) for r in rows if r[1][1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[1][4:8]) if v == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows),
                "power_w_max": max((float(r[1][2]) for r in rows
                                    if r[1][2].replace(".", "").isdigit()), default=None)}


# ----------------------------------------------------------------- the GPU arm

class Layer:
    def __init__(self, nv, spec, M, x_cpu, w_cpu, device, row_scales=False, fp8=False,
                 stale=False, m_global=None, sharded=False):
        self.spec = spec
        # Token shards: this rank's M of the workload's m_global rows; its
        # drawn input is quantized with the group's amax (one all-reduce).
        self.m_global = M if m_global is None else m_global
        self.sharded = sharded and not spec.x_from_prev
        self.row_scales = row_scales
        self.fp8 = fp8
        # One-pass quantize with the previous call's amax: two amax words,
        # read one and write the other, swapped every call.
        self.stale = stale and not spec.x_from_prev and not fp8 and not row_scales
        self.amax_pair = [torch.empty(1, dtype=torch.float32, device=device) for _ in range(2)]
        self.calls = 0
        if fp8 and spec.x_from_prev:
            raise ValueError("the FP8 variant takes no NVFP4 fused input")
        self.M, self.K = M, spec.K
        self.N = w_cpu.shape[0]
        self.x_cpu = x_cpu
        self.x = None if x_cpu is None else x_cpu.to(device)
        if fp8:
            self.lin = nv.FP8Linear(w_cpu.to(device))
            self.xq = nv.FP8Tensor(torch.empty(self.M, self.K, dtype=torch.uint8, device=device),
                                   torch.empty(1, dtype=torch.float32, device=device),
                                   self.M, self.K)
        else:
            self.lin = nv.NVFP4Linear(w_cpu.to(device))
            self.xq = (None if spec.x_from_prev
                       else nv.empty_nvfp4(self.M, self.K, device, row_scales=row_scales))
        self.amax = torch.empty(1, dtype=torch.float32, device=device)
        if self.stale:   # the first call's "previous" amax: this tensor's own
            nv.tensor_amax(self.x, self.amax_pair[0])
        self.y = (torch.empty(self.M, self.N, dtype=torch.bfloat16, device=device)
                  if spec.keep_y else None)
        self.fused = None
        if spec.fused_out:
            # Next-layer tensor scale: static; calibrate() replaces this first
            # guess (amax 8) with 2688 / amax of an untimed pass.
            self.fused = nv.FusedQuant(torch.tensor([2688.0 / 8.0], device=device),
                                       nv.empty_nvfp4(self.M, self.N, device),
                                       torch.empty(1, dtype=torch.float32, device=device),
                                       nv.ACT_GELU if spec.act == "gelu" else nv.ACT_NONE)

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.K

    @property
    def gemm_bytes(self) -> int:
        """Algorithmic bytes of the GEMM: codes + scales of X and W read once,
        Y (bf16) written once (plus the fused codes + scales when fused)."""
        import nvfp4_block_scaled_19_b200 as nv
        if self.fp8:
            b = (self.M + self.N) * self.K
        else:
            b = ((self.M + self.N) * self.K // 2 + nv.sf_bytes(self.M, self.K)
                 + nv.sf_bytes(self.N, self.K))
        b += 2 * self.M * self.N
        if self.fused is not None:
            b += self.M * self.N // 2 + nv.sf_bytes(self.M, self.N)
        return b

    @property
    def quant_bytes(self) -> int:
        """Algorithmic bytes of amax (read X) + quantize (read X, write codes +
        scales); 0 for a layer fed by the previous layer's fused output."""
        import nvfp4_block_scaled_19_b200 as nv
        if self.spec.x_from_prev:
            return 0
        n = self.M * self.K
        if self.fp8:          # amax (read X) + quantize (read X, write 1 B codes)
            return 2 * n + 2 * n + n
        if self.row_scales:   # one pass over X (the second read of a row hits L1/L2)
            return 2 * n + n // 2 + nv.sf_bytes(self.M, self.K) + 4 * self.M
        if self.stale:        # one pass over X with the previous call's amax
            return 2 * n + n // 2 + nv.sf_bytes(self.M, self.K)
        return 2 * n + 2 * n + n // 2 + nv.sf_bytes(self.M, self.K)


def layer_input(layers, i):
    """The quantized X of layer i: its own buffer, or the previous layer's
    fused output."""
    L = layers[i]
    return layers[i - 1].fused.out if L.spec.x_from_prev else L.xq


def run_step(nv, layers, ev=None):
    """One pass of the hot path; ev: optional per-layer event triples around
    the quantize and the GEMM (the quantize span is empty for a chained layer)."""
    for i, L in enumerate(layers):
        if ev is not None:
            ev[i][0].record()
        if L.spec.x_from_prev:
            pass
        elif L.fp8:
            nv.tensor_amax(L.x, L.amax)
            nv.quantize_fp8(L.x, L.amax, L.xq)
        elif L.row_scales:
            nv.quantize_rowwise(L.x, L.xq)
        elif L.sharded:
            from nvfp4_block_scaled_19_b200 import sharded
            sharded.quantize_sharded(L.x, L.xq, L.amax)
        elif L.stale:
            k = L.calls & 1
            nv.quantize_one_pass(L.x, L.amax_pair[k], L.amax_pair[1 - k], L.xq)
            L.calls += 1
        else:
            nv.quantize_dynamic(L.x, L.xq, L.amax)
        if ev is not None:
            ev[i][1].record()
        if L.fp8:
            nv.gemm_fp8(L.xq, L.lin.w, L.y, L.fused, want_y=L.y is not None)
        else:
            nv.gemm(layer_input(layers, i), L.lin.w, L.y, L.fused, want_y=L.y is not None)
        if ev is not None:
            ev[i][2].record()


def calibrate(nv, layers) -> None:
    """Static tensor scales of the fused outputs: one untimed pass, then
    S_enc = 2688 / amax of each fused output (device-side, before timing)."""
    run_step(nv, layers)
    for L in layers:
        if L.fused is not None:
            if L.m_global != L.M:   # token shards: one static output scale for the group
                from nvfp4_block_scaled_19_b200 import sharded
                sharded.all_reduce_max(L.fused.amax)
            a = L.fused.amax.clamp_min(torch.finfo(torch.float32).tiny)
            L.fused.s_enc.copy_(torch.full_like(a, 2688.0) / a)
    torch.cuda.synchronize()


def graph_timing(nv, layers, flush, steps, dist, device, world) -> dict:
    """The same step captured once in a CUDA graph and replayed (no host
    launch overhead between the kernels); L2 flushed before every replay,
    outside the timed span."""
    if world > 1 and any(L.sharded for L in layers):
        return {"value": None, "note": "not captured: the token-sharded step holds an NCCL "
                                       "all-reduce"}
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        run_step(nv, layers)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=side):
            run_step(nv, layers)
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(3):
        flush.zero_()
        g.replay()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    barrier(dist, device)
    for a, b in ev:
        flush.zero_()
        a.record()
        g.replay()
        b.record()
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in ev)
    sec = max_over_ranks(ms / 1e3, dist, device)
    del g
    flops = job_flops(layers, world) * steps
    return {"value": round(flops / sec / 1e12, 3), "unit": UNIT,
            "ms_per_step": round(ms / steps, 5), "steps": steps,
            "kernels_per_step": launches_per_step(layers),
            "note": "one CUDA graph per step (captured once), events around each replay"}


def launches_per_step(layers) -> int:
    return sum(1 + (0 if L.spec.x_from_prev else 2 if (L.fp8 or L.sharded) else 1)
               for L in layers)


def job_flops(layers, world: int) -> int:
    """FLOPs of one step over the whole job: replicas each run the whole
    workload; token shards run it once between them."""
    if any(L.m_global != L.M for L in layers) or any(L.sharded for L in layers):
        return sum(2 * L.m_global * L.N * L.K for L in layers)
    return sum(L.flops for L in layers) * world


def gpu_arm(args) -> dict | None:
    import nvfp4_block_scaled_19_b200 as nv
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    nv.lib()
    peaks, peak_src = load_peaks()
    w = WORKLOADS[args.workload]
    row = args.act_scale == "row"
    stale = args.act_scale == "stale"
    fp8 = args.variant == "fp8"
    shard = args.shard == "tokens"
    if shard and (fp8 or row or stale):
        raise SystemExit("--shard tokens runs the per-tensor dynamic NVFP4 path only")
    from nvfp4_block_scaled_19_b200.sharded import shard_rows
    r0, r1 = shard_rows(w.M, world, rank) if shard else (0, w.M)
    layers = []
    for i, l in enumerate(w.layers):
        x, wt = layer_inputs(w, i)
        if shard and x is not None:
            x = x[r0:r1].contiguous()
        layers.append(Layer(nv, l, r1 - r0, x, wt, device, row_scales=row, fp8=fp8, stale=stale,
                            m_global=w.M, sharded=shard))
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    torch.cuda.synchronize()
    calibrate(nv, layers)

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        run_step(nv, layers)
    torch.cuda.synchronize()
    code, detail = nv.device_error()
    if code != 0:
        raise RuntimeError(f"device wait timed out during warm-up (tag {detail})")

    n_l = len(layers)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    barrier(dist, device)
    torch.cuda.synchronize()
    t_wall0 = time.time()
    q_ms, g_ms = timed_steps(nv, layers, flush, args.steps)
    t_wall1 = time.time()
    barrier(dist, device)
    time.sleep(0.1)
    sampler.window = (t_wall0, t_wall1)
    sampler.stop()
    code, detail = nv.device_error()
    if code != 0:
        raise RuntimeError(f"device wait timed out (tag {detail})")

    step_ms = [sum(q_ms[i][s] + g_ms[i][s] for i in range(n_l)) for s in range(args.steps)]
    total_s = sum(step_ms) / 1e3
    total_s = max_over_ranks(total_s, dist, device)
    value = job_flops(layers, world) * args.steps / total_s / 1e12

    # Roofline of the dominant kernel (the GEMM), live CUDA-event durations.
    g_avg = [sum(g) / len(g) for g in g_ms]
    q_avg = [sum(q) / len(q) for q in q_ms]
    top = max(range(n_l), key=lambda i: g_avg[i])
    bf16_burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    bf16_sust = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    per_bf16 = FP8_PER_BF16 if fp8 else FP4_PER_BF16
    fp4_peak, regime, peak_note = tensor_peak(per_bf16, bf16_burst, bf16_sust, total_s)
    gemm_tflops = layers[top].flops / (g_avg[top] * 1e-3) / 1e12
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    q_bytes = sum(L.quant_bytes for L in layers)
    q_ms_sum = sum(q_avg[i] for i, L in enumerate(layers) if not L.spec.x_from_prev)
    q_gbs = q_bytes / (q_ms_sum * 1e-3) / 1e9 if q_bytes else 0.0

    traffic, traffic_src = ((None, "no ncu summary for the FP8 variant") if fp8
                            else profiled_traffic(profile_name(w, layers[top].spec)))
    per_layer = []
    for i, L in enumerate(layers):
        g_tf = L.flops / (g_avg[i] * 1e-3) / 1e12
        incl = L.flops / ((g_avg[i] + q_avg[i]) * 1e-3) / 1e12
        per_layer.append({
            "layer": L.spec.name, "M": L.M, "N": L.N, "K": L.K,
            "quantize_us": round(q_avg[i] * 1e3, 2), "gemm_us": round(g_avg[i] * 1e3, 2),
            "gemm_tflops": round(g_tf, 1), "gemm_frac": round(g_tf / fp4_peak, 4),
            "tflops_incl_quantize": round(incl, 1),
            "frac_incl_quantize": round(incl / fp4_peak, 4),
            "fused_output": L.fused is not None})
    modes = (ffn_down_modes(nv, args, flush, device, fp4_peak)
             if w.name == "ffn_2048" and not (fp8 or row or stale or shard) else None)
    graph = graph_timing(nv, layers, flush, args.steps, dist, device, world)
    code, detail = nv.device_error()
    if code != 0:
        raise RuntimeError(f"device wait timed out in the graph replays (tag {detail})")
    e2e = host_e2e(nv, layers, args, device, dist, world)
    clocks = sampler.summary()

    if rank != 0:
        return None
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3),
        "ms_per_step": round(sum(step_ms) / args.steps, 5),
        "higher_is_better": True, "scaling": "strong" if shard else "weak", "vs_baseline": None,
        "dtype": ("fp8 (e4m3, per-tensor fp32 scales, fp32 accumulate, bf16 out)" if fp8 else
                  "nvfp4 (e2m1 x ue4m3 block scales, fp32 accumulate, bf16 out)"),
        "data": "synthetic (seeded DiT-shaped activations and N(0,1/K) weights)",
        "config": {"workload": w.name, "description": w.description, "M": w.M,
                   "layers": [[l.name, l.K, l.N] + (["gelu"] if l.act == "gelu" else [])
                              + (["input: previous fused output"] if l.x_from_prev else [])
                              for l in w.layers],
                   "l2": "flushed between steps (256 MiB write, outside the timed spans)",
                   "variant": args.variant,
                   "activation_scale": ("per token (nvfp4_quantize_rowwise, one pass)" if row
                                        else "per tensor, previous call's amax "
                                             "(nvfp4_quantize_one_pass, one pass)" if stale
                                        else "per tensor, dynamic (amax + nvfp4_fp8_quantize)"
                                        if fp8 else
                                        "per tensor, dynamic (nvfp4_quantize_dynamic)"),
                   "parallelism": (f"tokens x{world} (rows {r0}..{r1 - 1} on rank {rank}; "
                                   "one all-reduce(MAX) of the amax per layer and step)"
                                   if shard else f"replicas x{world}")},
        # Both measured figures; `regime` names the one this run's length calls
        # for (the roofline's peak).
        "pct_fp4_peak": {"of_4x_measured_bf16_burst":
                             round(value / world / (per_bf16 * bf16_burst), 4),
                         "of_4x_measured_bf16_sustained":
                             round(value / world / (per_bf16 * bf16_sust), 4),
                         "of_nominal_9pf": round(value / world / NOMINAL_FP4_TFLOPS, 4),
                         "regime": regime}
        if not fp8 else
        {"of_2x_measured_bf16_burst": round(value / world / (per_bf16 * bf16_burst), 4),
         "of_2x_measured_bf16_sustained": round(value / world / (per_bf16 * bf16_sust), 4),
         "of_nominal_4_5pf": round(value / world / (NOMINAL_FP4_TFLOPS / 2), 4),
         "regime": regime},
        "quantize": {"gbs": round(q_gbs, 1), "pct_hbm": round(q_gbs / hbm, 4),
                     "pct_hbm_nominal_8tbs": round(q_gbs / NOMINAL_HBM_GBS, 4),
                     "ms_per_step": round(q_ms_sum, 5),
                     "note": ("per-token quantize, one pass: algorithmic bytes 2.5625 B/elem "
                              "+ per-row scales" if row else
                              "one-pass quantize with the previous call's amax: algorithmic "
                              "bytes 2.5625 B/elem + scales" if stale else
                              "single-launch amax + dynamic quantize of every layer input; "
                              "algorithmic bytes 4.5625 B/elem + scales (the second read from "
                              "shared memory where a slice per SM fits, else from L2)")},
        "gemm": {"tflops": round(gemm_tflops, 1), "ms": round(g_avg[top], 5),
                 "layer": layers[top].spec.name},
        "per_layer": per_layer,
        "roofline": {"bound": "tensor",
                     "kernel": ("gemm_pair_kernel FP8 (tcgen05.mma cta_group::2 kind::f8f6f4)"
                                if fp8 else gemm_kernel_name(layers[top].M, layers[top].N)),
                     "achieved": round(gemm_tflops, 1), "peak": round(fp4_peak, 1),
                     "unit": "TFLOP/s", "frac": round(gemm_tflops / fp4_peak, 4),
                     "traffic": traffic, "traffic_source": traffic_src,
                     "algorithmic_bytes": layers[top].gemm_bytes,
                     "peak_source": f"{peak_src}: {peak_note}"},
        "clocks": clocks,
        "graph": graph,
        "e2e": e2e,
        "gpu_launches": launches_per_step(layers) * args.steps,
    }
    if modes is not None:
        line["ffn_down_modes"] = modes
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    return line


def timed_steps(nv, layers, flush, steps):
    """`steps` passes of the step with the L2 flushed before each, outside the
    timed spans; per layer the CUDA-event durations (ms) of its quantize and
    its GEMM in every step."""
    n_l = len(layers)
    ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_l)]
          for _ in range(steps)]
    for s in range(steps):
        flush.zero_()          # L2 flush between steps, outside the timed spans
        run_step(nv, layers, ev[s])
    torch.cuda.synchronize()
    q_ms = [[ev[s][i][0].elapsed_time(ev[s][i][1]) for s in range(steps)] for i in range(n_l)]
    g_ms = [[ev[s][i][1].elapsed_time(ev[s][i][2]) for s in range(steps)] for i in range(n_l)]
    return q_ms, g_ms


def tensor_peak(per_bf16: float, bf16_burst: float, bf16_sust: float,
                timed_s: float) -> tuple[float, str, str]:
    """The tensor roofline for a run whose timed steps took timed_s seconds of
    device time back to back: per_bf16 x the burst bf16 figure for a short
    run, x the sustained one from SUSTAINED_AFTER_S on (the GPU then sits at
    its power cap, where the sustained figure was measured).  Returns (peak
    TFLOP/s, "burst" | "sustained", a note naming the figure)."""
    if timed_s >= SUSTAINED_AFTER_S:
        return (per_bf16 * bf16_sust, "sustained",
                f"{per_bf16:g} x bf16_tflops_sustained ({bf16_sust}): the timed steps ran "
                f"{timed_s:.2f} s back to back (>= {SUSTAINED_AFTER_S} s, at the power cap); "
                f"burst would be {per_bf16 * bf16_burst:.1f}")
    return (per_bf16 * bf16_burst, "burst",
            f"{per_bf16:g} x bf16_tflops burst ({bf16_burst}): the timed steps ran "
            f"{timed_s:.3f} s (< {SUSTAINED_AFTER_S} s); sustained would be "
            f"{per_bf16 * bf16_sust:.1f}")


def ffn_down_modes(nv, args, flush, device, fp4_peak) -> dict:
    """The FFN down-projection at 2048^2 (M=16896, K=12288, N=3072) in the
    three ways its input can be produced, each timed like the step (L2 flushed
    before every pass, CUDA events, `steps` passes):
      dynamic: amax + quantize of the bf16 input in one launch, then the GEMM
        (the headline step's second layer, timed here again on its own);
      stale_scale: one pass over the input with the previous call's amax;
      fused_producer: the input's codes come straight from the up-projection's
        epilogue (GELU + NVFP4 quantize), so the down-projection has no
        quantize of its own; reported for the down GEMM and for the whole FFN
        block (up-projection with its input quantize, then down)."""
    def run(wname, stale):
        w = WORKLOADS[wname]
        layers = []
        for i, l in enumerate(w.layers):
            x, wt = layer_inputs(w, i)
            layers.append(Layer(nv, l, w.M, x, wt, device, stale=stale))
        calibrate(nv, layers)
        for _ in range(max(args.warmup, 3)):
            flush.zero_()
            run_step(nv, layers)
        q, g = timed_steps(nv, layers, flush, args.steps)
        code, detail = nv.device_error()
        if code != 0:
            raise RuntimeError(f"device wait timed out (tag {detail})")
        out = [(L.flops, L.quant_bytes, sum(q[i]) / len(q[i]), sum(g[i]) / len(g[i]))
               for i, L in enumerate(layers)]
        del layers
        torch.cuda.empty_cache()
        return out

    res = {}
    for name, stale in (("dynamic", False), ("stale_scale", True)):
        (fl, qb, q, g), = run("ffn_down_2048", stale)
        res[name] = {"quantize_us": round(q * 1e3, 2), "gemm_us": round(g * 1e3, 2),
                     "tflops_incl_quantize": round(fl / ((q + g) * 1e-3) / 1e12, 1),
                     "frac_incl_quantize": round(fl / ((q + g) * 1e-3) / 1e12 / fp4_peak, 4),
                     "quantize_gbs": round(qb / (q * 1e-3) / 1e9, 1)}
    (fu, _, qu, gu), (fd, _, _, gd) = run("ffn_block_2048", False)
    flops = fu + fd
    res["fused_producer"] = {
        "down_gemm_us": round(gd * 1e3, 2),
        "down_tflops": round(fd / (gd * 1e-3) / 1e12, 1),
        "up_quantize_us": round(qu * 1e3, 2), "up_gemm_gelu_quantize_us": round(gu * 1e3, 2),
        "block_tflops_incl_quantize": round(flops / ((qu + gu + gd) * 1e-3) / 1e12, 1),
        "block_frac_incl_quantize": round(flops / ((qu + gu + gd) * 1e-3) / 1e12 / fp4_peak, 4),
        "note": "ffn_block_2048: the up-projection's epilogue applies GELU and writes the "
                "down-projection's NVFP4 codes and scales (static scale calibrated once)"}
    res["peak_tflops"] = round(fp4_peak, 1)
    return res


def host_e2e(nv, layers, args, device, dist, world) -> dict:
    """Same metric end to end: pinned host X in, host Y out, copies timed.
    Independent layers go through nvfp4_linear_host; a chain (a layer fed by
    the previous layer's fused output) through the Python API, copying every
    drawn X in and the last layer's Y out.  Each independent layer runs on a
    stream of its own (with its own workspaces), so one layer's host-to-device
    copy can overlap another's device-to-host copy and compute; a layer's
    steps stay in order on its stream."""
    if any(L.spec.x_from_prev or L.row_scales or L.fp8 or L.stale or L.sharded for L in layers):
        return chain_e2e(nv, layers, args, device, dist, world)
    main = torch.cuda.current_stream()
    hosts = []
    for L in layers:
        xh = L.x_cpu.contiguous().pin_memory()
        yh = torch.empty(L.M, L.N, dtype=torch.bfloat16).pin_memory()
        hosts.append((xh, yh, L.lin.host_workspace(L.M, device), torch.cuda.Stream(device)))
    steps = max(1, min(args.steps, args.e2e_steps))
    for _ in range(2):
        for L, (xh, yh, ws, st) in zip(layers, hosts):
            L.lin.forward_host(xh, yh, ws, stream=st)
    torch.cuda.synchronize()
    barrier(dist, device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    for _, _, _, st in hosts:
        st.wait_event(e0)
    for _ in range(steps):
        for L, (xh, yh, ws, st) in zip(layers, hosts):
            L.lin.forward_host(xh, yh, ws, stream=st)
    for _, _, _, st in hosts:
        main.wait_stream(st)
    e1.record(main)
    torch.cuda.synchronize()
    sec = max_over_ranks(e0.elapsed_time(e1) / 1e3, dist, device)
    flops = sum(L.flops for L in layers) * steps
    return {"value": round(aggregate(flops, world, sec) / 1e12, 3), "unit": UNIT,
            "h2d_bytes_per_step": sum(L.M * L.K * 2 for L in layers),
            "d2h_bytes_per_step": sum(L.M * L.N * 2 for L in layers),
            "steps": steps, "api": "nvfp4_linear_host (C ABI, pinned host buffers; "
                                   "one stream per independent layer)"}


def chain_e2e(nv, layers, args, device, dist, world) -> dict:
    """End to end through the Python API: every drawn X copied in, every bf16
    Y the workload produces copied out, pinned host buffers."""
    xs = [(L, L.x_cpu.contiguous().pin_memory()) for L in layers if L.x_cpu is not None]
    ys = [(L, torch.empty(L.M, L.N, dtype=torch.bfloat16).pin_memory())
          for L in layers if L.y is not None]
    steps = max(1, min(args.steps, args.e2e_steps))

    def one():
        for L, xh in xs:
            L.x.copy_(xh, non_blocking=True)
        run_step(nv, layers)
        for L, yh in ys:
            yh.copy_(L.y, non_blocking=True)

    for _ in range(2):
        one()
    torch.cuda.synchronize()
    barrier(dist, device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        one()
    e1.record()
    torch.cuda.synchronize()
    sec = max_over_ranks(e0.elapsed_time(e1) / 1e3, dist, device)
    flops = job_flops(layers, world) * steps
    return {"value": round(flops / sec / 1e12, 3), "unit": UNIT,
            "h2d_bytes_per_step": sum(L.M * L.K * 2 for L, _ in xs),
            "d2h_bytes_per_step": sum(L.M * L.N * 2 for L, _ in ys), "steps": steps,
            "api": "Python API (quantize_dynamic / quantize_rowwise / quantize_one_pass / "
                   "quantize_fp8, gemm), "
                   "pinned host buffers"}


# ----------------------------------------------------------------- CPU oracle (baseline / reference)

def oracle_sample(w, rows: int) -> tuple[float, int, str]:
    """One bounded oracle pass: for every layer, amax + quantize of a `rows`-row
    slice of X (for a chained layer: the previous layer's output, activated and
    rounded to bf16, quantized with its own tensor scale), quantize of W (its
    static scale), and the dequantize-then-fp64 GEMM of that slice.
    Returns (seconds, flops, description)."""
    import numpy as np
    import oracle
    from workloads import bf16_bits
    secs, flops = 0.0, 0
    prev = None
    for li, l in enumerate(w.layers):
        x, wt = layer_inputs(w, li, M=rows)
        bq, bsf, bsd, _ = oracle.quantize_dynamic(bf16_bits(wt), l.N, l.K)  # static: untimed
        t0 = time.perf_counter()
        if l.x_from_prev:
            xb = bf16_bits(torch.from_numpy(prev.astype(np.float32)).to(torch.bfloat16))
            aq, asf, asd, _ = oracle.quantize_dynamic(xb, rows, l.K)
        else:
            aq, asf, asd, _ = oracle.quantize_dynamic(bf16_bits(x), rows, l.K)
        y = oracle.gemm(aq, asf, asd, bq, bsf, bsd, rows, l.N, l.K)
        prev = oracle.gelu(y) if l.act == "gelu" else y
        secs += time.perf_counter() - t0
        flops += 2 * rows * l.N * l.K
    desc = (f"{rows} rows of every layer input of {w.name} (full K, full N): amax + quantize "
            f"+ dequantize-then-fp64 GEMM; weight quantize untimed (static)")
    return secs, flops, desc


def sample_rows(w, seconds_per_pass: float) -> int:
    """Rows per oracle pass so that one pass takes about `seconds_per_pass`
    (from a timed 64-row pass), between 64 and the workload's M."""
    t64, _, _ = oracle_sample(w, 64)
    rows = int(64 * seconds_per_pass / max(t64, 1e-6))
    return max(64, min(w.M, rows))


def cpu_baseline(w, target_s: float) -> dict:
    """The oracle as it stands on the host cores: passes over a row slice of
    the workload (all rows when they fit) until about target_s of work."""
    import oracle
    oracle.lib()
    rows = sample_rows(w, target_s / 4)
    secs, flops, passes, desc = 0.0, 0, 0, ""
    while passes == 0 or secs < target_s:
        s, f, desc = oracle_sample(w, rows)
        secs, flops, passes = secs + s, flops + f, passes + 1
    return {"value": round(flops / secs / 1e12, 6), "unit": UNIT,
            "cores": oracle.num_threads(), "cpu_model": cpu_model(), "kind": "oracle",
            "sample": f"{passes} passes of: {desc}", "seconds": round(secs, 3)}


def cpu_model() -> str:
    """The host CPU's model name (Linux /proc/cpuinfo), or "unknown"."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def quantize_sweep(args) -> dict:
    """Quantize throughput over sizes: 2^20 .. 2^29 bf16 elements as
    [n / 4096, 4096] N(0,1) (seeded, drawn on the device), each path timed
    with CUDA events over `sweep_iters` calls, L2 flushed (256 MiB write)
    before every call, outside the timed span.  Algorithmic bytes: dynamic
    4.5625 B/elem (amax read + quantize read + codes and scales written),
    one pass 2.5625 B/elem, amax alone 2 B/elem."""
    import nvfp4_block_scaled_19_b200 as nv
    torch.cuda.set_device(0)
    peaks, _ = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    gen = torch.Generator(device="cuda")
    rows_out = []
    for lg in range(20, 30):
        n = 1 << lg
        gen.manual_seed(lg)
        x = torch.randn(n // 4096, 4096, generator=gen, device="cuda").to(torch.bfloat16)
        out = nv.empty_nvfp4(n // 4096, 4096)
        amax = torch.empty(1, device="cuda")
        a_pair = [torch.empty(1, device="cuda") for _ in range(2)]
        nv.tensor_amax(x, a_pair[0])
        paths = {
            "dynamic": (lambda: nv.quantize_dynamic(x, out, amax), 4.5625),
            "one_pass_stale": (lambda: nv.quantize_one_pass(x, a_pair[0], a_pair[1], out), 2.5625),
            "amax": (lambda: nv.tensor_amax(x, amax), 2.0),
        }
        row = {"elements": n, "shape": [n // 4096, 4096]}
        for name, (fn, bpe) in paths.items():
            for _ in range(3):
                fn()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.sweep_iters)]
            for e0, e1 in ev:
                flush.zero_()
                e0.record()
                fn()
                e1.record()
            torch.cuda.synchronize()
            us = statistics.median(e0.elapsed_time(e1) for e0, e1 in ev) * 1e3
            gbs = n * bpe / (us * 1e-6) / 1e9
            row[name] = {"us": round(us, 2), "gbs": round(gbs, 1), "pct_hbm": round(gbs / hbm, 4),
                         "pct_hbm_nominal_8tbs": round(gbs / NOMINAL_HBM_GBS, 4)}
        rows_out.append(row)
        del x, out
    code, detail = nv.device_error()
    if code != 0:
        raise RuntimeError(f"device wait timed out (tag {detail})")
    return {"metric": "quantize GB/s (% HBM) over sizes", "unit": "GB/s", "hbm_gbs": hbm,
            "data": "synthetic N(0,1), seeded on the device", "iters": args.sweep_iters,
            "l2": "flushed before every call (256 MiB write, outside the timed span)",
            "sweep": rows_out}


def reference_arm(args) -> dict | None:
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    import oracle
    oracle.lib()
    w = WORKLOADS[args.workload]
    for _ in range(max(args.warmup, 1)):
        oracle_sample(w, 64)
    rows = sample_rows(w, args.cpu_seconds / 8)
    secs, flops = 0.0, 0
    desc = ""
    steps = max(1, args.steps if args.steps <= 20 else 20)
    for _ in range(steps):
        s, f, desc = oracle_sample(w, rows)
        secs += s
        flops += f
    value = flops / secs / 1e12
    cores = oracle.num_threads()
    return {"metric": METRIC, "value": round(value, 6), "unit": UNIT, "impl": "reference",
            "n_gpus": world, "steps": steps, "warmup": max(args.warmup, 1),
            "ms_per_step": round(secs / steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
            "data": "synthetic", "config": {"workload": w.name, "M": w.M,
                                            "layers": [[l.name, l.K, l.N] for l in w.layers]},
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cores,
                             "cpu_model": cpu_model(), "kind": "oracle", "sample": desc},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="oracle work timed for cpu_baseline (per reference step: 1/8 of it)")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--variant", choices=["nvfp4", "fp8"], default="nvfp4",
                    help="nvfp4 (the path) or the FP8 per-tensor variant")
    ap.add_argument("--act-scale", choices=["tensor", "row", "stale"], default="tensor",
                    help="activation tensor scale: per tensor (the pages' scheme), per token, "
                         "or per tensor from the previous call's amax (one pass)")
    ap.add_argument("--shard", choices=["replicas", "tokens"], default="replicas",
                    help="N > 1: independent replicas (weak scaling) or the workload's tokens "
                         "split across ranks with one amax all-reduce per layer (strong)")
    ap.add_argument("--quantize-sweep", action="store_true",
                    help="instead of the step: quantize throughput over 2^20..2^29 elements")
    ap.add_argument("--sweep-iters", type=int, default=20)
    args = ap.parse_args(argv)
    if args.quantize_sweep:
        print(json.dumps(quantize_sweep(args)), flush=True)
        return 0
    line = reference_arm(args) if args.impl == "reference" else gpu_arm(args)
    if line is not None:
        print(json.dumps(line), flush=True)
    rank, world, _ = dist_env()
    if world > 1 and args.impl != "reference":
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
