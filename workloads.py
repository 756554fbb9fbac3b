"""Seeded synthetic inputs for the NVFP4 linear-layer workloads.

This module only draws random tensors with the shapes and value distributions
of FLUX diffusion-transformer linear layers. It holds none of the NVFP4
arithmetic (no amax, scales, rounding or packing), so both the CPU oracle and
the CUDA path can take their inputs from it without sharing method code.

Sources for the shapes: the FLUX pages describe a DiT that mixes text and
image tokens with joint attention ("NVIDIA показала, как сократить генерацию
FLUX 3 Image Klein с 22 до 6 секунд", section "Как устроена FLUX 3 Image
Klein") and time its 2048x2048 runs with classifier-free guidance ("NVIDIA
介绍用TensorRT LLM VisualGen加速Blackwell上的FLUX 3 Image Klein", paragraph on
the time breakdown).  The token counts (4096 image + 512 text tokens at
1024^2, 16384 + 512 at 2048^2, doubled for a guidance batch of 2), hidden
size 3072 and FFN width 12288 are this library's synthetic stand-ins; no
trained weights, prompts or images are used.

Every tensor is drawn from its own torch CPU generator seeded from the
workload seed and the tensor's index, as float32, transformed, then rounded
once to bfloat16 (round-to-nearest-even).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Layer:
    """One linear layer Y[M,N] = X[M,K] . W[N,K]^T and how its X is drawn."""
    name: str
    K: int
    N: int
    x_dist: str          # "normal_outliers" | "lognormal_channels" | "gelu" | "normal"
    w_std: float | None  # None -> 1/sqrt(K)
    fused_out: bool = False  # output feeds a next-layer NVFP4 quantize
    act: str = "none"        # activation of a fused epilogue: "none" | "gelu"
    x_from_prev: bool = False  # X is the previous layer's fused NVFP4 output (not drawn)
    keep_y: bool = True      # the bf16 Y is needed (False: only the fused output)
    # Draw X and W exactly as layer `source[1]` of workload `source[0]` does
    # (same seed and generator indices), so a step that strings together the
    # layers of several single-layer workloads times the same tensors.
    source: tuple[str, int] | None = None


@dataclass(frozen=True)
class Workload:
    name: str
    description: str
    M: int
    seed: int
    layers: tuple[Layer, ...] = field(default_factory=tuple)

    @property
    def flops(self) -> int:
        return sum(2 * self.M * l.N * l.K for l in self.layers)


WORKLOADS: dict[str, Workload] = {
    "tiny_linear": Workload(
        "tiny_linear",
        "Tiny NVFP4 linear: X[256,512] N(0,1) with 1% x20 outliers, "
        "W[512,512] N(0,0.02^2)",
        M=256, seed=0,
        layers=(Layer("linear", K=512, N=512, x_dist="normal_outliers", w_std=0.02),)),
    "qkv_1024": Workload(
        "qkv_1024",
        "DiT joint-attention QKV projection at 1024^2: M=4608 (4096 image + "
        "512 text tokens), K=3072, N=9216",
        M=4608, seed=1,
        layers=(Layer("qkv", K=3072, N=9216, x_dist="lognormal_channels", w_std=None),)),
    "ffn_up_2048": Workload(
        "ffn_up_2048",
        "DiT FFN up-projection at 2048^2: M=16896 (16384 + 512), K=3072, N=12288",
        M=16896, seed=2,
        layers=(Layer("ffn_up", K=3072, N=12288, x_dist="lognormal_channels", w_std=None),)),
    "ffn_down_2048": Workload(
        "ffn_down_2048",
        "DiT FFN down-projection at 2048^2: M=16896, K=12288, N=3072, X=GELU(N(0,1)); "
        "output feeds a fused next-layer NVFP4 quantize",
        M=16896, seed=3,
        layers=(Layer("ffn_down", K=12288, N=3072, x_dist="gelu", w_std=None, fused_out=True),)),
    "ffn_2048": Workload(
        "ffn_2048",
        "The DiT FFN GEMMs at 2048^2, each with the dynamic NVFP4 quantize of its input: "
        "up-projection M=16896, K=3072, N=12288, then down-projection M=16896, K=12288, "
        "N=3072 whose output feeds a fused next-layer NVFP4 quantize (inputs drawn as in "
        "ffn_up_2048 and ffn_down_2048)",
        M=16896, seed=2,
        layers=(Layer("ffn_up", K=3072, N=12288, x_dist="lognormal_channels", w_std=None,
                      source=("ffn_up_2048", 0)),
                Layer("ffn_down", K=12288, N=3072, x_dist="gelu", w_std=None, fused_out=True,
                      source=("ffn_down_2048", 0)))),
    "block_chain_2048": Workload(
        "block_chain_2048",
        "Full DiT block linear chain, CFG batch 2 at 2048^2: M=33792 through QKV "
        "(3072->9216), attn-out (3072->3072), FFN up (3072->12288), FFN down (12288->3072)",
        M=33792, seed=4,
        layers=(Layer("qkv", K=3072, N=9216, x_dist="lognormal_channels", w_std=None),
                Layer("attn_out", K=3072, N=3072, x_dist="lognormal_channels", w_std=None),
                Layer("ffn_up", K=3072, N=12288, x_dist="lognormal_channels", w_std=None),
                Layer("ffn_down", K=12288, N=3072, x_dist="gelu", w_std=None, fused_out=True))),
    "ffn_block_2048": Workload(
        "ffn_block_2048",
        "DiT FFN block at 2048^2: M=16896; up-projection 3072->12288 whose epilogue applies "
        "GELU and the NVFP4 quantize, feeding the down-projection 12288->3072 directly",
        M=16896, seed=5,
        layers=(Layer("ffn_up", K=3072, N=12288, x_dist="lognormal_channels", w_std=None,
                      fused_out=True, act="gelu", keep_y=False),
                Layer("ffn_down", K=12288, N=3072, x_dist="gelu", w_std=None,
                      x_from_prev=True))),
}


# Workloads that draw tensors of their own (not only layers of other workloads).
OWN_WORKLOADS = [n for n, w in WORKLOADS.items() if not all(l.source for l in w.layers)]


def _gen(seed: int, index: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed * 1000 + index)
    return g


def draw_x(dist: str, M: int, K: int, seed: int, index: int = 0) -> torch.Tensor:
    """Activation X[M,K] as a CPU bfloat16 tensor."""
    g = _gen(seed, index)
    z = torch.randn(M, K, generator=g, dtype=torch.float32)
    if dist == "normal":
        pass
    elif dist == "normal_outliers":
        # 1% of entries (Bernoulli(0.01)) are multiplied by 20.
        mask = torch.rand(M, K, generator=g) < 0.01
        z = torch.where(mask, z * 20.0, z)
    elif dist == "lognormal_channels":
        # Per input channel k a lognormal(0, 0.5) scale exp(0.5 * g_k).
        ch = torch.exp(0.5 * torch.randn(K, generator=g, dtype=torch.float32))
        z = z * ch
    elif dist == "gelu":
        # Exact (erf) GELU of a standard normal: skewed, heavy right tail.
        z = 0.5 * z * (1.0 + torch.erf(z * (1.0 / math.sqrt(2.0))))
    else:
        raise ValueError(f"unknown activation distribution {dist!r}")
    return z.to(torch.bfloat16)


def draw_w(N: int, K: int, std: float | None, seed: int, index: int = 1) -> torch.Tensor:
    """Weight W[N,K] (nn.Linear layout) as a CPU bfloat16 tensor, N(0, std^2)."""
    g = _gen(seed, index)
    s = (1.0 / math.sqrt(K)) if std is None else std
    return (torch.randn(N, K, generator=g, dtype=torch.float32) * s).to(torch.bfloat16)


def layer_inputs(w: Workload, li: int, M: int | None = None):
    """(X, W) for layer li of workload w; M may be overridden (smaller) for
    tests.  X is None for a layer whose input is the previous layer's fused
    output."""
    l = w.layers[li]
    seed = w.seed
    if l.source is not None:
        seed, li = WORKLOADS[l.source[0]].seed, l.source[1]
    m = w.M if M is None else M
    x = None if l.x_from_prev else draw_x(l.x_dist, m, l.K, seed, index=10 * li)
    wt = draw_w(l.N, l.K, l.w_std, seed, index=10 * li + 1)
    return x, wt


def sweep_x(numel: int, seed: int = 4) -> torch.Tensor:
    """Quantize-only sweep input: [numel/4096, 4096] N(0,1) bfloat16."""
    assert numel % 4096 == 0
    return draw_x("normal", numel // 4096, 4096, seed, index=900 + int(math.log2(numel)))


def bf16_bits(t: torch.Tensor):
    """Raw bfloat16 bit patterns of a CPU tensor as a numpy uint16 array."""
    import numpy as np
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
