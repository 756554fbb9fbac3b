"""Token-sharded NVFP4 linear layers over several GPUs, one process per GPU.

The tokens (rows of X) of a linear layer are independent, so each rank can
take a slice of them with the weights replicated, as the pages' sequence-
parallel split of the DiT's hidden states along the token axis does
("英伟达B200狂飙10.2倍！AI绘图告别龟速！", section "多GPU支持：集群协作，释放超级计算
潜能").  The one exchange the NVFP4 path then needs is the dynamic per-tensor
scale: each rank reduces the amax of its rows, one all-reduce(MAX) over the
group makes it the whole tensor's amax, and every rank quantizes its rows
with it.  Each row then gets exactly the codes and block scales that the
single-GPU quantize of the concatenated tensor gives it (the block scales
and codes of a row depend only on the row and on S_enc).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import NVFP4Linear, NVFP4Tensor, gemm, quantize, tensor_amax


def shard_rows(rows: int, world: int, rank: int) -> tuple[int, int]:
    """[start, stop) of rank's slice of `rows` tokens: contiguous slices whose
    sizes differ by at most one, in rank order."""
    if world < 1 or not 0 <= rank < world or rows < 0:
        raise ValueError("need world >= 1, 0 <= rank < world, rows >= 0")
    return rows * rank // world, rows * (rank + 1) // world


def all_reduce_max(t: torch.Tensor, group=None) -> torch.Tensor:
    """In-place MAX over the ranks of `group` (the default group if None);
    nothing to do when no process group is initialised (a single process)."""
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return t


def quantize_sharded(x_local: torch.Tensor, out: NVFP4Tensor | None = None,
                     amax: torch.Tensor | None = None, group=None, stream=None) -> NVFP4Tensor:
    """Dynamic NVFP4 quantize of this rank's rows with the tensor scale of the
    whole row-sharded tensor: local amax, all-reduce(MAX), quantize.  `amax`
    (device fp32, optional) receives the whole tensor's amax."""
    amax = tensor_amax(x_local, amax, stream=stream)
    all_reduce_max(amax, group)
    return quantize(x_local, amax, out, stream=stream)


class ShardedNVFP4Linear:
    """The NVFP4 linear layer on this rank's tokens: replicated weights
    (quantized once, static scale), activations quantized with the group's
    dynamic tensor scale."""

    def __init__(self, w: torch.Tensor, group=None):
        self.lin = NVFP4Linear(w)
        self.group = group
        self.amax = torch.empty(1, dtype=torch.float32, device=w.device)

    def __call__(self, x_local: torch.Tensor, y: torch.Tensor | None = None, fused=None,
                 want_y: bool = True) -> torch.Tensor | None:
        xq = quantize_sharded(x_local, amax=self.amax, group=self.group)
        return gemm(xq, self.lin.w, y, fused, want_y)
