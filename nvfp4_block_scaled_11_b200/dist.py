"""Sharded NVFP4 quantization across ranks (one process per GPU).

A tensor split into contiguous 16-element-aligned shards, one per rank, has one FP32 tensor scale
(the NVFP4 second-level scale, "NVIDIAのFP4推論が50倍の効率を実現", 超低精度推論を支えるアーキテクチャ), so the
ranks exchange exactly one value: the maximum of their shard amaxes.  Max is exact and order-free,
so every rank obtains the single-GPU result bit for bit:

    local amax  ->  all_reduce(MAX) of one float  ->  g = amax / 2688  ->  quantize the shard with g

With the NCCL backend the all-reduce moves 4 bytes over NVLink; it is latency-bound, and no other
communication is needed because blocks are independent once g is known.

The per-shard steps are passed in as `ops` so that the exchange logic can run with the CUDA library
(the default) or with any other implementation of the same three steps.
"""
from __future__ import annotations

import dataclasses
from typing import Any, Callable

import torch
import torch.distributed as dist


@dataclasses.dataclass
class ShardOps:
    amax: Callable[[torch.Tensor], torch.Tensor]                 # x -> float32[1]
    global_scale: Callable[[torch.Tensor], torch.Tensor]         # amax float32[1] -> g float32[1]
    quantize: Callable[..., Any]                                 # (x, f_lo, f_hi, g) -> (codes, scales)


def cuda_ops() -> ShardOps:
    """The library's CUDA entry points."""
    import nvfp4_block_scaled_11_b200 as nv

    def _q(x, f_lo, f_hi, g):
        codes, scales, _, _, _ = nv.quantize_ex(x, f_lo, f_hi, gscale_in=g, want_f=False, want_sse=False)
        return codes, scales

    return ShardOps(amax=nv.tensor_amax, global_scale=nv.global_scale, quantize=_q)


def sharded_quantize(x_shard: torch.Tensor, f_lo: int = -2, f_hi: int = 6, group=None, ops: ShardOps | None = None):
    """Quantize this rank's shard with the tensor scale of the whole (sharded) tensor.

    Returns (codes, scales, g) for the shard; g is identical on every rank."""
    ops = cuda_ops() if ops is None else ops
    amax = ops.amax(x_shard)
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    g = ops.global_scale(amax)
    codes, scales = ops.quantize(x_shard, f_lo, f_hi, g)
    return codes, scales, g


def shard_bounds(n: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous, 16-element-aligned shard [lo, hi) of n elements for `rank` of `world`."""
    if n % 16:
        raise ValueError("n must be a multiple of 16")
    blocks = n // 16
    per = blocks // world
    extra = blocks % world
    lo_b = rank * per + min(rank, extra)
    hi_b = lo_b + per + (1 if rank < extra else 0)
    return 16 * lo_b, 16 * hi_b
