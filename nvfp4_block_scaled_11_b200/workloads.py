"""Seeded synthetic inputs shaped like the pages' workloads.

This module only draws random numbers and arranges them; it holds none of the quantization
arithmetic, so both the CUDA path and the CPU oracle can take their inputs from it.

Workloads (stand-ins for data the pages measure on, which is not available here):

* ``act_f32``   -- FP32 activations [1024, 4096], i.i.d. N(0,1), seed 0.
* ``act_bf16``  -- BF16 LLM-activation-like [8192, 8192]: 0.5 * Student-t(nu=3), with 1% of the columns
                   (82, chosen by a seeded permutation) multiplied by 20 as outlier channels.
* ``kv_bf16``   -- BF16 KV-cache keys [1, 8, 32768, 128]: N(0,1) plus a per-channel bias ~ N(0, 2)
                   on 4 seeded channels of head_dim (the same channels for every head), seed 2.
* ``stream_f32``-- FP32 stream of 2^30 elements: per-element mixture 0.9*N(0,1) + 0.1*N(0, 16), seed 3.
* ``bev_f16``   -- FP16 deformable-attention value map [6 cams, 30825 keys, 8 heads, 32 ch]; the keys
                   are 4 levels (116x200, 58x100, 29x50, 15x25) and each level's N(0,1) entries are
                   multiplied by a gain of 1, 2, 4, 8 respectively, seed 5.

Each generator takes ``scale`` in (0, 1] to shrink the leading dimension for small parity cases
while keeping the recipe (distribution, outlier structure, layout) unchanged.
"""
from __future__ import annotations

import dataclasses
import math

import torch

LEVELS = ((116, 200), (58, 100), (29, 50), (15, 25))


@dataclasses.dataclass
class Workload:
    name: str
    x: torch.Tensor          # the input tensor (float32 / bfloat16 / float16)
    f_lo: int
    f_hi: int
    kind: str                # "quantize" | "kv"
    note: str


def _gen(seed: int, device, shard: int = 0) -> torch.Generator:
    """Generator for one workload; shard k > 0 (another rank's slice) gets its own stream."""
    g = torch.Generator(device=device)
    g.manual_seed(seed + 7919 * shard)
    return g


def act_f32(device="cpu", scale: float = 1.0) -> torch.Tensor:
    rows = max(1, int(1024 * scale))
    return torch.randn((rows, 4096), generator=_gen(0, device), device=device, dtype=torch.float32)


def act_bf16(device="cpu", scale: float = 1.0, cols: int = 8192) -> torch.Tensor:
    rows = max(1, int(8192 * scale))
    g = _gen(1, device)
    z = torch.randn((rows, cols), generator=g, device=device, dtype=torch.float32)
    chi2 = torch.zeros_like(z)
    for _ in range(3):
        w = torch.randn((rows, cols), generator=g, device=device, dtype=torch.float32)
        chi2.add_(w * w)
    t = z / torch.sqrt(chi2 / 3.0)
    t.mul_(0.5)
    n_out = max(1, round(0.01 * cols))
    gcols = torch.Generator(device="cpu")
    gcols.manual_seed(1)
    idx = torch.randperm(cols, generator=gcols)[:n_out].to(device)
    t[:, idx] *= 20.0
    return t.to(torch.bfloat16)


def kv_bf16(device="cpu", scale: float = 1.0, heads: int = 8, head_dim: int = 128) -> torch.Tensor:
    T = max(64, int(32768 * scale))
    g = _gen(2, device)
    k = torch.randn((1, heads, T, head_dim), generator=g, device=device, dtype=torch.float32)
    gc = torch.Generator(device="cpu")
    gc.manual_seed(2)
    chans = torch.randperm(head_dim, generator=gc)[:4]
    bias = torch.randn((4,), generator=gc) * math.sqrt(2.0)
    for c, b in zip(chans.tolist(), bias.tolist()):
        k[..., c] += b
    return k.to(torch.bfloat16)


def stream_f32(device="cpu", scale: float = 1.0, shard: int = 0) -> torch.Tensor:
    n = max(1 << 14, int((1 << 30) * scale))
    n -= n % 16
    g = _gen(3, device, shard)
    a = torch.randn((n,), generator=g, device=device, dtype=torch.float32)
    b = torch.randn((n,), generator=g, device=device, dtype=torch.float32)
    pick = torch.rand((n,), generator=g, device=device) < 0.1
    b.mul_(4.0)
    return torch.where(pick, b, a)


def bev_f16(device="cpu", scale: float = 1.0) -> torch.Tensor:
    cams = max(1, int(round(6 * scale)))
    g = _gen(5, device)
    keys = sum(h * w for h, w in LEVELS)
    v = torch.randn((cams, keys, 8, 32), generator=g, device=device, dtype=torch.float32)
    start = 0
    for lvl, (h, w) in enumerate(LEVELS):
        v[:, start:start + h * w] *= float(1 << lvl)
        start += h * w
    return v.to(torch.float16)


def weight_bf16(device="cpu", n_out: int = 8192, n_in: int = 8192) -> torch.Tensor:
    """Linear-layer weights [n_out, n_in]: N(0, 1/n_in) (variance-preserving init), BF16, seed 11."""
    g = _gen(11, device)
    w = torch.randn((n_out, n_in), generator=g, device=device, dtype=torch.float32)
    return (w * n_in ** -0.5).to(torch.bfloat16)


def msda_inputs(device="cpu", nq: int = 10000, bs: int = 6, heads: int = 8, points: int = 4, scale: float = 1.0):
    """Sampling locations and attention weights for deformable attention over the `bev_f16` value maps
    (levels LEVELS): loc [bs, nq, heads, L, P, 2] ~ U(-0.05, 1.05) (some points fall off the map),
    w [bs, nq, heads, L, P] = softmax over the L*P points of N(0, 1) logits; seed 13."""
    nq = max(1, int(nq * scale))
    g = _gen(13, device)
    L = len(LEVELS)
    loc = torch.rand((bs, nq, heads, L, points, 2), generator=g, device=device) * 1.1 - 0.05
    logits = torch.randn((bs, nq, heads, L * points), generator=g, device=device)
    w = torch.softmax(logits, dim=-1).reshape(bs, nq, heads, L, points)
    return loc.contiguous(), w.contiguous()


def kv_decode_keys(device="cpu", n: int = 4096, heads: int = 8, head_dim: int = 128) -> torch.Tensor:
    """Keys of n newly decoded tokens for the `kv_bf16` cache, [heads, n, head_dim] BF16: the same recipe
    (N(0,1) plus the bias of the same 4 channels, from seed 2's channel draw) with their own seed, 4."""
    g = _gen(4, device)
    k = torch.randn((heads, n, head_dim), generator=g, device=device, dtype=torch.float32)
    gc = torch.Generator(device="cpu")
    gc.manual_seed(2)
    chans = torch.randperm(head_dim, generator=gc)[:4]
    bias = torch.randn((4,), generator=gc) * math.sqrt(2.0)
    for c, b in zip(chans.tolist(), bias.tolist()):
        k[..., c] += b
    return k.to(torch.bfloat16).contiguous()


def attn_inputs(device="cpu", Tq: int = 2048, scale: float = 1.0):
    """FP4-attention inputs over the KV-cache keys: q [8, Tq, 128] ~ N(0,1) (seed 21), k = kv_bf16's keys
    [8, 32768, 128] (seed 2), v [8, 32768, 128] ~ N(0,1) (seed 22), all BF16; `scale` shrinks the tokens."""
    Tk = max(128, int(32768 * scale)) // 128 * 128
    Tq = max(64, int(Tq * scale)) // 64 * 64
    k = kv_bf16(device, scale=Tk / 32768)[0]
    q = torch.randn((8, Tq, 128), generator=_gen(21, device), device=device).to(torch.bfloat16)
    v = torch.randn((8, Tk, 128), generator=_gen(22, device), device=device).to(torch.bfloat16)
    return q, k[:, :Tk].contiguous(), v


def make(name: str, device="cpu", scale: float = 1.0, shard: int = 0) -> Workload:
    if name == "act_f32":
        return Workload(name, act_f32(device, scale), -2, 6, "quantize", "FP32 [1024,4096] N(0,1), seed 0")
    if name == "act_bf16":
        return Workload(name, act_bf16(device, scale), -2, 6, "quantize",
                        "BF16 [8192,8192] 0.5*Student-t(3), 1% outlier columns x20, seed 1")
    if name == "kv_bf16":
        return Workload(name, kv_bf16(device, scale), -2, 6, "kv",
                        "BF16 K [1,8,32768,128] N(0,1) + N(0,2) bias on 4 channels, seed 2")
    if name == "stream_f32":
        return Workload(name, stream_f32(device, scale, shard), -2, 6, "quantize",
                        "FP32 2^30 mixture 0.9 N(0,1) + 0.1 N(0,16), seed 3")
    if name == "bev_f16":
        return Workload(name, bev_f16(device, scale), -2, 6, "quantize",
                        "FP16 [6,30825,8,32] N(0,1) x level gain {1,2,4,8}, seed 5")
    raise KeyError(name)


NAMES = ("act_f32", "act_bf16", "kv_bf16", "stream_f32", "bev_f16")
