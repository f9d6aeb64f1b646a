"""Attention-sink mixed-precision K/V cache that grows during decode.

"Search your block floating-point scales!" (gist.science summary of arXiv 2605.12464),
ScaleSearchAttention > attention-sink-aware mixed-precision caching: the first and the last block of
the KV cache stay in full precision and the blocks in between are NVFP4.  During decode the last block
moves: every new token enters a BF16 window of recent tokens, and once the window holds two groups of
`recent` tokens the older group is quantized (one `nvfp4_kv_append` launch, Hadamard-rotated along
head_dim when `rotate`) into the NVFP4 middle.  The window therefore always keeps between `recent` and
2 * recent - 1 of the newest tokens in BF16.

The tensor scale is fixed by the prefill (`nvfp4_kv_gscale` over the rotated middle tokens, as in
`nvfp4_kv_mixed`); later tokens use it unchanged, so values beyond 448 * 6 * g saturate.

Host-side bookkeeping only: token rows are moved with tensor copies, every quantization runs in the
library's kernels.
"""
from __future__ import annotations

import torch

from . import KV_APPEND_BATCH_MAX, KvAppendBatch, kv_append, kv_gscale, sf_mma_bytes


class NVFP4KVCache:
    """K (or V) cache of B x H heads of dimension D with room for `capacity` NVFP4 middle tokens.

    Attributes (device tensors):
      sink   [B, H, sink, D] bf16      first tokens, verbatim
      window [B, H, 2*recent, D] bf16  ring of the newest tokens; valid slots head .. head + n_window - 1
      codes  [B, H, capacity, D/2]     NVFP4 middle, rows 0 .. n_mid - 1 valid
      scales [B, H, capacity, D/16]    or the tensor-core tile layout of the B*H [capacity, D] matrices
      gscale [1] float32               tensor scale (fixed at prefill)
    """

    def __init__(self, B: int, H: int, D: int, capacity: int, sink: int = 16, recent: int = 16, rotate: bool = True,
                 f_lo: int = -2, f_hi: int = 6, tile_layout: bool = False, device="cuda"):
        if D % 16 or recent <= 0 or sink < 0 or capacity < 0:
            raise ValueError("D must be a multiple of 16; recent > 0; sink, capacity >= 0")
        self.B, self.H, self.D, self.capacity = B, H, D, capacity
        self.n_sink_max, self.recent, self.rotate, self.f_lo, self.f_hi = sink, recent, rotate, f_lo, f_hi
        self.tile_layout = tile_layout
        dev = torch.device(device)
        self.sink = torch.zeros((B, H, sink, D), dtype=torch.bfloat16, device=dev)
        self.window = torch.zeros((B, H, 2 * recent, D), dtype=torch.bfloat16, device=dev)
        self.codes = torch.zeros((B, H, capacity, D // 2), dtype=torch.uint8, device=dev)
        if tile_layout:
            self.scales = torch.zeros(max(sf_mma_bytes(capacity, D, B * H), 1), dtype=torch.uint8, device=dev)
        else:
            self.scales = torch.zeros((B, H, capacity, D // 16), dtype=torch.uint8, device=dev)
        self.gscale = torch.zeros(1, dtype=torch.float32, device=dev)
        self.n_sink = 0
        self.n_mid = 0
        self.head = 0        # first valid window slot: 0 or recent
        self.n_window = 0
        self.prefilled = False

    @property
    def length(self) -> int:
        return self.n_sink + self.n_mid + self.n_window

    def prefill(self, k: torch.Tensor) -> None:
        """Start the cache from K[B, H, T, D] (BF16), T >= sink + recent: the tensor scale over the rotated
        middle, the middle quantized into rows 0 .. T - sink - recent - 1, sink and window verbatim."""
        B, H, T, D = k.shape
        if (B, H, D) != (self.B, self.H, self.D) or k.dtype != torch.bfloat16:
            raise ValueError("k must be bfloat16 [B, H, T, D] matching the cache")
        s, r = self.n_sink_max, self.recent
        if T < s + r:
            raise ValueError("prefill needs at least sink + recent tokens")
        k = k.contiguous()
        n_mid = T - s - r
        if n_mid > self.capacity:
            raise ValueError("prefill middle exceeds the cache capacity")
        kv_gscale(k, s, r, self.rotate, out=self.gscale)
        if n_mid:
            kv_append(k, s, n_mid, self.gscale, self.codes, self.scales, 0, self.rotate, self.f_lo, self.f_hi,
                      self.tile_layout)
        self.sink.copy_(k[:, :, :s])
        self.window[:, :, :r].copy_(k[:, :, T - r:])
        self.n_sink, self.n_mid, self.head, self.n_window = s, n_mid, 0, r
        self.prefilled = True

    def append(self, k_new: torch.Tensor) -> None:
        """Append tokens K_new[B, H, n, D] (BF16) in order."""
        if not self.prefilled:
            raise RuntimeError("prefill first")
        for i in range(k_new.shape[2]):
            if self._full():
                kv_append(*self._flush_args()[:7], self.rotate, self.f_lo, self.f_hi, self.tile_layout)
                self._flushed()
            self._push(k_new[:, :, i])

    def _full(self) -> bool:
        return self.n_window == 2 * self.recent

    def _flush_args(self):
        """kv_append's arguments for the oldest `recent` window tokens (the contiguous slots head ..
        head + recent - 1) going to rows n_mid .. of the middle, as a kv_append_batch item."""
        r = self.recent
        if self.n_mid + r > self.capacity:
            raise RuntimeError("NVFP4 cache capacity exceeded")
        return (self.window, self.head, r, self.gscale, self.codes, self.scales, self.n_mid, self.rotate,
                self.tile_layout)

    def _flushed(self) -> None:
        r = self.recent
        self.n_mid += r
        self.head = (self.head + r) % (2 * r)
        self.n_window -= r

    def _push(self, token: torch.Tensor) -> None:
        slot = (self.head + self.n_window) % (2 * self.recent)
        self.window[:, :, slot].copy_(token)
        self.n_window += 1

    def recent_tokens(self) -> torch.Tensor:
        """The BF16 window in token order, [B, H, n_window, D]."""
        idx = [(self.head + i) % (2 * self.recent) for i in range(self.n_window)]
        return self.window[:, :, idx]


class NVFP4KVCacheGroup:
    """Caches that advance together, e.g. the K and V caches of every layer of a model: append() steps all
    of them token by token, and whenever windows are full they flush together in one
    nvfp4_kv_append_batch launch per 64 caches, through descriptors prepared once (each flush only sets
    the rows).  The caches must share the ScaleSearch window [f_lo, f_hi] and one device; the result is the same as
    calling append on each cache."""

    def __init__(self, caches):
        self.caches = list(caches)
        if len({(c.f_lo, c.f_hi) for c in self.caches}) > 1:
            raise ValueError("caches in one group must share the offset window")
        if len({c.codes.device for c in self.caches}) > 1:
            raise ValueError("caches in one group must live on one device (each flush is one launch)")
        self._parts = []
        for j in range(0, len(self.caches), KV_APPEND_BATCH_MAX):
            part = self.caches[j:j + KV_APPEND_BATCH_MAX]
            batch = KvAppendBatch([(c.window, c.gscale, c.codes, c.scales, c.rotate, c.tile_layout) for c in part],
                                  part[0].f_lo, part[0].f_hi)
            self._parts.append((part, batch))

    def append(self, ks) -> None:
        """Append ks[i] [B, H, n, D] (BF16) to caches[i], the same n for every cache."""
        ks = list(ks)
        if len(ks) != len(self.caches):
            raise ValueError("one token tensor per cache")
        if not ks:
            return
        for c in self.caches:
            if not c.prefilled:
                raise RuntimeError("prefill first")
        n = ks[0].shape[2]
        if any(k.shape[2] != n for k in ks):
            raise ValueError("every cache receives the same number of tokens")
        for i in range(n):
            for part, batch in self._parts:
                full = [c._full() for c in part]
                if any(full):
                    for c, f in zip(part, full):
                        if f and c.n_mid + c.recent > c.capacity:
                            raise RuntimeError("NVFP4 cache capacity exceeded")
                    # full windows flush their oldest `recent` slots (head ..) into rows n_mid ..; others skip
                    batch([c.head for c in part], [c.recent if f else 0 for c, f in zip(part, full)],
                          [c.n_mid for c in part])
                    for c, f in zip(part, full):
                        if f:
                            c._flushed()
            for c, k in zip(self.caches, ks):
                c._push(k[:, :, i])


def append_many(caches, ks) -> None:
    """Append one decode step's new tokens to several caches at once (a one-off NVFP4KVCacheGroup; keep a
    group for a decode loop, so that its descriptors are prepared once)."""
    NVFP4KVCacheGroup(caches).append(ks)
