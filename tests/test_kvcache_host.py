"""Host logic of the decode caches, without a GPU: which caches of a group flush when, with which rows,
and the errors raised before anything is launched.  The batched launch is replaced by a recorder."""
import pytest
import torch

import nvfp4_block_scaled_11_b200.kvcache as kc


class Recorder:
    """Stands in for KvAppendBatch: remembers the caches it was built over and every (first, n, t0)."""
    made = []

    def __init__(self, items, f_lo, f_hi):
        self.items, self.window, self.calls = list(items), (f_lo, f_hi), []
        Recorder.made.append(self)

    def __call__(self, first, n, t0):
        self.calls.append((list(first), list(n), list(t0)))


@pytest.fixture
def fake_batch(monkeypatch):
    Recorder.made = []
    monkeypatch.setattr(kc, "KvAppendBatch", Recorder)
    return Recorder


def _cache(H=2, D=32, capacity=64, recent=16, window=16, f=(-2, 6)):
    """A cache in the state prefill leaves (sink full, `window` tokens in the ring), on the CPU."""
    c = kc.NVFP4KVCache(1, H, D, capacity=capacity, recent=recent, f_lo=f[0], f_hi=f[1], device="cpu")
    c.prefilled, c.n_sink, c.n_window = True, 16, window
    return c


def _tok(c, v=0.0):
    return torch.full((1, c.H, 1, c.D), v, dtype=torch.bfloat16)


def test_group_flushes_full_windows_only(fake_batch):
    cs = [_cache(), _cache(window=17), _cache(H=3)]
    g = kc.NVFP4KVCacheGroup(cs)
    (b,) = fake_batch.made
    assert [it[0] is c.window and it[2] is c.codes for it, c in zip(b.items, cs)] == [True] * 3
    for step in range(40):
        g.append([_tok(c, step) for c in cs])
    # cache 1 fills a token earlier; the others are items with n = 0 in its flush and vice versa
    assert b.calls == [([0, 0, 0], [0, 16, 0], [0, 0, 0]),
                       ([0, 16, 0], [16, 0, 16], [0, 16, 0]),
                       ([16, 16, 16], [0, 16, 0], [16, 16, 16]),
                       ([16, 0, 16], [16, 0, 16], [16, 32, 16])]
    assert [(c.n_mid, c.n_window, c.head) for c in cs] == [(32, 24, 0), (32, 25, 0), (32, 24, 0)]
    # the window ring holds the newest tokens in order
    assert [v.item() for v in cs[0].recent_tokens()[0, 0, :, 0]] == [float(v) for v in range(16, 40)]


def test_group_splits_into_batches_of_64(fake_batch):
    cs = [_cache(H=1, D=16) for _ in range(70)]
    g = kc.NVFP4KVCacheGroup(cs)
    assert [len(b.items) for b in fake_batch.made] == [64, 6]
    for step in range(17):
        g.append([_tok(c) for c in cs])
    assert [len(b.calls) for b in fake_batch.made] == [1, 1]


def test_group_errors_before_any_launch(fake_batch):
    with pytest.raises(ValueError):
        kc.NVFP4KVCacheGroup([_cache(), _cache(f=(-8, 8))])          # windows differ
    cs = [_cache(capacity=16), _cache(capacity=8)]
    g = kc.NVFP4KVCacheGroup(cs)
    with pytest.raises(RuntimeError):                                # the second cache has no room
        g.append([torch.zeros((1, 2, 17, 32), dtype=torch.bfloat16)] * 2)
    assert fake_batch.made[-1].calls == [] and cs[0].n_mid == 0
    with pytest.raises(ValueError):
        g.append([torch.zeros((1, 2, 1, 32), dtype=torch.bfloat16)])  # one tensor for two caches
    with pytest.raises(ValueError):
        g.append([torch.zeros((1, 2, 1, 32), dtype=torch.bfloat16), torch.zeros((1, 2, 2, 32), dtype=torch.bfloat16)])
    fresh = kc.NVFP4KVCache(1, 2, 32, capacity=16, device="cpu")
    with pytest.raises(RuntimeError):
        kc.NVFP4KVCacheGroup([fresh]).append([torch.zeros((1, 2, 1, 32), dtype=torch.bfloat16)])


def test_append_many_is_a_one_off_group(fake_batch):
    cs = [_cache(), _cache()]
    for step in range(20):
        kc.append_many(cs, [_tok(c, step) for c in cs])
    flushes = [call for b in fake_batch.made for call in b.calls]
    assert flushes == [([0, 0], [16, 16], [0, 0])]
    assert [(c.n_mid, c.n_window, c.head) for c in cs] == [(16, 20, 16)] * 2


def test_single_cache_argument_errors_and_window_order():
    """Errors a cache raises before any launch, and the ring's token order after wrap-around."""
    with pytest.raises(ValueError):
        kc.NVFP4KVCache(1, 2, 30, capacity=8, device="cpu")                    # D not a multiple of 16
    c = kc.NVFP4KVCache(1, 2, 32, capacity=8, device="cpu")
    with pytest.raises(RuntimeError):
        c.append(torch.zeros((1, 2, 1, 32), dtype=torch.bfloat16))            # no prefill yet
    with pytest.raises(ValueError):
        c.prefill(torch.zeros((1, 2, 40, 32), dtype=torch.float32))           # not BF16
    with pytest.raises(ValueError):
        c.prefill(torch.zeros((1, 3, 40, 32), dtype=torch.bfloat16))          # heads differ
    with pytest.raises(ValueError):
        c.prefill(torch.zeros((1, 2, 31, 32), dtype=torch.bfloat16))          # fewer than sink + recent
    with pytest.raises(ValueError):
        c.prefill(torch.zeros((1, 2, 41, 32), dtype=torch.bfloat16))          # middle of 9 > capacity 8
    w = _cache(H=1, D=16, window=16)
    w.head = 16                                                               # the ring has wrapped once
    for i in range(16):
        w.window[0, 0, (16 + i) % 32, 0] = float(i)
    for i in range(5):
        w._push(torch.full((1, 1, 16), 100.0 + i, dtype=torch.bfloat16))
    got = [v.item() for v in w.recent_tokens()[0, 0, :, 0]]
    assert got == [float(i) for i in range(16)] + [100.0 + i for i in range(5)]
    assert w.length == 16 + 0 + 21


def test_group_refuses_caches_on_two_devices(fake_batch):
    """One flush is one launch on one device: a group over caches on different devices is refused before
    any batch is built (here a CPU cache and a meta-device cache stand in for two GPUs)."""
    a = _cache()
    b = kc.NVFP4KVCache(1, 2, 32, capacity=64, device="meta")
    with pytest.raises(ValueError, match="one device"):
        kc.NVFP4KVCacheGroup([a, b])
    assert fake_batch.made == []


def test_batch_refuses_items_on_two_devices(monkeypatch):
    """KvAppendBatch checks every tensor of every item against the first item's device before it builds a
    descriptor (the CUDA-tensor check is relaxed here so that CPU and meta tensors can stand in for two
    GPUs; nothing is launched)."""
    import nvfp4_block_scaled_11_b200 as nv
    monkeypatch.setattr(nv, "_cuda", lambda t, name: t)

    def item(dev, gdev=None):
        k = torch.zeros(2, 32, 32, dtype=torch.bfloat16, device=dev)
        g = torch.zeros(1, dtype=torch.float32, device=gdev or dev)
        codes = torch.zeros(2, 64, 16, dtype=torch.uint8, device=dev)
        scales = torch.zeros(2, 64, 2, dtype=torch.uint8, device=dev)
        return (k, g, codes, scales, True, False)

    with pytest.raises(ValueError, match="item 1: k_rows is on meta"):
        nv.KvAppendBatch([item("cpu"), item("meta")])
    with pytest.raises(ValueError, match="item 0: gscale is on meta"):
        nv.KvAppendBatch([item("cpu", gdev="meta")])
    assert len(nv.KvAppendBatch([item("cpu"), item("cpu")])) == 2
