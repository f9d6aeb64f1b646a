"""The seeded synthetic inputs follow the stated recipes (shape, distribution, structure) and are
reproducible; CPU only, at reduced sizes where a recipe allows it."""
import math

import torch

from nvfp4_block_scaled_11_b200 import workloads as W


def test_act_f32_is_standard_normal():
    x = W.act_f32("cpu")
    assert x.shape == (1024, 4096) and x.dtype == torch.float32
    assert abs(x.mean().item()) < 0.01 and abs(x.std().item() - 1.0) < 0.01
    assert torch.equal(x, W.act_f32("cpu"))


def test_act_bf16_heavy_tails_and_outlier_columns():
    x = W.act_bf16("cpu", scale=64 / 8192).float()                   # 64 rows of the recipe
    assert x.shape == (64, 8192)
    col = x.abs().mean(0)
    out = col > 5 * col.median()
    assert out.sum().item() == 82                                     # 1 % of 8192 columns
    inner = x[:, ~out]
    # 0.5 * Student-t(3): median |x| = 0.5 * 0.765, and far more mass beyond 5 sigma than a normal
    assert abs(inner.abs().median().item() - 0.5 * 0.7649) < 0.02
    assert (inner.abs() > 2.5).float().mean().item() > 1e-3
    ratio = col[out].mean() / col[~out].mean()
    assert 15 < ratio.item() < 25                                     # the x20 outlier gain
    assert torch.equal(W.act_bf16("cpu", scale=64 / 8192), W.act_bf16("cpu", scale=64 / 8192))


def test_kv_keys_bias_channels():
    k = W.kv_bf16("cpu", scale=2048 / 32768).float()                  # [1, 8, 2048, 128]
    assert k.shape == (1, 8, 2048, 128)
    means = k[0].mean(1)                                              # [heads, channels]
    biased = means.abs() > 0.2
    # 4 biased channels per head, b ~ N(0, 2): with this seed one |b| is 0.03, below what 2048 tokens
    # resolve, so 3 stand out -- the same 3 in every head
    assert biased.sum(1).tolist() == [3] * 8
    assert bool((biased == biased[0]).all())
    assert (means.abs() > 0.1).sum(1).max().item() <= 4
    other = k[0][:, :, ~biased[0]]
    assert abs(other.std().item() - 1.0) < 0.02
    d = W.kv_decode_keys("cpu", n=2048).float()                       # decode keys: same channels and biases
    dm = d.mean(1)
    assert bool(((dm.abs() > 0.2) == biased).all())
    assert torch.allclose(dm[:, biased[0]], means[:, biased[0]], atol=0.1)


def test_stream_mixture_moments():
    x = W.stream_f32("cpu", scale=(1 << 21) / (1 << 30))
    assert x.numel() == 1 << 21
    assert abs(x.var().item() - 2.5) < 0.05                           # 0.9 * 1 + 0.1 * 16
    # P(|x| > 4) = 0.9 * P(|N(0,1)| > 4) + 0.1 * P(|N(0,1)| > 1)
    want = 0.9 * math.erfc(4 / math.sqrt(2)) + 0.1 * math.erfc(1 / math.sqrt(2))
    assert abs((x.abs() > 4).float().mean().item() - want) < 0.002
    assert not torch.equal(x[:1000], W.stream_f32("cpu", scale=(1 << 21) / (1 << 30), shard=1)[:1000])


def test_bev_levels_and_gains():
    v = W.bev_f16("cpu", scale=1 / 6).float()                         # one camera
    assert v.shape == (1, sum(h * w for h, w in W.LEVELS), 8, 32)
    start = 0
    for lvl, (h, w) in enumerate(W.LEVELS):
        s = v[:, start:start + h * w].std().item()
        assert abs(s / (1 << lvl) - 1.0) < 0.05, (lvl, s)
        start += h * w


def test_msda_inputs_shapes_and_weights():
    loc, w = W.msda_inputs("cpu", scale=0.01)
    assert loc.shape == (6, 100, 8, 4, 4, 2) and w.shape == (6, 100, 8, 4, 4)
    assert float(loc.min()) >= -0.05 and float(loc.max()) <= 1.05
    assert torch.allclose(w.sum((-1, -2)), torch.ones(6, 100, 8), atol=1e-5)
