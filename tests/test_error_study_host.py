"""The error study's host-side sums (float64, chunked) equal numpy's on CPU tensors."""
import numpy as np
import torch

from nvfp4_block_scaled_11_b200 import error_study as E


def test_error_sums_are_chunked_float64(monkeypatch):
    monkeypatch.setattr(E, "CHUNK", 1000)                         # several chunks and a ragged last one
    g = torch.Generator().manual_seed(5)
    x = torch.randn(10_007, generator=g) * 3
    xh = (x + torch.randn(10_007, generator=g) * 0.1).to(torch.bfloat16).float()
    se, ae, ax = E._errors(x, xh)
    a, b = x.numpy().astype(np.float64), xh.numpy().astype(np.float64)
    assert np.isclose(se, ((b - a) ** 2).sum(), rtol=1e-12)
    assert np.isclose(ae, np.abs(b - a).sum(), rtol=1e-12)
    assert np.isclose(ax, np.abs(a).sum(), rtol=1e-12)
