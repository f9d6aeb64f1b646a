"""MXFP4 (comparison format) through the C ABI against the oracle: bit-exact."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_11_b200 as nv
from nvfp4_block_scaled_11_b200 import workloads as W
from oracle import oracle as O

pytestmark = pytest.mark.gpu


def _host(t):
    t = t.cpu().contiguous()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def _odt(dtype):
    return {torch.float32: O.F32, torch.bfloat16: O.BF16, torch.float16: O.F16}[dtype]


def _data(kind, n, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(n, generator=g)
    if kind == "tiny":
        x = x * 1e-39
    elif kind == "huge":
        x = x * 1e37
    elif kind == "mixed":
        x = x * torch.repeat_interleave(10.0 ** (torch.rand(n // 32, generator=g) * 40 - 20), 32)
    x[:32] = 0.0
    x[64 + 5] = float("nan")
    x[96 + 9] = float("-inf")
    return x


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("kind", ["normal", "tiny", "huge", "mixed"])
def test_mxfp4_quantize_bit_exact(dtype, kind):
    if dtype == torch.float16 and kind in ("tiny", "huge", "mixed"):
        pytest.skip("outside the FP16 range")
    x = _data(kind, 32 * 4099, 7).to(dtype)           # odd block count: a ragged last wave
    c, s = nv.mxfp4_quantize(x.cuda())
    rc, rs = O.mxfp4_quantize(_host(x), _odt(dtype))
    assert np.array_equal(s.cpu().numpy(), rs)
    assert np.array_equal(c.cpu().numpy(), rc)


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_mxfp4_dequantize_bit_exact(out_dtype):
    x = _data("mixed", 32 * 2051, 8) if out_dtype != torch.float16 else _data("normal", 32 * 2051, 8)
    rc, rs = O.mxfp4_quantize(x.numpy())
    d = nv.mxfp4_dequantize(torch.from_numpy(rc).cuda(), torch.from_numpy(rs).cuda(), out_dtype)
    want = O.mxfp4_dequantize(rc, rs, _odt(out_dtype))
    got = _host(d)
    # NaN blocks (scale byte 0xFF) must be NaN at the same places; NaN bit patterns are not compared
    if out_dtype == torch.float32:
        wf = want
    else:
        wf = torch.from_numpy(want.view(np.int16)).view(out_dtype).float().numpy()
    nan = np.isnan(wf)
    assert nan.any() and np.array_equal(np.isnan(d.float().cpu().numpy()), nan)
    assert np.array_equal(got[~nan].view(np.uint8), want[~nan].view(np.uint8))


def test_mxfp4_full_size_stream_sampled():
    x = W.stream_f32("cuda")
    c, s = nv.mxfp4_quantize(x)
    torch.cuda.synchronize()
    nb = x.numel() // 32
    idx = np.unique(np.concatenate([np.random.default_rng(1).choice(nb, 4096, replace=False), [0, nb - 1]]))
    xs = x.view(nb, 32)[torch.from_numpy(idx).cuda()].cpu().numpy()
    rc, rs = O.mxfp4_quantize(xs.reshape(-1))
    assert np.array_equal(s[torch.from_numpy(idx).cuda()].cpu().numpy(), rs)
    assert np.array_equal(c.view(nb, 16)[torch.from_numpy(idx).cuda()].cpu().numpy().reshape(-1), rc)


def test_mxfp4_errors():
    x = torch.zeros(48, device="cuda")
    with pytest.raises(nv.NVFP4Error) as e:
        nv.mxfp4_quantize(x)
    assert e.value.status == -2
