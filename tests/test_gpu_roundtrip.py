"""The fused round trip (nvfp4_quantize_dequantize) against the oracle: codes, scales and g equal the
oracle's ScaleSearch quantize, and the dequantized output equals the oracle's dequantize of those codes
in the input's dtype, for the fused windows (1, 9, 17 offsets), another width (two passes), a given
tensor scale, in place, zero and non-finite blocks and ragged sizes."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_11_b200 as nv
from oracle import oracle as O

pytestmark = pytest.mark.gpu
DT_CODE = {torch.float32: O.F32, torch.bfloat16: O.BF16, torch.float16: O.F16}


def _bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.float32:
        return t.numpy().reshape(-1).view(np.uint32)
    return t.view(torch.int16).numpy().view(np.uint16).reshape(-1)


def _host(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().reshape(-1) if t.dtype == torch.float32 else _bits(t)


def _same(got: np.ndarray, want: np.ndarray, dtype) -> bool:
    """Bit equality, NaNs compared as NaN (their payloads are not part of the definition)."""
    if dtype == torch.float32:
        g, w = got.view(np.float32), np.asarray(want, np.float32).reshape(-1)
        nan = np.isnan(g)
        return np.array_equal(nan, np.isnan(w)) and np.array_equal(got[~nan], w[~nan].view(np.uint32))
    w = np.asarray(want).reshape(-1)
    exp_mask = 0x7F80 if dtype == torch.bfloat16 else 0x7C00
    nan_g, nan_w = (got & 0x7FFF) > exp_mask, (w & 0x7FFF) > exp_mask
    return np.array_equal(nan_g, nan_w) and np.array_equal(got[~nan_g], w[~nan_w])


def _input(n, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(n, generator=g) * torch.where(torch.rand(n, generator=g) < 0.1, 4.0, 1.0)
    x[16:32] = 0.0                  # a zero block
    x[48:64] = -0.0                 # a negative-zero block: sign-only codes, -0 out
    return x.to(dtype)


def _check(x, f_lo, f_hi, gscale_in=None, inplace=False):
    xh = _host(x)
    ref_g = None if gscale_in is None else float(gscale_in.item())
    rc, rs, rg, _, _ = O.quantize(xh, f_lo, f_hi, dtype=DT_CODE[x.dtype],
                                  gscale_in=None if ref_g is None else np.float32(ref_g))
    xd = x.cuda()
    out = xd if inplace else None
    o, c, s, g = nv.quantize_dequantize(xd, f_lo, f_hi, gscale_in=None if gscale_in is None else gscale_in.cuda(),
                                        out=out)
    torch.cuda.synchronize()
    assert np.array_equal(c.cpu().numpy(), rc) and np.array_equal(s.cpu().numpy(), rs)
    if g is not None:
        gv = g.cpu().numpy()[0]
        assert np.isnan(gv) if np.isnan(rg) else gv.view(np.uint32) == np.float32(rg).view(np.uint32)
    want = O.dequantize(rc, rs, rg, out_dtype=DT_CODE[x.dtype])
    assert _same(_bits(o), want, x.dtype)
    return o, c, s


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("window", [(-2, 6), (0, 0), (-8, 8), (-1, 3)])
def test_round_trip_matches_oracle(dtype, window):
    _check(_input(16 * 20011, dtype, 3), *window)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_round_trip_given_scale_and_in_place(dtype):
    x = _input(16 * 4099, dtype, 4)
    _check(x, -2, 6, gscale_in=torch.tensor([0.0123], dtype=torch.float32))
    _check(x.clone(), -2, 6, inplace=True)


def test_round_trip_equals_two_passes_and_poisons_nonfinite():
    x = _input(16 * 65536 + 16 * 5, torch.float32, 5).cuda()
    o, c, s, g = nv.quantize_dequantize(x)
    c2, s2, g2 = nv.quantize(x)
    assert torch.equal(c, c2) and torch.equal(s, s2) and torch.equal(g, g2)
    assert torch.equal(o.view(torch.int32), nv.dequantize(c2, s2, g2).view(torch.int32))
    x[100] = float("inf")           # g becomes Inf: every block poisoned, every output NaN
    o, c, s, g = nv.quantize_dequantize(x)
    assert bool((s == 0x7F).all()) and bool(torch.isnan(o).all())
    xb = _input(16 * 999, torch.bfloat16, 6)
    xb[200] = float("nan")
    _check(xb, -2, 6)


def test_round_trip_errors():
    x = torch.randn(64, device="cuda")
    with pytest.raises(ValueError):
        nv.quantize_dequantize(x, out=torch.empty(64, dtype=torch.bfloat16, device="cuda"))
    p = lambda t: t.data_ptr()
    c, s, g = torch.empty(32, dtype=torch.uint8, device="cuda"), torch.empty(4, dtype=torch.uint8, device="cuda"), \
        torch.empty(1, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    L = nv.lib()
    assert L.nvfp4_quantize_dequantize(p(x), 64, 0, -2, 6, None, p(c), p(s), p(g), None, st) == -1
    assert L.nvfp4_quantize_dequantize(p(x), 60, 0, -2, 6, None, p(c), p(s), p(g), p(x), st) == -2
    assert L.nvfp4_quantize_dequantize(p(x), 64, 0, -2, 6, None, p(c), p(s), p(g), p(x) + 4, st) == -3


@pytest.mark.parametrize("window", [(-2, 6), (0, 0), (-8, 8), (-1, 3)])
@pytest.mark.parametrize("rotate,sink,recent", [(True, 16, 16), (False, 16, 16), (True, 0, 0), (True, 5, 27)])
def test_kv_round_trip_matches_oracle(window, rotate, sink, recent):
    """kv_mixed_dequantize: the KV layout's outputs equal the oracle's, and the middle's values equal the
    oracle's dequantize of the oracle's codes (BF16, rotated space when rotating)."""
    g = torch.Generator().manual_seed(41)
    k = torch.randn((2, 3, 200, 64), generator=g)
    k[..., 7] += 3.0                                     # an outlier channel, as in the KV recipe
    k = k.to(torch.bfloat16)
    kh = k.view(torch.int16).numpy().view(np.uint16)
    rso, rro, rc, rs, rg = O.kv_mixed(kh, sink, recent, int(rotate), *window)
    so, ro, c, s, gs, mid = nv.kv_mixed_dequantize(k.cuda(), sink, recent, rotate, *window)
    torch.cuda.synchronize()
    assert np.array_equal(c.cpu().numpy().reshape(-1), rc.reshape(-1))
    assert np.array_equal(s.cpu().numpy().reshape(-1), rs.reshape(-1))
    assert gs.cpu().numpy().view(np.uint32)[0] == np.float32(rg).view(np.uint32)
    assert np.array_equal(_bits(so), rso.reshape(-1)) and np.array_equal(_bits(ro), rro.reshape(-1))
    want = O.dequantize(rc.reshape(-1), rs.reshape(-1), rg, out_dtype=O.BF16)
    assert _same(_bits(mid), want, torch.bfloat16)
    # and the same as the two calls it fuses
    so2, ro2, c2, s2, g2 = nv.kv_mixed(k.cuda(), sink, recent, rotate, *window)
    assert torch.equal(c, c2) and torch.equal(s, s2)
    assert torch.equal(mid.view(torch.int16), nv.dequantize(c2, s2, g2, torch.bfloat16).view(mid.shape).view(torch.int16))


@pytest.mark.parametrize("mag", [1e-44, 1e-40, 1e-36, 1e-20, 1e20, 1e35, 3e38])
def test_round_trip_extreme_tensor_scales(mag):
    """Tensor scales computed from extreme tensors: g subnormal or zero (tiny inputs, subnormal ones
    included) and g near the top of the range; codes, scales, g and values against the oracle."""
    g = torch.Generator().manual_seed(int(abs(np.log10(mag))) + 7)
    x = (torch.randn(16 * 2003, generator=g, dtype=torch.float64) * mag).clamp(-3.4e38, 3.4e38).to(torch.float32)
    _check(x, -2, 6)
    _check(x, -8, 8)
    xd = x.cuda()
    c, s, gs = nv.quantize(xd)
    rc, rs, rg, _, _ = O.quantize(x.numpy(), -2, 6)
    assert np.array_equal(c.cpu().numpy(), rc) and np.array_equal(s.cpu().numpy(), rs)
