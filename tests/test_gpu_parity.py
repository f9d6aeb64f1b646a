"""GPU parity: libnvfp4 (through its C ABI) against the CPU oracle, element by element.

The bar is bit-exact for everything: codes, scale bytes, the tensor scale g, the chosen offsets and
the FP32 block SSEs (NaN compared as NaN).  Aggregate MSE statistics agree to 1e-6 relative."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_11_b200 as nv
from nvfp4_block_scaled_11_b200 import workloads as W
from oracle import oracle as O

pytestmark = pytest.mark.gpu

DT_CODE = {torch.float32: O.F32, torch.bfloat16: O.BF16, torch.float16: O.F16}


def host_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.float32:
        return t.numpy().reshape(-1)
    return t.view(torch.int16).numpy().view(np.uint16).reshape(-1)


def same_f32(a, b):
    a = np.asarray(a, np.float32).reshape(-1)
    b = np.asarray(b, np.float32).reshape(-1)
    nan = np.isnan(a)
    return np.array_equal(nan, np.isnan(b)) and np.array_equal(a[~nan].view(np.uint32), b[~nan].view(np.uint32))


def check_quantize(x: torch.Tensor, f_lo=-2, f_hi=6, gscale_in=None):
    xc = x if x.is_cuda else x.cuda()  # device views keep their (mis)alignment
    gin = None if gscale_in is None else torch.tensor([gscale_in], dtype=torch.float32, device="cuda")
    codes, scales, g, bf, bs = nv.quantize_ex(xc, f_lo, f_hi, gscale_in=gin)
    if g is None:  # an external tensor scale is used as given
        g = gin
    torch.cuda.synchronize()
    xn = host_np(x)
    rc, rs, rg, rbf, rbs = O.quantize(xn, f_lo, f_hi, dtype=DT_CODE[x.dtype], gscale_in=gscale_in)
    assert same_f32(g.cpu().numpy(), [rg]), (g.item(), rg)
    assert np.array_equal(scales.cpu().numpy(), rs), "scale bytes differ"
    assert np.array_equal(bf.cpu().numpy(), rbf), "chosen offsets differ"
    assert np.array_equal(codes.cpu().numpy(), rc), "codes differ"
    assert same_f32(bs.cpu().numpy(), rbs), "block SSE differs"
    # the plain entry point gives the same codes/scales/g
    c2, s2, g2 = nv.quantize(xc, f_lo, f_hi)
    if gscale_in is None:
        assert torch.equal(c2, codes) and torch.equal(s2, scales) and same_f32(g2.cpu().numpy(), [rg])
    return codes, scales, g, rbs


SMALL = {
    "act_f32": 1 / 16,      # [64, 4096]
    "act_bf16": 1 / 64,     # [128, 8192]
    "stream_f32": 2 ** -10,  # 2^20 elements
    "bev_f16": 1 / 6,       # one camera
}


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("window", [(-2, 6), (0, 0), (-8, 8)])
def test_quantize_small_workloads(name, window):
    w = W.make(name, "cpu", SMALL[name])
    check_quantize(w.x, *window)


def test_mse_reduction_statistic():
    x = W.make("act_bf16", "cpu", 1 / 64).x
    _, _, _, bs = check_quantize(x, -2, 6)
    xc = x.cuda()
    *_, bs0 = nv.quantize_ex(xc, 0, 0)
    gpu_ss = nv.quantize_ex(xc, -2, 6)[4].double().sum().item()
    gpu_s0 = bs0.double().sum().item()
    ref_ss = bs.astype(np.float64).sum()
    assert abs(gpu_ss - ref_ss) <= 1e-6 * ref_ss
    assert gpu_ss < gpu_s0


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_dequantize_round_trip(out_dtype):
    x = W.make("stream_f32", "cpu", 2 ** -10).x
    codes, scales, g, _ = check_quantize(x)
    out = nv.dequantize(codes, scales, g, out_dtype)
    ref = O.dequantize(codes.cpu().numpy(), scales.cpu().numpy(), g.item(), DT_CODE[out_dtype])
    got = host_np(out)
    if out_dtype == torch.float32:
        assert same_f32(got, ref)
    else:
        assert np.array_equal(got, ref)


def test_dequantize_poison_and_zero_scales():
    codes = torch.tensor([0x98, 0x21] * 4 + [0] * 8, dtype=torch.uint8, device="cuda")
    scales = torch.tensor([0x7F, 0x00], dtype=torch.uint8, device="cuda")
    g = torch.tensor([1.0], device="cuda")
    out = nv.dequantize(codes, scales, g).cpu().numpy()
    assert np.all(np.isnan(out[:16]))
    assert np.all(out[16:] == 0)
    ref = O.dequantize(codes.cpu().numpy(), scales.cpu().numpy(), 1.0)
    assert np.array_equal(np.signbit(out[16:]), np.signbit(ref[16:]))


@pytest.mark.parametrize("rotate", [True, False])
def test_kv_mixed_small(rotate):
    k = W.kv_bf16("cpu", scale=96 / 32768, heads=2)
    so, ro, codes, scales, g = nv.kv_mixed(k.cuda(), 16, 16, rotate)
    torch.cuda.synchronize()
    rso, rro, rc, rs, rg = O.kv_mixed(host_np(k).reshape(k.shape), 16, 16, int(rotate))
    assert np.array_equal(host_np(so), rso.reshape(-1))
    assert np.array_equal(host_np(ro), rro.reshape(-1))
    assert same_f32(g.cpu().numpy(), [rg])
    assert np.array_equal(scales.cpu().numpy().reshape(-1), rs.reshape(-1))
    assert np.array_equal(codes.cpu().numpy().reshape(-1), rc.reshape(-1))


def test_kv_mixed_degenerate_windows():
    k = W.kv_bf16("cpu", scale=64 / 32768, heads=1)
    # no sink / recent tokens, and a cache that is only sink + recent
    for sink, recent in ((0, 0), (16, 48), (32, 32)):
        so, ro, codes, scales, g = nv.kv_mixed(k.cuda(), sink, recent, True)
        torch.cuda.synchronize()
        rso, rro, rc, rs, rg = O.kv_mixed(host_np(k).reshape(k.shape), sink, recent, 1)
        assert same_f32(g.cpu().numpy(), [rg])
        assert np.array_equal(codes.cpu().numpy().reshape(-1), rc.reshape(-1))
        assert np.array_equal(host_np(so), rso.reshape(-1)) and np.array_equal(host_np(ro), rro.reshape(-1))


@pytest.mark.parametrize("din", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("dout", [torch.float32, torch.bfloat16, torch.float16])
def test_hadamard16(din, dout):
    x = (torch.randn(4096 * 16 + 16 * 7, generator=torch.Generator().manual_seed(9)) * 3).to(din)
    out = nv.hadamard16(x.cuda(), dout)
    ref = O.hadamard16(host_np(x), dtype=DT_CODE[din], out_dtype=DT_CODE[dout])
    got = host_np(out)
    assert same_f32(got, ref) if dout == torch.float32 else np.array_equal(got, ref)


@pytest.mark.parametrize("din,dout", [(torch.float32, torch.float32), (torch.bfloat16, torch.float32),
                                      (torch.float16, torch.bfloat16)])
@pytest.mark.parametrize("signs", [0x0001, 0xA5C3, 0xFFFF])
@pytest.mark.parametrize("inverse", [False, True])
def test_hadamard16_signs(din, dout, signs, inverse):
    x = (torch.randn(4096 * 16 + 16 * 7, generator=torch.Generator().manual_seed(signs)) * 3).to(din)
    x[5] = float("nan")                          # a NaN group: all 16 outputs NaN (payloads may differ)
    out = nv.hadamard16(x.cuda(), dout, signs=signs, inverse=inverse)
    ref = O.hadamard16_ex(host_np(x), signs, inverse, dtype=DT_CODE[din], out_dtype=DT_CODE[dout])
    got = host_np(out)
    if dout == torch.float32:
        assert same_f32(got, ref)
    else:
        nan_g, nan_r = (got & 0x7FFF) > 0x7F80, (ref & 0x7FFF) > 0x7F80
        assert np.array_equal(nan_g, nan_r) and nan_r[:16].all() and np.array_equal(got[~nan_g], ref[~nan_r])


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("n", [0, 1, 7, 15, 16, 33, 1000, 4096 * 1024 + 13])
def test_tensor_amax(dtype, n):
    x = torch.randn(n + 8, generator=torch.Generator().manual_seed(n)).to(dtype)
    xg = x.cuda()
    for off in (0, 16 // x.element_size()):  # 32-byte aligned (256-bit loads) and 16-byte aligned views
        xs = x[off:off + n]
        xc = xg[off:off + n]
        a = nv.tensor_amax(xc).item()
        ref = O.tensor_amax(host_np(xs), DT_CODE[dtype]) if n else 0.0
        assert a == ref
    if n >= 16:
        y = x[:n].clone()
        y[n // 2] = float("inf")
        assert nv.tensor_amax(y.cuda()).item() == float("inf")
        y[n // 3] = float("nan")
        assert np.isnan(nv.tensor_amax(y.cuda()).item())


def test_edge_blocks():
    rows = []
    rows.append(np.zeros(16, np.float32))
    z = np.zeros(16, np.float32)
    z[1::2] = -0.0
    rows.append(z)
    rows.append(np.full(16, 3.0, np.float32))
    rows.append(np.array([1e-30] + [0] * 15, np.float32))
    rows.append(np.linspace(-1, 1, 16).astype(np.float32))
    rows.append(np.array([1000.0] + [1e-3] * 15, np.float32))
    x = torch.from_numpy(np.concatenate(rows))
    for window in ((-2, 6), (0, 0), (1, 5), (-8, -1), (-126, 126)):
        check_quantize(x, *window)
    # one block
    check_quantize(torch.from_numpy(rows[4]))
    # external tensor scales: normal, tiny (subnormal scale codes), zero (no usable candidate),
    # small (saturated default code), subnormal g
    for gin in (1.0, 1e-3, 0.0, 1e-8, 1e-40, 3.0e5):
        check_quantize(x, -2, 6, gscale_in=gin)
        check_quantize(x, 0, 4, gscale_in=gin)


def test_nonfinite_inputs_poison_in_band():
    x = torch.randn(16 * 64, generator=torch.Generator().manual_seed(3))
    for bad in (float("nan"), float("inf"), float("-inf")):
        y = x.clone()
        y[100] = bad
        codes, scales, g, _ = check_quantize(y)
        assert np.all(scales.cpu().numpy() == 0x7F)
        assert np.all(codes.cpu().numpy() == 0)
    # with an external finite g only the block holding the bad value is poisoned
    y = x.clone()
    y[100] = float("nan")
    codes, scales, g, _ = check_quantize(y, gscale_in=0.002)
    s = scales.cpu().numpy()
    assert s[100 // 16] == 0x7F and np.sum(s == 0x7F) == 1
    for gin in (float("nan"), float("inf"), -1.0):
        check_quantize(x, gscale_in=gin)


def test_unaligned_and_ragged_inputs():
    base = torch.randn(16 * 100003 + 16, generator=torch.Generator().manual_seed(4))
    xc = base.cuda()
    # a 16-byte but not 32-byte aligned view exercises the 128-bit load path
    v = xc[4:4 + 16 * 100003]
    assert v.data_ptr() % 32 == 16
    check_quantize(v)
    hb = base.to(torch.bfloat16).cuda()
    check_quantize(hb[8:8 + 16 * 100003])
    with pytest.raises(nv.NVFP4Error) as e:
        nv.quantize(xc[2:2 + 160])
    assert e.value.status == -3
    with pytest.raises(nv.NVFP4Error) as e:
        nv.quantize(xc[:100])
    assert e.value.status == -2


def test_e2m1_encode_sweep_through_max_scaling():
    """With g = 1 and every block's largest element 6, the default scale is exactly 1 (d = r = 1), so the
    codes are the hardware E2M1 encode of the raw values: sweep all float32 in [2^-7, 6] of both signs."""
    m = np.arange(1 << 23, dtype=np.uint32)
    vals = []
    for e in range(120, 130):
        v = ((np.uint32(e) << np.uint32(23)) | m).view(np.float32)
        vals.append(v[v <= 6.0])
    v = np.concatenate(vals + [np.array([0.0, -0.0, 1e-45, -1e-45], np.float32)])
    v = np.concatenate([v, -v])
    nb = (v.size + 14) // 15
    blk = np.zeros((nb, 16), np.float32)
    blk[:, 0] = 6.0
    flat = np.zeros(nb * 15, np.float32)
    flat[: v.size] = v
    blk[:, 1:] = flat.reshape(nb, 15)
    x = torch.from_numpy(blk.reshape(-1))
    codes, scales, g, bf, bs = nv.quantize_ex(x.cuda(), 0, 0, gscale_in=torch.ones(1, device="cuda"))
    assert np.all(scales.cpu().numpy() == 0x38)  # E4M3 code of 1.0
    c = codes.cpu().numpy()
    nib = np.stack([c & 0xF, c >> 4], -1).reshape(nb, 16)[:, 1:].reshape(-1)[: v.size]
    assert np.array_equal(nib, O.e2m1_encode(v))


def test_e4m3_encode_sweep_through_default_scale():
    """With g = 1 the scale byte of max-scaling is E4M3(fl(amax_b / 6)): sweep amax_b across every E4M3
    rounding boundary (subnormal and normal) and a dense grid, compare with the oracle."""
    vals = np.arange(1, 127, dtype=np.uint8)
    import ml_dtypes as md
    e4 = vals.view(md.float8_e4m3fn).astype(np.float32)
    mids = (e4[:-1] + e4[1:]) / 2
    pts = np.concatenate([e4, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9), [448.0, 460, 464, 470, 1e4]])
    pts = np.concatenate([pts, np.geomspace(1e-4, 500, 200000).astype(np.float32)]).astype(np.float32)
    amax_b = (pts * np.float32(6.0)).astype(np.float32)
    blk = np.zeros((amax_b.size, 16), np.float32)
    blk[:, 0] = amax_b
    blk[:, 1] = amax_b * np.float32(0.3)
    check_quantize(torch.from_numpy(blk.reshape(-1)), 0, 0, gscale_in=1.0)


FULL = ["act_f32", "act_bf16", "kv_bf16", "stream_f32", "bev_f16"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled(name):
    """Full-size workloads in the benchmark's launch configuration: g exact, sampled blocks exact."""
    torch.cuda.empty_cache()
    w = W.make(name, "cuda")
    rng = np.random.default_rng(11)
    if w.kind == "kv":
        so, ro, codes, scales, g = nv.kv_mixed(w.x, 16, 16, True)
        torch.cuda.synchronize()
        k = w.x
        B, H, T, D = k.shape
        mid = k[:, :, 16:T - 16].contiguous()
        xh = host_np(mid)
        rot = O.hadamard16(xh, dtype=O.BF16)
        rg = O.global_scale(O.tensor_amax(rot))
        assert same_f32(g.cpu().numpy(), [rg])
        nb = rot.size // 16
        idx = np.unique(np.concatenate([[0, nb - 1], rng.integers(0, nb, 4096)]))
        sel = rot.reshape(-1, 16)[idx]
        rc, rs, _, _ = O.quantize_blocks(sel.reshape(-1), 0, idx.size, rg, -2, 6)
        assert np.array_equal(scales.reshape(-1)[torch.from_numpy(idx).cuda()].cpu().numpy(), rs)
        assert np.array_equal(codes.reshape(-1, 8)[torch.from_numpy(idx).cuda()].cpu().numpy().reshape(-1), rc)
        assert torch.equal(so, k[:, :, :16]) and torch.equal(ro, k[:, :, -16:])
        return
    x = w.x.reshape(-1)
    codes, scales, g = nv.quantize(x, w.f_lo, w.f_hi)
    torch.cuda.synchronize()
    xh = host_np(x)
    rg = O.global_scale(O.tensor_amax(xh, DT_CODE[x.dtype]))
    assert same_f32(g.cpu().numpy(), [rg])
    nb = x.numel() // 16
    idx = np.unique(np.concatenate([[0, nb - 1], rng.integers(0, nb, 8192)]))
    sel = xh.reshape(-1, 16)[idx].reshape(-1)
    rc, rs, _, _ = O.quantize_blocks(np.ascontiguousarray(sel), 0, idx.size, rg, w.f_lo, w.f_hi, dtype=DT_CODE[x.dtype])
    ti = torch.from_numpy(idx).cuda()
    assert np.array_equal(scales[ti].cpu().numpy(), rs)
    assert np.array_equal(codes.view(-1, 8)[ti].cpu().numpy().reshape(-1), rc)
    # dequantize at full size: sampled blocks equal the oracle's dequantize of the same codes
    out = nv.dequantize(codes, scales, g, torch.float32)
    rd = O.dequantize(codes.view(-1, 8)[ti].cpu().numpy().reshape(-1), rs, rg)
    assert same_f32(out.view(-1, 16)[ti].cpu().numpy(), rd)
    del out
    # the fused round trip in the same configuration: codes, scales and g byte-equal to the two passes;
    # sampled blocks of its output equal the oracle's dequantize in the input's dtype
    fo, fc, fs, fg = nv.quantize_dequantize(x, w.f_lo, w.f_hi)
    assert torch.equal(fc, codes) and torch.equal(fs, scales) and torch.equal(fg, g)
    rdx = O.dequantize(codes.view(-1, 8)[ti].cpu().numpy().reshape(-1), rs, rg, out_dtype=DT_CODE[x.dtype])
    got = host_np(fo.view(-1, 16)[ti])
    assert same_f32(got, rdx) if x.dtype == torch.float32 else np.array_equal(got.reshape(-1), rdx.reshape(-1))


def test_many_blocks_with_natural_near_ties():
    """2^20 blocks: about 0.1% of them have a runner-up within 2e-4 of the best score, which exercises
    the fast score's certification and its fall back to the definition."""
    x = W.stream_f32("cpu", 2 ** -6)
    check_quantize(x, -2, 6)
    check_quantize(x, -8, 8)


def test_exact_ties_on_dyadic_blocks():
    """Dyadic values with a power-of-two tensor scale make many candidates' SSEs exactly equal; the
    definition's tie rule (smaller |f|, then smaller f) must decide."""
    rng = np.random.default_rng(21)
    vals = rng.integers(-24, 25, size=(1 << 16, 16)) / 8.0
    vals[:, 0] = np.where(rng.random(1 << 16) < 0.5, 3.0, -3.0)
    x = torch.from_numpy(vals.astype(np.float32).reshape(-1))
    for gin in (2.0 ** -6, 2.0 ** -8, 3.0 * 2.0 ** -9):
        check_quantize(x, -2, 6, gscale_in=gin)
        check_quantize(x, -8, 8, gscale_in=gin)


def test_certificate_blocks_on_the_thread_per_block_kernel():
    """The adversarial blocks of tests/golden/certificate_blocks.txt (the fast score orders the two best
    candidates against the definition, or breaks a definition tie, or sits at the edge of the covered
    magnitude range) through the thread-per-block kernel (launch policy forced), each group of blocks
    sharing a tensor scale and window interleaved with ordinary blocks so that they sit in warps whose
    other lanes are decided by the fast score: codes, scales, offsets and SSE bit-exact."""
    from tests import certblocks
    rows = certblocks.load()
    groups = {}
    for kind, g, f_lo, nc, x in rows:
        groups.setdefault((float(g), f_lo, nc), []).append(x)
    prev = nv.search_policy(0, 0)
    try:
        rng = np.random.default_rng(9)
        for (g, f_lo, nc), blocks in groups.items():
            adv = np.stack(blocks)
            fill = (rng.standard_normal((31 * len(blocks), 16)) * np.abs(adv).max() / 3).astype(np.float32)
            allb = np.empty((32 * len(blocks), 16), np.float32)
            allb[::32] = adv
            rest = np.ones(len(allb), bool)
            rest[::32] = False
            allb[rest] = fill
            check_quantize(torch.from_numpy(allb.reshape(-1)), f_lo, f_lo + nc - 1, gscale_in=g)
    finally:
        nv.search_policy(*prev)
