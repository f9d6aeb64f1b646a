"""Every entry point writes only its outputs: each output is a view into the middle of a larger buffer
whose 512 guard bytes on either side hold 0xA5, and the guards must be intact after the call (ragged
sizes, padded tile layouts, partial KV rows).  Values are covered by the parity tests; this is about
where the kernels write."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_11_b200 as nv

pytestmark = pytest.mark.gpu
G = 512          # guard bytes on each side (a multiple of 256, so views keep the allocation's alignment)
FILL = 0xA5


class Guarded:
    def __init__(self):
        self.bufs = []

    def out(self, shape, dtype):
        """A tensor of `shape` / `dtype` inside a guarded byte buffer (contents 0xA5 as well)."""
        shape = (shape,) if isinstance(shape, int) else tuple(shape)
        nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        buf = torch.full((nbytes + 2 * G,), FILL, dtype=torch.uint8, device="cuda")
        self.bufs.append((buf, nbytes))
        return buf[G:G + nbytes].view(dtype).view(shape)

    def check(self):
        torch.cuda.synchronize()
        for i, (buf, nbytes) in enumerate(self.bufs):
            h = buf.cpu().numpy()
            assert (h[:G] == FILL).all(), f"output {i}: bytes written before the buffer"
            assert (h[G + nbytes:] == FILL).all(), f"output {i}: bytes written past the end"


def _x(shape, seed, dtype=torch.float32, scale=3.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(dtype).cuda()


def test_quantize_dequantize_hadamard_guards():
    n = 16 * 1001
    x = _x(n, 1)
    gd = Guarded()
    codes, scales, gs = gd.out(n // 2, torch.uint8), gd.out(n // 16, torch.uint8), gd.out(1, torch.float32)
    bf, sse = gd.out(n // 16, torch.int8), gd.out(n // 16, torch.float32)
    nv.quantize_ex(x, codes=codes, scales=scales, gscale=gs, block_f=bf, block_sse=sse)
    nv.dequantize(codes, scales, gs, torch.float32, out=gd.out(n, torch.float32))
    nv.dequantize(codes, scales, gs, torch.bfloat16, out=gd.out(n, torch.bfloat16), ctas_per_sm=1)
    nv.hadamard16(x, out=gd.out(n, torch.bfloat16))
    nv.hadamard16(x, out=gd.out(n, torch.float32), signs=0x3C3C, inverse=True)
    # the fused round trip, with its own outputs guarded (and the same in place on a guarded copy)
    nv.quantize_dequantize(x, codes=gd.out(n // 2, torch.uint8), scales=gd.out(n // 16, torch.uint8),
                           gscale=gd.out(1, torch.float32), out=gd.out(n, torch.float32))
    xi = gd.out(n, torch.float32)
    xi.copy_(x)
    nv.quantize_dequantize(xi, -8, 8, codes=gd.out(n // 2, torch.uint8), scales=gd.out(n // 16, torch.uint8),
                           gscale=gd.out(1, torch.float32), out=xi)
    mc, ms = gd.out(n // 2, torch.uint8), gd.out(n // 32, torch.uint8)
    nv.mxfp4_quantize(x[: n // 32 * 32], codes=mc, scales=ms)
    nv.mxfp4_dequantize(mc, ms, torch.float16, out=gd.out(n // 32 * 32, torch.float16))
    gd.check()


def test_tile_layout_guards():
    gd = Guarded()
    x = _x((3, 200, 96), 2)      # 200 rows: the second row tile is padded; 6 block columns: padded to 8
    nv.quantize_mma(x, codes=gd.out((3, 200, 48), torch.uint8), sf=gd.out(nv.sf_mma_bytes(200, 96, 3), torch.uint8),
                    gscale=gd.out(1, torch.float32))
    xt = _x((2, 64, 40), 3)      # transposed: 40 rows of 4 blocks each
    nv.quantize_mma_t(xt, codes=gd.out((2, 40, 32), torch.uint8), sf=gd.out(nv.sf_mma_bytes(40, 64, 2), torch.uint8),
                      gscale=gd.out(1, torch.float32))
    s = _x((2, 37, 96), 4, scale=2.0)
    nv.softmax_quantize_mma(s, True, 59, codes=gd.out((2, 37, 48), torch.uint8),
                            sf=gd.out(nv.sf_mma_bytes(37, 96, 2), torch.uint8), g=gd.out(1, torch.float32),
                            m=gd.out(74, torch.float32), l=gd.out(74, torch.float32))
    gd.check()


def test_gemm_and_kv_guards():
    gd = Guarded()
    ac, asf, ag = nv.quantize_mma(_x((2, 130, 64), 5))
    bc, bsf, bg = nv.quantize_mma(_x((2, 72, 64), 6))
    nv.gemm_nt(ac, asf, ag, bc, bsf, bg, out=gd.out((2, 130, 72), torch.float32), alpha_work=gd.out(1, torch.float32))
    nv.gemm_nt(ac, asf, ag, bc, bsf, bg, out_dtype=torch.bfloat16, out=gd.out((2, 130, 72), torch.bfloat16))
    k = _x((1, 2, 70, 64), 7, torch.bfloat16)
    nv.kv_mixed_mma(k, 16, 16, True, codes=gd.out((1, 2, 38, 32), torch.uint8),
                    sf=gd.out(nv.sf_mma_bytes(38, 64, 2), torch.uint8), gscale=gd.out(1, torch.float32))
    # the linear-layout call through the C ABI, every output guarded
    so, ro = gd.out((1, 2, 16, 64), torch.bfloat16), gd.out((1, 2, 16, 64), torch.bfloat16)
    kc, ks, kg = gd.out((1, 2, 38, 32), torch.uint8), gd.out((1, 2, 38, 4), torch.uint8), gd.out(1, torch.float32)
    p = lambda t: t.data_ptr()
    rc = nv.lib().nvfp4_kv_mixed(p(k), 1, 2, 70, 64, 16, 16, 1, -2, 6, p(so), p(ro), p(kc), p(ks), p(kg),
                                 torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    # append 16 tokens into rows 20..35 of a 50-row cache: the other rows and the tile padding untouched
    cap = 50
    codes = gd.out((2, cap, 32), torch.uint8)
    sf = gd.out(nv.sf_mma_bytes(cap, 64, 2), torch.uint8)
    nv.kv_append(k[0], 3, 16, kg, codes, sf, 20, tile_layout=True)
    gd.check()
    rows = codes.cpu().numpy()
    assert (rows[:, :20] == FILL).all() and (rows[:, 36:] == FILL).all()


def test_msda_guards():
    gd = Guarded()
    shapes = [(8, 10), (4, 5)]
    nk = sum(h * w for h, w in shapes)
    bs, nq, heads, ch, P = 2, 7, 2, 32, 4
    value = _x((bs, nk, heads, ch), 8, torch.float16)
    g = torch.Generator().manual_seed(9)
    loc = torch.rand((bs, nq, heads, len(shapes), P, 2), generator=g).cuda()
    w = torch.rand((bs, nq, heads, len(shapes), P), generator=g).cuda()
    nv.msda_forward(value, shapes, loc, w, out=gd.out((bs, nq, heads, ch), torch.float32))
    codes, scales, gs = nv.quantize(value.reshape(-1))
    q3 = (codes.view(bs, nk, heads, ch // 2), scales.view(bs, nk, heads, ch // 16), gs)
    nv.msda_forward(q3, shapes, loc, w, out=gd.out((bs, nq, heads, ch), torch.float32))
    gd.check()
