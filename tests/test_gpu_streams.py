"""Calls on different CUDA streams with different outputs do not interfere: the library keeps no
scratch between or during calls (a quantize call's amax accumulates in its own gscale word)."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_11_b200 as nv
from oracle import oracle as O

pytestmark = pytest.mark.gpu


def test_concurrent_streams_quantize_independently():
    g = torch.Generator().manual_seed(17)
    xs = [torch.randn(1 << 20, generator=g) * s for s in (1.0, 37.0, 1e-3, 5e4)]
    ref = [O.quantize(x.numpy(), -2, 6)[:3] for x in xs]
    streams = [torch.cuda.Stream() for _ in range(2)]
    dev = [x.cuda() for x in xs]
    torch.cuda.synchronize()
    outs = []
    for rep in range(8):                        # interleave the four tensors over two streams, repeatedly
        for i, x in enumerate(dev):
            with torch.cuda.stream(streams[(i + rep) % 2]):
                c, s, gs = nv.quantize(x, -2, 6)
                d = nv.dequantize(c, s, gs)
                outs.append((i, c, s, gs, d))
    torch.cuda.synchronize()
    for i, c, s, gs, d in outs:
        rc, rs, rg = ref[i]
        assert gs.item() == rg
        assert np.array_equal(c.cpu().numpy(), rc) and np.array_equal(s.cpu().numpy(), rs)
        assert np.array_equal(d.cpu().numpy().view(np.uint32), O.dequantize(rc, rs, rg).view(np.uint32))


def test_concurrent_streams_mma_layout_and_product():
    g = torch.Generator().manual_seed(18)
    a = [torch.randn(256, 512, generator=g) * (k + 1) for k in range(3)]
    b = torch.randn(128, 512, generator=g)
    bc, bsf, bg = nv.quantize_mma(b.cuda())
    streams = [torch.cuda.Stream() for _ in range(3)]
    res = []
    torch.cuda.synchronize()
    for k in range(3):
        with torch.cuda.stream(streams[k]):
            ac, asf, ag = nv.quantize_mma(a[k].cuda())
            res.append((ac, asf, ag, nv.gemm_nt(ac, asf, ag, bc, bsf, bg)))
    torch.cuda.synchronize()
    for k in range(3):
        ac, asf, ag, d = res[k]
        rc, rsf, rg = O.quantize_mma(a[k].numpy())
        assert ag.item() == rg
        assert np.array_equal(ac.cpu().numpy().reshape(-1), rc) and np.array_equal(asf.cpu().numpy(), rsf)
        d_seq = nv.gemm_nt(ac, asf, ag, bc, bsf, bg)          # the same product, alone
        assert torch.equal(d, d_seq)


def test_dequantize_footprint_and_chunked_overlap_are_identical():
    g = torch.Generator().manual_seed(19)
    x = (torch.randn(1 << 22, generator=g) * 3).cuda()
    codes, scales, gs = nv.quantize(x)
    ref = nv.dequantize(codes, scales, gs)
    for cps in (1, 2, 8):
        assert torch.equal(nv.dequantize(codes, scales, gs, ctas_per_sm=cps), ref)
    with pytest.raises(nv.NVFP4Error):
        nv.dequantize(codes, scales, gs, ctas_per_sm=9)
    # search chunk i+1 on the main stream while chunk i is dequantized on a second one
    n, nch = x.numel(), 4
    c = n // nch
    c2, s2, d2 = torch.empty_like(codes), torch.empty_like(scales), torch.empty_like(ref)
    main, aux = torch.cuda.current_stream(), torch.cuda.Stream()
    for i in range(nch):
        nv.quantize_ex(x[i * c:(i + 1) * c], gscale_in=gs, want_f=False, want_sse=False,
                       codes=c2[i * c // 2:(i + 1) * c // 2], scales=s2[i * c // 16:(i + 1) * c // 16], gscale=None)
        ev = torch.cuda.Event()
        ev.record(main)
        aux.wait_event(ev)
        with torch.cuda.stream(aux):
            nv.dequantize(c2[i * c // 2:(i + 1) * c // 2], s2[i * c // 16:(i + 1) * c // 16], gs,
                          out=d2[i * c:(i + 1) * c], ctas_per_sm=2)
    torch.cuda.synchronize()
    assert torch.equal(c2, codes) and torch.equal(s2, scales) and torch.equal(d2, ref)
