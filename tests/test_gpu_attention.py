"""FP4 attention (ScaleSearchAttention numerics, unfused) against the oracle.

* softmax_quantize_mma on host-made scores: codes, tile-layout scales, g and row maxima bit-exact
  (exp is the same published method on both sides); row sums within the FP32 summation bound.
* The whole pipeline: the GPU's scores come from FP32 tensor-core accumulation, the oracle's from the
  float64 product rounded once, so a softmax numerator can land on the other side of a rounding
  boundary now and then.  The test bounds how often P codes differ (< 0.5 %) and the output's
  deviation (relative Frobenius < 2e-3), far below what a wrong layout, scale or mask produces."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_11_b200 as nv
from oracle import oracle as O

pytestmark = pytest.mark.gpu
U = 2.0 ** -24


def _scores(batch, Tq, Tk, seed, scale=2.5):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn((batch, Tq, Tk), generator=g) * scale).float()


@pytest.mark.parametrize("batch,Tq,Tk,causal,q_offset,window", [
    (2, 37, 96, False, 0, (-2, 6)), (1, 130, 2048, True, 1918, (-2, 6)), (3, 8, 64, True, 0, (-2, 6)),
    (1, 64, 256, False, 0, (0, 0)), (1, 64, 256, True, 192, (-8, 8)),
    # several warps per row: 8 (ragged 75-block chunks), 4 with an odd row count (the last CTA round has
    # warps without a row), 8 with the causal limit inside a chunk, 2 with NC = 17
    (1, 5, 9600, False, 0, (-2, 6)), (3, 7, 4800, True, 4790, (-2, 6)), (1, 33, 8192, True, 4000, (-2, 6)),
    (2, 9, 2064, True, 1000, (-8, 8)),
    # square causal: whole 32-block rounds past the limit are written as zero blocks directly
    (2, 64, 1024, True, 0, (-2, 6)), (1, 96, 2048, True, 0, (-2, 6)), (1, 40, 640, True, -100, (-2, 6))])
def test_softmax_quantize_matches_oracle(batch, Tq, Tk, causal, q_offset, window):
    s = _scores(batch, Tq, Tk, Tq + Tk)
    codes, sf, g, m, l = nv.softmax_quantize_mma(s.cuda(), causal, q_offset, *window)
    torch.cuda.synchronize()
    rc, rs, rm, rl, rg = O.softmax_quantize(s.numpy(), causal, q_offset, *window)
    assert g.item() == rg
    assert np.array_equal(m.cpu().numpy(), rm.reshape(-1))
    assert np.array_equal(codes.cpu().numpy().reshape(-1), rc.reshape(-1))
    assert np.array_equal(sf.cpu().numpy(), O.scales_to_mma(rs, batch, Tq, Tk // 16))
    assert (np.abs(l.cpu().numpy() - rl.reshape(-1)) <= (Tk + 4) * U * rl.reshape(-1)).all()


def test_softmax_quantize_poisons_nan_block():
    s = _scores(1, 4, 64, 3)
    s[0, 2, 37] = float("nan")
    codes, sf, g, m, l = nv.softmax_quantize_mma(s.cuda())
    rc, rs, rm, rl, _ = O.softmax_quantize(s.numpy())
    assert np.array_equal(codes.cpu().numpy().reshape(-1), rc.reshape(-1))
    assert np.array_equal(sf.cpu().numpy(), O.scales_to_mma(rs, 1, 4, 4))
    assert rs[0, 2, 2] == 0x7F


def test_rows_divide_exact():
    g = torch.Generator().manual_seed(4)
    x = torch.randn((3, 5, 8), generator=g)
    l = torch.rand(15, generator=g) + 0.5
    y = nv.rows_divide(x.clone().cuda(), l.cuda()).cpu().numpy()
    want = (x.numpy().reshape(15, 8) / l.numpy()[:, None]).astype(np.float32)
    assert np.array_equal(y.reshape(15, 8), want)


def _u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("causal", [False, True])
def test_attention_fp4_pipeline_matches_oracle(causal):
    H, Tq, Tk, D = 2, 64, 256, 128
    g = torch.Generator().manual_seed(11)
    q = torch.randn((H, Tq, D), generator=g).to(torch.bfloat16)
    k = torch.randn((H, Tk, D), generator=g).to(torch.bfloat16)
    v = torch.randn((H, Tk, D), generator=g).to(torch.bfloat16)
    o = nv.attention_fp4(q.cuda(), k.cuda(), v.cuda(), causal=causal).cpu().numpy().astype(np.float64)
    # the oracle's pipeline
    scale = D ** -0.5
    qr = O.hadamard16(_u16(q).reshape(-1), dtype=O.BF16, out_dtype=O.F32)
    kr = O.hadamard16(_u16(k).reshape(-1), dtype=O.BF16, out_dtype=O.F32)
    qc, qs, qg, _, _ = O.quantize(qr)
    kc, ks, kg, _, _ = O.quantize(kr)
    s = O.gemm_nt(qc, qs, qg, kc, ks, kg, Tq, Tk, D, scale, H).astype(np.float32)
    pc, ps, pm, pl, pg = O.softmax_quantize(s, causal, Tk - Tq)
    vc, vsf, vg = O.quantize_mma_t(_u16(v).reshape(H, Tk, D), dtype=O.BF16)
    vcodes, vscales, _, _, _ = O.quantize(np.ascontiguousarray(np.swapaxes(_u16(v).reshape(H, Tk, D), 1, 2)).reshape(-1),
                                          dtype=O.BF16)
    ov = O.gemm_nt(pc, ps, pg, vcodes, vscales, vg, Tq, D, Tk, 1.0, H) / pl[..., None]
    # the GPU's P for the same comparison
    qc_g, qsf_g, qg_g = nv.quantize_mma(nv.hadamard16(q.cuda(), out_dtype=torch.float32))
    kc_g, ksf_g, kg_g = nv.quantize_mma(nv.hadamard16(k.cuda(), out_dtype=torch.float32))
    s_g = nv.gemm_nt(qc_g, qsf_g, qg_g, kc_g, ksf_g, kg_g, alpha=scale)
    pc_g, _, _, _, _ = nv.softmax_quantize_mma(s_g, causal, Tk - Tq)
    differ = np.mean(pc_g.cpu().numpy().reshape(-1) != pc.reshape(-1))
    assert differ < 5e-3, differ
    rel = np.linalg.norm(o - ov) / np.linalg.norm(ov)
    assert rel < 2e-3, rel
    # and against full-precision attention: the quantization error of NVFP4 attention
    qf, kf, vf = q.double(), k.double(), v.double()
    sf = torch.einsum("hqd,hkd->hqk", qf, kf) * scale
    if causal:
        sf = sf.masked_fill(torch.arange(Tk)[None, :] > torch.arange(Tq)[:, None] + (Tk - Tq), float("-inf"))
    of = torch.einsum("hqk,hkd->hqd", torch.softmax(sf, -1), vf).numpy()
    nae = np.abs(o - of).mean() / np.abs(of).mean()
    assert nae < 0.25, nae


def test_attention_fp4_sign_diagonal_keeps_the_product():
    """Q and K rotated with the same random signs: the scores are those of the unrotated inputs up to
    NVFP4 error, and the pipeline equals the oracle's with the same signs."""
    H, Tq, Tk, D = 2, 64, 256, 64
    g = torch.Generator().manual_seed(12)
    q = torch.randn((H, Tq, D), generator=g).to(torch.bfloat16)
    k = torch.randn((H, Tk, D), generator=g).to(torch.bfloat16)
    v = torch.randn((H, Tk, D), generator=g).to(torch.bfloat16)
    signs = 0x5A93
    qr = nv.hadamard16(q.cuda(), out_dtype=torch.float32, signs=signs)
    kr = nv.hadamard16(k.cuda(), out_dtype=torch.float32, signs=signs)
    assert np.array_equal(qr.cpu().numpy().reshape(-1),
                          O.hadamard16_ex(_u16(q).reshape(-1), signs, dtype=O.BF16, out_dtype=O.F32))
    s_rot = torch.einsum("hqd,hkd->hqk", qr.double(), kr.double()).cpu()
    s_ref = torch.einsum("hqd,hkd->hqk", q.double(), k.double())
    assert torch.allclose(s_rot, s_ref, rtol=0, atol=1e-4)
    o = nv.attention_fp4(q.cuda(), k.cuda(), v.cuda(), causal=True, signs=signs).cpu().double()
    sf = (s_ref * D ** -0.5).masked_fill(torch.arange(Tk)[None, :] > torch.arange(Tq)[:, None] + (Tk - Tq),
                                         float("-inf"))
    of = torch.einsum("hqk,hkd->hqd", torch.softmax(sf, -1), v.double())
    assert ((o - of).abs().mean() / of.abs().mean()).item() < 0.25


def test_softmax_quantize_full_size_sampled():
    """The attention step's softmax shape (8 heads x 2048 queries x 32768 keys, causal, queries at the end)
    in the benchmark's launch configuration (one warp per row): seeded scores made on the device, sampled
    rows against the oracle run on those rows alone."""
    H, Tq, Tk = 8, 2048, 32768
    bpr = Tk // 16
    gen = torch.Generator(device="cuda").manual_seed(23)
    s = torch.randn((H, Tq, Tk), generator=gen, device="cuda") * 2.5
    codes, sf, g, m, l = nv.softmax_quantize_mma(s, True, Tk - Tq)
    torch.cuda.synchronize()
    rng = np.random.default_rng(24)
    picks = [(0, 0), (0, Tq - 1), (7, Tq - 1), (3, 777), (5, 1)] + [
        (int(h), int(q)) for h, q in zip(rng.integers(0, H, 19), rng.integers(0, Tq, 19))]
    codes_h = codes.view(H, Tq, Tk // 2)
    sf_h = sf.cpu().numpy()
    mat = O.sf_mma_bytes(Tq, bpr)
    for h, q in picks:
        row = s[h, q].cpu().numpy()[None, None, :]
        rc, rs, rm, rl, rg = O.softmax_quantize(row, True, q + Tk - Tq)   # key k allowed iff k <= q + Tk - Tq
        assert g.item() == rg
        assert np.array_equal(codes_h[h, q].cpu().numpy(), rc.reshape(-1)), (h, q)
        offs = [h * mat + O.sf_mma_offset(q, c, bpr) for c in range(bpr)]
        assert np.array_equal(sf_h[offs], rs.reshape(-1)), (h, q)
        assert m[h * Tq + q].item() == rm.item()
        assert abs(l[h * Tq + q].item() - rl.item()) <= (Tk + 4) * U * rl.item()


def test_fused_prologue_equals_rotate_then_quantize():
    """attention_fp4's fused Q/K prologue (rotation inside the amax and search kernels) gives the same
    operand bits as rotating into FP32 and quantizing that."""
    g = torch.Generator().manual_seed(31)
    x = (torch.randn((4, 192, 128), generator=g) * 3).to(torch.bfloat16).cuda()
    x[1, 7, 5] = 40.0
    c1, s1, g1 = nv._prologue_operand(x, True, 0, -2, 6)
    c2, s2, g2 = nv.quantize_mma(nv.hadamard16(x, out_dtype=torch.float32), -2, 6)
    assert torch.equal(g1, g2) and torch.equal(c1, c2) and torch.equal(s1, s2)
