"""FP4 attention (ScaleSearchAttention numerics, unfused) against the oracle.

* softmax_quantize_mma on host-made scores: codes, tile-layout scales, g and row maxima bit-exact
  (exp is the same published method on both sides); row sums within the FP32 summation bound.
* The whole pipeline, stage by stage and element by element: operands bit-exact; scores within the
  FP32-accumulation bound of the exact product; P~ bit-exact when the oracle is given the GPU's own
  scores (the only inputs where FP32 summation order may differ); O within the product bound of the
  exact P~ V divided by the row sum."""
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


def _rotated(x, signs):
    """The oracle's Hadamard-16 (with the sign diagonal `signs`) of a BF16 tensor, FP32 out."""
    u = _u16(x).reshape(-1)
    if signs:
        return O.hadamard16_ex(u, signs, dtype=O.BF16, out_dtype=O.F32)
    return O.hadamard16(u, dtype=O.BF16, out_dtype=O.F32)


def _check_chain(q, k, v, causal, signs=0):
    """Every stage of the GPU chain (the calls attention_fp4 makes) against the oracle, element by element:
    * Q, K (rotated) and V (quantized along the tokens) operands: codes, tile-layout scales and g bit-exact;
    * S = scale * Q K^T: each element within the FP32-accumulation bound (K + 4) 2^-24 |alpha g_q g_k|
      sum_d |q_d k_d| of the exact product of the same operands;
    * P~ from the GPU's own S: codes, tile-layout scales and row maxima bit-exact, row sums within the
      FP32 summation bound;
    * O = (P~ V) / l: each element within (Tk + 4) 2^-24 g_p g_v sum_k |p_k v_k| / l of the exact product
      divided by the GPU's row sum, plus the division's rounding (2^-24 |O|).
    Returns O."""
    H, Tq, D = q.shape
    Tk = k.shape[1]
    scale = D ** -0.5
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = nv.attention_fp4(qd, kd, vd, causal=causal, signs=signs)
    qc_g, qsf_g, qg_g = nv._prologue_operand(qd, True, signs, -2, 6)
    kc_g, ksf_g, kg_g = nv._prologue_operand(kd, True, signs, -2, 6)
    s_g = nv.gemm_nt(qc_g, qsf_g, qg_g, kc_g, ksf_g, kg_g, alpha=scale)
    pc_g, psf_g, pg_g, pm_g, pl_g = nv.softmax_quantize_mma(s_g, causal, Tk - Tq)
    vc_g, vsf_g, vg_g = nv.quantize_mma_t(vd)
    d_g = nv.gemm_nt(pc_g, psf_g, pg_g, vc_g, vsf_g, vg_g)
    o_chain = nv.rows_divide(d_g.clone(), pl_g)
    torch.cuda.synchronize()
    assert torch.equal(o, o_chain)                       # attention_fp4 is exactly this chain

    # operands
    qc, qs, qg, _, _ = O.quantize(_rotated(q, signs))
    kc, ks, kg, _, _ = O.quantize(_rotated(k, signs))
    assert qg_g.item() == qg and kg_g.item() == kg
    assert np.array_equal(qc_g.cpu().numpy().reshape(-1), qc) and np.array_equal(kc_g.cpu().numpy().reshape(-1), kc)
    assert np.array_equal(qsf_g.cpu().numpy(), O.scales_to_mma(qs, H, Tq, D // 16))
    assert np.array_equal(ksf_g.cpu().numpy(), O.scales_to_mma(ks, H, Tk, D // 16))
    vt = np.ascontiguousarray(np.swapaxes(_u16(v).reshape(H, Tk, D), 1, 2)).reshape(-1)
    vcodes, vscales, vg, _, _ = O.quantize(vt, dtype=O.BF16)
    assert vg_g.item() == vg and np.array_equal(vc_g.cpu().numpy().reshape(-1), vcodes)
    assert np.array_equal(vsf_g.cpu().numpy(), O.scales_to_mma(vscales, H, D, Tk // 16))

    # S
    s_h = s_g.cpu().numpy().astype(np.float64).reshape(H, Tq, Tk)
    s_ref = O.gemm_nt(qc, qs, qg, kc, ks, kg, Tq, Tk, D, scale, H)
    mag = np.stack([np.abs(O.block_values(qc.reshape(H, -1)[h], qs.reshape(H, -1)[h], Tq, D)) @
                    np.abs(O.block_values(kc.reshape(H, -1)[h], ks.reshape(H, -1)[h], Tk, D)).T for h in range(H)])
    s_bound = (D + 4) * U * abs(scale * float(qg) * float(kg)) * mag + 1e-37
    assert (np.abs(s_h - s_ref) <= s_bound).all()

    # P~ from the GPU's scores
    rc, rs, rm, rl, rg = O.softmax_quantize(s_g.cpu().numpy().reshape(H, Tq, Tk), causal, Tk - Tq)
    assert pg_g.item() == rg
    assert np.array_equal(pc_g.cpu().numpy().reshape(-1), rc.reshape(-1))
    assert np.array_equal(psf_g.cpu().numpy(), O.scales_to_mma(rs, H, Tq, Tk // 16))
    assert np.array_equal(pm_g.cpu().numpy(), rm.reshape(-1))
    l_g = pl_g.cpu().numpy().astype(np.float64).reshape(H, Tq)
    assert (np.abs(l_g - rl) <= (Tk + 4) * U * rl).all()

    # O
    d_ref = O.gemm_nt(rc, rs, rg, vcodes, vscales, vg, Tq, D, Tk, 1.0, H)
    pmag = np.stack([np.abs(O.block_values(rc.reshape(H, -1)[h], rs.reshape(H, -1)[h], Tq, Tk)) @
                     np.abs(O.block_values(vcodes.reshape(H, -1)[h], vscales.reshape(H, -1)[h], D, Tk)).T
                     for h in range(H)])
    d_bound = (Tk + 4) * U * float(rg) * float(vg) * pmag + 1e-37
    o_h = o.cpu().numpy().astype(np.float64)
    assert (np.abs(o_h - d_ref / l_g[..., None]) <= d_bound / l_g[..., None] + U * np.abs(o_h)).all()
    return o_h


@pytest.mark.parametrize("causal", [False, True])
def test_attention_fp4_pipeline_matches_oracle(causal):
    H, Tq, Tk, D = 2, 64, 256, 128
    g = torch.Generator().manual_seed(11)
    q = torch.randn((H, Tq, D), generator=g).to(torch.bfloat16)
    k = torch.randn((H, Tk, D), generator=g).to(torch.bfloat16)
    v = torch.randn((H, Tk, D), generator=g).to(torch.bfloat16)
    _check_chain(q, k, v, causal)


def test_attention_fp4_sign_diagonal_matches_oracle():
    """Q and K rotated with the same random signs (QuIP#-style diagonal before the Hadamard): the rotated
    operands equal the oracle's rotation with the same signs, and the whole chain is element-wise within
    the bounds above; the rotation keeps dot products (exact on the rotated FP32 values up to rounding)."""
    H, Tq, Tk, D = 2, 64, 256, 64
    g = torch.Generator().manual_seed(12)
    q = torch.randn((H, Tq, D), generator=g).to(torch.bfloat16)
    k = torch.randn((H, Tk, D), generator=g).to(torch.bfloat16)
    v = torch.randn((H, Tk, D), generator=g).to(torch.bfloat16)
    signs = 0x5A93
    qr = nv.hadamard16(q.cuda(), out_dtype=torch.float32, signs=signs)
    assert np.array_equal(qr.cpu().numpy().reshape(-1), _rotated(q, signs))
    _check_chain(q, k, v, True, signs)


def test_attention_fp4_quantization_error():
    """Not a parity check: the accuracy of NVFP4 attention (Q, K, V and P~ all quantized) against
    float64 attention on the unquantized inputs, the figure the design notes report (about 17 %)."""
    H, Tq, Tk, D = 2, 64, 256, 128
    g = torch.Generator().manual_seed(11)
    q = torch.randn((H, Tq, D), generator=g).to(torch.bfloat16)
    k = torch.randn((H, Tk, D), generator=g).to(torch.bfloat16)
    v = torch.randn((H, Tk, D), generator=g).to(torch.bfloat16)
    o = nv.attention_fp4(q.cuda(), k.cuda(), v.cuda(), causal=True).cpu().double()
    sf = torch.einsum("hqd,hkd->hqk", q.double(), k.double()) * D ** -0.5
    sf = sf.masked_fill(torch.arange(Tk)[None, :] > torch.arange(Tq)[:, None] + (Tk - Tq), float("-inf"))
    of = torch.einsum("hqk,hkd->hqd", torch.softmax(sf, -1), v.double())
    nae = ((o - of).abs().mean() / of.abs().mean()).item()
    assert 0.05 < nae < 0.25, nae


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
