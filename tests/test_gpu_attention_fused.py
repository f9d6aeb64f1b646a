"""The fused FP4-attention kernel (nvfp4_attention_fused) against the oracle, stage by stage, on the
kernel's own intermediate values (returned only when asked for, for verification):
* S: each score within the FP32-accumulation bound (D + 4) 2^-24 |alpha g_q g_k| sum_d |q_d k_d| of the
  exact product of the same NVFP4 operands;
* P~: the oracle's softmax quantizer applied to the kernel's scores gives the kernel's codes, tile-layout
  scales and row maxima bit for bit, and its row sums within the FP32 summation bound; the oracle's
  numerators summed in the call's order (per range, column block, even/odd accumulators) give the
  kernel's row sums bit for bit;
* O: each element within (Tk + 4) 2^-24 g_p g_v sum_k |p_k v_k| / l of the exact product of the oracle's
  P~ and V divided by the kernel's row sum, plus the division's rounding."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_11_b200 as nv
from oracle import oracle as O

pytestmark = pytest.mark.gpu
U = 2.0 ** -24


def _u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _inputs(H, Tq, Tk, seed, D=128):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((H, Tq, D), generator=g).to(torch.bfloat16)
    k = (torch.randn((H, Tk, D), generator=g) * 1.3).to(torch.bfloat16)
    v = torch.randn((H, Tk, D), generator=g).to(torch.bfloat16)
    return q, k, v


def _row_sums_in_call_order(s, m, causal, q_offset, splits):
    """The row sums the fused call forms, from the oracle's numerators exp(S - m) of the call's scores: per
    key range (the 64-key tiles with an allowed key of the query tile, cut into `splits` ranges), per 16-key
    column block cb of each tile, the even and odd elements summed in two FP32 accumulators tile by tile
    and added; the four column blocks added in order; the ranges added in order."""
    f = np.float32
    H, Tq, Tk = s.shape
    exp_ss = np.vectorize(lambda d: O.exp_ss(d), otypes=[np.float32])
    keys = np.arange(Tk)[None, :]
    out = np.zeros((H, Tq), np.float32)
    for h in range(H):
        for q0 in range(0, Tq, 128):
            rows = np.arange(q0, q0 + 128)
            lim = (rows + q_offset)[:, None] if causal else np.full((128, 1), Tk - 1)
            lim_cta = q0 + 127 + q_offset if causal else Tk - 1
            live = 0 if lim_cta < 0 else min(Tk // 64, lim_cta // 64 + 1)
            with np.errstate(invalid="ignore"):   # rows with no allowed key: m = -inf, every key masked
                d = (s[h, q0:q0 + 128].astype(np.float32) - m[h, q0:q0 + 128, None].astype(np.float32)).astype(np.float32)
                x = np.where(keys <= lim, exp_ss(d), f(0))
            total = np.zeros(128, np.float32)
            for sp in range(splits):
                t0, t1 = live * sp // splits, live * (sp + 1) // splits
                part = np.zeros(128, np.float32)
                for cb in range(4):
                    lo = np.zeros(128, np.float32)
                    hi = np.zeros(128, np.float32)
                    for j in range(t0, t1):
                        for kk in range(8):
                            lo = (lo + x[:, 64 * j + 16 * cb + 2 * kk]).astype(np.float32)
                            hi = (hi + x[:, 64 * j + 16 * cb + 2 * kk + 1]).astype(np.float32)
                    part = (part + (lo + hi).astype(np.float32)).astype(np.float32) if cb else (lo + hi).astype(np.float32)
                total = (total + part).astype(np.float32)
            out[h, q0:q0 + 128] = total
    return out


def _check(H, Tq, Tk, causal, q_offset, window, seed, splits=None):
    D = 128
    q, k, v = _inputs(H, Tq, Tk, seed)
    f_lo, f_hi = window
    qc, qsf, qg = nv._prologue_operand(q.cuda(), True, 0, f_lo, f_hi)
    kc, ksf, kg = nv._prologue_operand(k.cuda(), True, 0, f_lo, f_hi)
    vc, vsf, vg = nv.quantize_mma_t(v.cuda(), f_lo, f_hi)
    alpha = D ** -0.5
    out, m, l, s, pc, psf, status = nv.attention_fused(
        qc.view(H, Tq, D // 2), qsf, qg, kc.view(H, Tk, D // 2), ksf, kg, vc.view(H, D, Tk // 2), vsf, vg,
        causal, q_offset, alpha, f_lo, f_hi, verify=True, splits=splits)
    torch.cuda.synchronize()
    assert status.item() == 0
    # operands from the oracle (linear scales), to form the exact products
    rq = O.hadamard16(_u16(q).reshape(-1), dtype=O.BF16, out_dtype=O.F32)
    rk = O.hadamard16(_u16(k).reshape(-1), dtype=O.BF16, out_dtype=O.F32)
    rqc, rqs, rqg, _, _ = O.quantize(rq, f_lo, f_hi)
    rkc, rks, rkg, _, _ = O.quantize(rk, f_lo, f_hi)
    vt = np.ascontiguousarray(np.swapaxes(_u16(v).reshape(H, Tk, D), 1, 2)).reshape(-1)
    rvc, rvs, rvg, _, _ = O.quantize(vt, f_lo, f_hi, dtype=O.BF16)
    assert qg.item() == rqg and kg.item() == rkg and vg.item() == rvg
    assert np.array_equal(qc.cpu().numpy().reshape(-1), rqc) and np.array_equal(kc.cpu().numpy().reshape(-1), rkc)
    # S on the tiles the kernel forms (every tile holding an allowed key of some row of the CTA)
    s_h = s.cpu().numpy().astype(np.float64)
    s_ref = O.gemm_nt(rqc, rqs, rqg, rkc, rks, rkg, Tq, Tk, D, alpha, H)
    mag = np.stack([np.abs(O.block_values(rqc.reshape(H, -1)[h], rqs.reshape(H, -1)[h], Tq, D)) @
                    np.abs(O.block_values(rkc.reshape(H, -1)[h], rks.reshape(H, -1)[h], Tk, D)).T for h in range(H)])
    bound = (D + 4) * U * abs(alpha * float(rqg) * float(rkg)) * mag + 1e-37
    qi = np.arange(Tq)[:, None]
    cta_last = (qi // 128) * 128 + 127 + q_offset if causal else np.full_like(qi, Tk - 1)
    formed = (np.arange(Tk)[None, :] // 64) * 64 <= cta_last
    err = np.abs(s_h - s_ref)
    assert (err[:, formed] <= bound[:, formed]).all()
    # P~ from the kernel's scores
    rc, rs, rm, rl, rg = O.softmax_quantize(s.cpu().numpy(), causal, q_offset, f_lo, f_hi)
    assert np.array_equal(pc.cpu().numpy().reshape(-1), rc.reshape(-1))
    assert np.array_equal(psf.cpu().numpy(), O.scales_to_mma(rs, H, Tq, Tk // 16))
    assert np.array_equal(m.cpu().numpy(), rm.reshape(-1))
    l_g = l.cpu().numpy().astype(np.float64).reshape(H, Tq)
    assert (np.abs(l_g - rl) <= (Tk + 4) * U * rl).all()
    # ... and bit for bit the oracle's numerators summed in the call's order
    nsplit = splits if splits is not None else nv.attention_fused_splits(H, Tq, Tk)
    assert np.array_equal(l.cpu().numpy().reshape(H, Tq),
                          _row_sums_in_call_order(s.cpu().numpy(), m.cpu().numpy().reshape(H, Tq), causal, q_offset,
                                                  nsplit))
    # O; a row with no allowed key has l = 0 and O = 0 / 0 (NaN), as in the unfused chain
    d_ref = O.gemm_nt(rc, rs, rg, rvc, rvs, rvg, Tq, D, Tk, 1.0, H)
    pmag = np.stack([np.abs(O.block_values(rc.reshape(H, -1)[h], rs.reshape(H, -1)[h], Tq, Tk)) @
                     np.abs(O.block_values(rvc.reshape(H, -1)[h], rvs.reshape(H, -1)[h], D, Tk)).T for h in range(H)])
    o_h = out.cpu().numpy().astype(np.float64)
    empty = l_g == 0
    assert np.isnan(o_h[empty]).all()
    with np.errstate(divide="ignore", invalid="ignore"):
        want = d_ref / l_g[..., None]
        tol = (Tk + 4) * U * float(rg) * float(rvg) * pmag / l_g[..., None] + U * np.abs(o_h) + 1e-37
    assert (np.abs(o_h - want) <= tol)[~empty].all()
    return out


@pytest.mark.parametrize("H,Tq,Tk,causal,q_offset,window,splits", [
    (2, 128, 256, False, 0, (-2, 6), None),
    (2, 128, 256, False, 0, (-2, 6), 1),    # one range: the numerator kernel writes the result itself
    (1, 256, 512, True, 256, (-2, 6), 3),   # queries at the end of the keys; ranges of 2 and 3 tiles
    (1, 256, 256, True, 0, (-2, 6), 3),     # square causal: the first query tile has 2 live tiles, one range empty
    (2, 128, 192, True, 64, (-8, 8), 2),
    (1, 128, 64, False, 0, (0, 0), 2),      # one tile, max-scaling; the first range empty
    (1, 128, 1024, True, 896, (-2, 6), 5),  # ragged ranges of 3 and 4 tiles
    (1, 256, 192, True, -200, (-2, 6), 2),  # rows 0..199 see no key: m = -inf, l = 0, O = 0 / 0
    (2, 384, 1536, True, 1152, (-2, 6), None),   # three query tiles, the device's split count
    (3, 256, 768, False, 0, (-8, 8), 7),    # odd head count, seven ranges (a CTA's second half idle)
    (1, 512, 512, True, 0, (0, 0), 4),      # square causal over four query tiles, max-scaling
    (2, 128, 1024, True, 300, (-2, 6), 3),  # the limit inside a tile
])
def test_fused_attention_stages_match_oracle(H, Tq, Tk, causal, q_offset, window, splits):
    _check(H, Tq, Tk, causal, q_offset, window, seed=H * 1000 + Tk + Tq, splits=splits)


def test_fused_attention_split_counts_agree():
    """Every split count gives the same scores, P~, row maxima and (within the summation bound) O."""
    H, Tq, Tk, D = 1, 128, 512, 128
    q, k, v = _inputs(H, Tq, Tk, 11)
    qc, qsf, qg = nv._prologue_operand(q.cuda(), True, 0, -2, 6)
    kc, ksf, kg = nv._prologue_operand(k.cuda(), True, 0, -2, 6)
    vc, vsf, vg = nv.quantize_mma_t(v.cuda(), -2, 6)
    res = [nv.attention_fused(qc.view(H, Tq, D // 2), qsf, qg, kc.view(H, Tk, D // 2), ksf, kg,
                              vc.view(H, D, Tk // 2), vsf, vg, True, Tk - Tq, D ** -0.5, -2, 6, verify=True,
                              splits=s) for s in (1, 2, 4, 8)]
    o1 = res[0][0].cpu().double()
    for r in res[1:]:
        assert r[6].item() == 0
        assert torch.equal(r[3], res[0][3]) and torch.equal(r[4], res[0][4]) and torch.equal(r[5], res[0][5])
        assert torch.equal(r[1], res[0][1])
        assert ((r[0].cpu().double() - o1).abs() <= 1e-5 * o1.abs().max()).all()


def test_fused_attention_end_to_end_entry_point():
    """attention_fp4_fused (prologue + fused kernel) returns the fused kernel's O for the prologue's
    operands, and stays as close to float64 attention on the unquantized inputs as the unfused chain."""
    H, Tq, Tk, D = 2, 128, 512, 128
    q, k, v = _inputs(H, Tq, Tk, 7)
    o_f = nv.attention_fp4_fused(q.cuda(), k.cuda(), v.cuda(), causal=True).cpu().double()
    o_u = nv.attention_fp4(q.cuda(), k.cuda(), v.cuda(), causal=True).cpu().double()
    sf = torch.einsum("hqd,hkd->hqk", q.double(), k.double()) * D ** -0.5
    sf = sf.masked_fill(torch.arange(Tk)[None, :] > torch.arange(Tq)[:, None] + (Tk - Tq), float("-inf"))
    of = torch.einsum("hqk,hkd->hqd", torch.softmax(sf, -1), v.double())
    nae_f = ((o_f - of).abs().mean() / of.abs().mean()).item()
    nae_u = ((o_u - of).abs().mean() / of.abs().mean()).item()
    assert abs(nae_f - nae_u) < 0.01 * nae_u, (nae_f, nae_u)


def test_fused_attention_argument_errors():
    dev = "cuda"
    z8 = torch.zeros(64, dtype=torch.uint8, device=dev)
    g = torch.ones(1, dtype=torch.float32, device=dev)
    L = nv.lib()
    import ctypes
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    o = torch.zeros(128 * 128, dtype=torch.float32, device=dev)
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device=dev)
    args = lambda Tq, Tk, D, lo, hi, splits=1, wsb=1 << 20: (
        P(z8), P(z8), P(g), P(z8), P(z8), P(g), P(z8), P(z8), P(g), 1, Tq, Tk, D, ctypes.c_float(1.0), 0, 0, lo, hi,
        splits, P(ws), wsb, P(o), P(g), P(g), None, None, None, None, None)
    assert L.nvfp4_attention_fused(*args(100, 64, 128, -2, 6)) == -2     # Tq % 128
    assert L.nvfp4_attention_fused(*args(128, 48, 128, -2, 6)) == -2     # Tk % 64
    assert L.nvfp4_attention_fused(*args(128, 64, 64, -2, 6)) == -2      # D != 128
    assert L.nvfp4_attention_fused(*args(128, 64, 128, -2, 5)) == -1     # 8 offsets
    assert L.nvfp4_attention_fused(*args(128, 64, 128, -2, 6, splits=0)) == -1
    assert L.nvfp4_attention_fused(*args(128, 64, 128, -2, 6, splits=65)) == -1
    need = L.nvfp4_attention_fused_workspace_bytes(1, 128, 64, 2)
    assert need == (2 * 128 * 4 + 2 * 128 * 129 * 4 + 255) // 256 * 256 + (2 * 64 + 128) * 128 * 2
    assert L.nvfp4_attention_fused(*args(128, 64, 128, -2, 6, splits=2, wsb=need - 1)) == -2   # workspace too small
