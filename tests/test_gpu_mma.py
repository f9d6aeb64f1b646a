"""Parity of the tensor-core consumer path against the oracle, through the C ABI.

* quantize_mma / kv_mixed_mma: codes and tile-layout scales (padding included) bit-exact with the
  oracle's quantize + tile layout.
* gemm_nt: D = alpha g_a g_b A B^T against the oracle's fp64 product.  Every product of two E2M1 values
  and two E4M3 scales is exact, so the only error is FP32 accumulation in some order (at most
  (K - 1) u sum|a b|, u = 2^-24) and the scale multiply in the epilogue (a few u): the bound used is
  (K + 4) u |alpha g_a g_b| sum|a b|, plus one BF16 rounding (2^-8 |D|) for BF16 output.  A wrong
  scale, code or layout changes entries by O(1) relative and fails it."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_11_b200 as nv
from oracle import oracle as O

pytestmark = pytest.mark.gpu
U = 2.0 ** -24


def _x(shape, seed, dtype=torch.float32, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(dtype)


def _np(t):
    t = t.cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def _odt(t):
    return {torch.float32: O.F32, torch.bfloat16: O.BF16, torch.float16: O.F16}[t.dtype]


@pytest.mark.parametrize("shape,dtype", [((1, 128, 64), torch.float32), ((2, 200, 96), torch.bfloat16),
                                         ((3, 129, 16), torch.float16), ((1, 1, 512), torch.float32),
                                         ((1, 256, 8192), torch.bfloat16)])
def test_quantize_mma_bit_exact(shape, dtype):
    x = _x(shape, 100 + shape[1], dtype)
    codes, sf, g = nv.quantize_mma(x.cuda())
    rc, rsf, rg = O.quantize_mma(_np(x).reshape(shape), dtype=_odt(x))
    assert g.item() == rg
    assert np.array_equal(codes.cpu().numpy().reshape(-1), rc)
    assert np.array_equal(sf.cpu().numpy(), rsf)


def test_quantize_mma_external_scale_and_windows():
    x = _x((2, 130, 64), 7)
    gin = torch.tensor([0.0125], dtype=torch.float32)
    for lo, hi in ((0, 0), (-2, 6), (-8, 8), (-1, 3)):
        codes, sf, _ = nv.quantize_mma(x.cuda(), lo, hi, gscale_in=gin.cuda())
        rc, rsf, _ = O.quantize_mma(x.numpy(), lo, hi, gscale_in=0.0125)
        assert np.array_equal(codes.cpu().numpy().reshape(-1), rc), (lo, hi)
        assert np.array_equal(sf.cpu().numpy(), rsf), (lo, hi)


def test_kv_mixed_mma_matches_oracle_layout():
    B, H, T, D = 1, 2, 100, 128        # T_mid = 68: a ragged 128-row tile
    k = _x((B, H, T, D), 21, torch.bfloat16)
    so, ro, codes, sf, g = nv.kv_mixed_mma(k.cuda())
    rso, rro, rc, rs, rg = O.kv_mixed(_np(k))
    Tm = T - 32
    assert g.item() == rg
    assert np.array_equal(_np(so), rso) and np.array_equal(_np(ro), rro)
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(sf.cpu().numpy(), O.scales_to_mma(rs, B * H, Tm, D // 16))


def _gemm_bound(a_codes, a_scales, b_codes, b_scales, M, N, K, batch, s):
    A = np.asarray(a_codes).reshape(batch, -1)
    As = np.asarray(a_scales).reshape(batch, -1)
    Bc = np.asarray(b_codes).reshape(batch, -1)
    Bs = np.asarray(b_scales).reshape(batch, -1)
    out = np.empty((batch, M, N))
    for l in range(batch):
        av = np.abs(O.block_values(A[l], As[l], M, K))
        bv = np.abs(O.block_values(Bc[l], Bs[l], N, K))
        out[l] = (av @ bv.T) * abs(s)
    return out


def _check_gemm(x_a, x_b, alpha, out_dtype, batch):
    M, K = x_a.shape[-2:]
    N = x_b.shape[-2]
    ac, asf, ga = nv.quantize_mma(x_a.cuda())
    bc, bsf, gb = nv.quantize_mma(x_b.cuda())
    d = nv.gemm_nt(ac, asf, ga, bc, bsf, gb, alpha=alpha, out_dtype=out_dtype)
    torch.cuda.synchronize()
    # oracle: quantize the same inputs itself, then the fp64 product
    rac, ras, rga, _, _ = O.quantize(_np(x_a).reshape(-1), dtype=_odt(x_a))
    rbc, rbs, rgb, _, _ = O.quantize(_np(x_b).reshape(-1), dtype=_odt(x_b))
    ref = O.gemm_nt(rac, ras, rga, rbc, rbs, rgb, M, N, K, alpha, batch)
    bound = _gemm_bound(rac, ras, rbc, rbs, M, N, K, batch, float(alpha) * float(rga) * float(rgb))
    tol = (K + 4) * U * bound + 1e-37
    got = d.float().cpu().numpy().reshape(batch, M, N).astype(np.float64)
    if out_dtype == torch.bfloat16:
        tol = tol + 2.0 ** -8 * np.abs(ref)
    err = np.abs(got - ref)
    assert np.isfinite(got).all()
    assert (err <= tol).all(), float((err / np.maximum(tol, 1e-300)).max())
    return err, bound


@pytest.mark.parametrize("B,M,N,K", [(1, 256, 256, 512), (1, 200, 136, 128), (2, 384, 128, 1024),
                                     (1, 1, 8, 32), (1, 130, 264, 96), (3, 64, 72, 256)])
def test_gemm_nt_matches_oracle_f32(B, M, N, K):
    _check_gemm(_x((B, M, K), 31 + M), _x((B, N, K), 37 + N, scale=0.05), 0.75, torch.float32, B)


@pytest.mark.parametrize("B,M,N,K", [(1, 256, 128, 256), (2, 136, 200, 128)])
def test_gemm_nt_matches_oracle_bf16(B, M, N, K):
    _check_gemm(_x((B, M, K), 41, torch.bfloat16), _x((B, N, K), 43, torch.bfloat16), 1.0, torch.bfloat16, B)


def test_gemm_nt_error_is_accumulation_sized():
    err, bound = _check_gemm(_x((1, 512, 2048), 51), _x((1, 256, 2048), 53), 1.0, torch.float32, 1)
    # observed error is a few ulps of sum|ab|, far inside the worst-case bound
    assert (err <= 16 * U * bound + 1e-37).all()


def test_gemm_nt_poisoned_block_gives_nan_row_only():
    M, N, K = 128, 64, 128
    xa = _x((M, K), 61)
    xa[5, 17] = float("nan")
    xb = _x((N, K), 62)
    gin = torch.tensor([0.01], dtype=torch.float32).cuda()
    ac, asf, _ = nv.quantize_mma(xa.cuda(), gscale_in=gin)
    bc, bsf, _ = nv.quantize_mma(xb.cuda(), gscale_in=gin)
    d = nv.gemm_nt(ac, asf, gin, bc, bsf, gin).cpu().numpy()
    assert np.isnan(d[5]).all()
    assert np.isfinite(np.delete(d, 5, axis=0)).all()


def test_gemm_nt_zero_k_and_errors():
    z = torch.empty((4, 0), dtype=torch.uint8, device="cuda")
    sf = torch.zeros(4096, dtype=torch.uint8, device="cuda")    # room for every shape below: the C statuses are tested
    g = torch.ones(1, device="cuda")
    d = nv.gemm_nt(z, sf, g, torch.empty((8, 0), dtype=torch.uint8, device="cuda"), sf, g)
    assert d.shape == (4, 8) and not d.any()
    a = torch.zeros((4, 8), dtype=torch.uint8, device="cuda")      # K = 16: not a multiple of 32
    with pytest.raises(nv.NVFP4Error) as e:
        nv.gemm_nt(a, sf, g, torch.zeros((8, 8), dtype=torch.uint8, device="cuda"), sf, g)
    assert e.value.status == -2
    a = torch.zeros((4, 16), dtype=torch.uint8, device="cuda")
    with pytest.raises(nv.NVFP4Error) as e:                          # N = 6: f32 rows not 16-byte multiples
        nv.gemm_nt(a, sf, g, torch.zeros((6, 16), dtype=torch.uint8, device="cuda"), sf, g)
    assert e.value.status == -3


def test_attention_scores_from_rotated_nvfp4_q_and_kv_cache():
    """Q K^T of the attention prologue: K through kv_mixed_mma (Hadamard-rotated, sink/recent in BF16),
    Q rotated the same way and quantized with quantize_mma, scores on the tensor cores per head."""
    H, Tq, T, D = 2, 64, 160, 128
    k = _x((1, H, T, D), 71, torch.bfloat16)
    q = _x((H, Tq, D), 72, torch.bfloat16)
    _, _, kc, ksf, kg = nv.kv_mixed_mma(k.cuda())
    qr = nv.hadamard16(q.cuda(), out_dtype=torch.float32)
    qc, qsf, qg = nv.quantize_mma(qr)
    Tm = T - 32
    s = nv.gemm_nt(qc, qsf, qg, kc.reshape(H, Tm, D // 2), ksf, kg, alpha=D ** -0.5)
    torch.cuda.synchronize()
    # oracle for the same pipeline
    _, _, rkc, rks, rkg = O.kv_mixed(_np(k))
    rq = O.hadamard16(_np(q).reshape(-1), dtype=O.BF16, out_dtype=O.F32)
    rqc, rqs, rqg, _, _ = O.quantize(rq)
    ref = O.gemm_nt(rqc, rqs, rqg, rkc, rks, rkg, Tq, Tm, D, D ** -0.5, H)
    bound = _gemm_bound(rqc, rqs, rkc, rks, Tq, Tm, D, H, D ** -0.5 * float(rqg) * float(rkg))
    got = s.cpu().numpy().astype(np.float64)
    assert (np.abs(got - ref) <= (D + 4) * U * bound + 1e-37).all()
    # the rotation is orthogonal: scores stay close to the full-precision Q K^T of the middle tokens
    full = torch.einsum("hqd,htd->hqt", q.float(), k[0, :, 16:T - 16].float()).numpy() * D ** -0.5
    rel = np.linalg.norm(got - full) / np.linalg.norm(full)
    assert rel < 0.25, rel


def test_gemm_nt_full_size_sampled():
    """8192^3 (activations of the [8192, 8192] workload against a weight-like matrix): sampled rows."""
    from nvfp4_block_scaled_11_b200 import workloads as W
    M = N = K = 8192
    xa = W.make("act_bf16", "cpu").x.reshape(M, K)
    xb = _x((N, K), 11, torch.bfloat16, scale=K ** -0.5)
    ac, asf, ga = nv.quantize_mma(xa.cuda())
    bc, bsf, gb = nv.quantize_mma(xb.cuda())
    d = nv.gemm_nt(ac, asf, ga, bc, bsf, gb)
    torch.cuda.synchronize()
    rga = O.global_scale(O.tensor_amax(_np(xa).reshape(-1), O.BF16))
    rgb = O.global_scale(O.tensor_amax(_np(xb).reshape(-1), O.BF16))
    assert ga.item() == rga and gb.item() == rgb
    rng = np.random.default_rng(3)
    rows = rng.choice(M, 6, replace=False)
    cols = np.sort(rng.choice(N, 64, replace=False))
    xa_np, xb_np = _np(xa).reshape(M, K), _np(xb).reshape(N, K)
    # blocks are independent once g is fixed: quantize only the sampled rows of A and B
    sel_b = np.ascontiguousarray(xb_np[cols]).reshape(-1)
    rbc, rbs, _, _ = O.quantize_blocks(sel_b, 0, sel_b.size // 16, rgb, dtype=O.BF16)
    dc = d.cpu().numpy()
    for r in rows:
        rac, ras, _, _ = O.quantize_blocks(xa_np[r].copy(), 0, K // 16, rga, dtype=O.BF16)
        ref = O.gemm_nt(rac, ras, rga, rbc, rbs, rgb, 1, len(cols), K)[0, 0]
        bound = _gemm_bound(rac, ras, rbc, rbs, 1, len(cols), K, 1, float(rga) * float(rgb))[0, 0]
        assert (np.abs(dc[r, cols].astype(np.float64) - ref) <= (K + 4) * U * bound + 1e-37).all(), r


@pytest.mark.parametrize("shape,dtype", [((1, 128, 64), torch.float32), ((2, 96, 130), torch.bfloat16),
                                         ((3, 16, 33), torch.float16), ((1, 4096, 128), torch.bfloat16)])
def test_quantize_mma_t_bit_exact(shape, dtype):
    x = _x(shape, 200 + shape[2], dtype)
    codes, sf, g = nv.quantize_mma_t(x.cuda())
    rc, rsf, rg = O.quantize_mma_t(_np(x).reshape(shape), dtype=_odt(x))
    assert g.item() == rg
    assert codes.shape == (shape[0], shape[2], shape[1] // 2)
    assert np.array_equal(codes.cpu().numpy().reshape(-1), rc)
    assert np.array_equal(sf.cpu().numpy(), rsf)


def test_quantize_mma_t_windows_and_external_scale():
    x = _x((2, 64, 40), 9)
    gin = torch.tensor([0.004], dtype=torch.float32)
    for lo, hi in ((0, 0), (-8, 8), (-1, 3)):
        codes, sf, _ = nv.quantize_mma_t(x.cuda(), lo, hi, gscale_in=gin.cuda())
        rc, rsf, _ = O.quantize_mma_t(x.numpy(), lo, hi, gscale_in=0.004)
        assert np.array_equal(codes.cpu().numpy().reshape(-1), rc), (lo, hi)
        assert np.array_equal(sf.cpu().numpy(), rsf), (lo, hi)
