"""nvfp4_gemm_nt_noalloc, the product for callers that cannot allocate device memory (code whose device
memory is all owned by a host framework's pool, or reserved up front, so it has no way to provide the
scratch word nvfp4_gemm_nt asks for): called through the C ABI, it must give exactly what nvfp4_gemm_nt
gives with a caller-provided word, on two calls in a row with different operands and alpha (the second
call must not see the first call's scale).  Collected last, so that a run stopping at the first failure
has run every other test before it; it also passes alone in a fresh process (its first call on the
device is the one that looks up the library's scratch address)."""
import ctypes

import pytest
import torch

import nvfp4_block_scaled_11_b200 as nv

pytestmark = pytest.mark.gpu


def _operands(seed, M, N, K, batch=1):
    g = torch.Generator().manual_seed(seed)
    a = torch.randn((batch, M, K), generator=g).cuda()
    b = (torch.randn((batch, N, K), generator=g) * 3.0).cuda()
    ac, asf, ag = nv.quantize_mma(a)
    bc, bsf, bg = nv.quantize_mma(b)
    return ac, asf, ag, bc, bsf, bg


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _call(fn, ops, batch, M, N, K, alpha, d, work=None):
    ac, asf, ag, bc, bsf, bg = ops
    args = [_p(ac), _p(asf), _p(ag), _p(bc), _p(bsf), _p(bg), batch, M, N, K, ctypes.c_float(alpha), _p(d), 0]
    if work is not None:
        args.append(_p(work))
    args.append(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return fn(*args)


def test_noalloc_product_equals_the_scratch_taking_entry_point():
    L = nv.lib()
    cases = [(1, 256, 192, 512, 0.125, 41), (2, 128, 64, 256, -3.0, 42)]
    for batch, M, N, K, alpha, seed in cases:          # two calls in a row, different alpha and operands
        ops = _operands(seed, M, N, K, batch)
        work = torch.empty(1, dtype=torch.float32, device="cuda")
        d_ref = torch.full((batch, M, N), float("nan"), dtype=torch.float32, device="cuda")
        d_new = torch.full((batch, M, N), float("nan"), dtype=torch.float32, device="cuda")
        assert _call(L.nvfp4_gemm_nt, ops, batch, M, N, K, alpha, d_ref, work) == 0
        assert _call(L.nvfp4_gemm_nt_noalloc, ops, batch, M, N, K, alpha, d_new) == 0
        torch.cuda.synchronize()
        assert torch.isfinite(d_ref).all()
        assert torch.equal(d_new.view(torch.int32), d_ref.view(torch.int32))
    # argument errors come back as nvfp4_gemm_nt's (NVFP4_ERR_SIZE = -2 for K % 32 != 0), before any launch
    assert _call(L.nvfp4_gemm_nt_noalloc, ops, batch, M, N, 48, alpha, d_new) == -2
