"""The Python binding refuses caller-provided buffers that a kernel would read or write past their end
(or that have the wrong dtype), before anything is launched."""
import pytest
import torch

import nvfp4_block_scaled_11_b200 as nv

pytestmark = pytest.mark.gpu


def E(n, dt=torch.uint8):
    return torch.empty(n, dtype=dt, device="cuda")


def test_short_or_mistyped_outputs_are_refused():
    x = torch.randn(1024, device="cuda")
    with pytest.raises(ValueError):
        nv.quantize(x, codes=E(511))
    with pytest.raises(ValueError):
        nv.quantize(x, scales=E(63))
    with pytest.raises(TypeError):
        nv.quantize(x, gscale=E(1, torch.float16))
    with pytest.raises(ValueError):
        nv.quantize_ex(x, block_f=E(63, torch.int8))
    with pytest.raises(ValueError):
        nv.quantize_ex(x, block_sse=E(63, torch.float32))
    c, s, g = nv.quantize(x)
    with pytest.raises(ValueError):
        nv.dequantize(c[:100], s, g)                       # codes shorter than the scales imply
    with pytest.raises(ValueError):
        nv.dequantize(c, s, g, out=E(1000, torch.float32))
    with pytest.raises(ValueError):
        nv.hadamard16(x, out=E(1008, torch.float32))
    with pytest.raises(ValueError):
        nv.quantize_dequantize(x, out=E(1008, torch.float32))
    with pytest.raises(ValueError):
        nv.mxfp4_quantize(x, codes=E(500))
    with pytest.raises(ValueError):
        nv.tensor_amax(x, out=E(0, torch.float32))


def test_tile_layout_gemm_and_attention_buffers_are_checked():
    a = torch.randn(130, 64, device="cuda")
    with pytest.raises(ValueError):
        nv.quantize_mma(a, sf=E(nv.sf_mma_bytes(130, 64) - 1))
    with pytest.raises(ValueError):
        nv.quantize_mma_t(torch.randn(64, 40, device="cuda"), codes=E(64 * 40 // 2 - 1))
    ac, asf, ag = nv.quantize_mma(a)
    bc, bsf, bg = nv.quantize_mma(torch.randn(72, 64, device="cuda"))
    with pytest.raises(ValueError):
        nv.gemm_nt(ac, asf[:100], ag, bc, bsf, bg)
    with pytest.raises(ValueError):
        nv.gemm_nt(ac, asf, ag, bc, bsf, bg, out=E(130 * 72 - 1, torch.float32))
    with pytest.raises(TypeError):
        nv.gemm_nt(ac, asf, ag, bc, bsf, bg, out=E(130 * 72, torch.float16))
    s = torch.randn(2, 8, 64, device="cuda")
    with pytest.raises(ValueError):
        nv.softmax_quantize_mma(s, l=E(15, torch.float32))
    with pytest.raises(TypeError):
        nv.softmax_quantize_mma(s.half())
    with pytest.raises(ValueError):
        nv.rows_divide(torch.randn(16, 8, device="cuda"), E(15, torch.float32))
    k = torch.randn(2, 40, 64, device="cuda").to(torch.bfloat16)
    g = nv.kv_gscale(k[None], 0, 0)
    with pytest.raises(ValueError):
        nv.kv_append(k, 0, 16, g, E((2, 20, 31)), E((2, 20, 4)), 0)


def test_kv_append_batch_buffers_are_checked():
    k = torch.randn(2, 32, 64, device="cuda").to(torch.bfloat16)
    g = torch.ones(1, device="cuda")
    ok = (k, g, E((2, 16, 32)), E((2, 16, 4)), True, False)
    with pytest.raises(ValueError):
        nv.KvAppendBatch([(k, g, E((2, 16, 31)), E((2, 16, 4)), True, False)])        # codes short
    with pytest.raises(ValueError):
        nv.KvAppendBatch([(k, g, E((2, 16, 32)), E(nv.sf_mma_bytes(16, 64, 2) - 1), True, True)])
    with pytest.raises(TypeError):
        nv.KvAppendBatch([(k.float(), g, E((2, 16, 32)), E((2, 16, 4)), True, False)])
    with pytest.raises(ValueError):
        nv.KvAppendBatch([ok] * 65)
    b = nv.KvAppendBatch([ok, ok[:2] + (E((2, 16, 32)), E((2, 16, 4))) + ok[4:]])
    b([0, 16], 16, [0, 0])                                  # per-item rows, one n for both
    with pytest.raises(nv.NVFP4Error):
        b(0, 16, 1)                                          # rows 1..16 exceed the 16-row caches
    torch.cuda.synchronize()
