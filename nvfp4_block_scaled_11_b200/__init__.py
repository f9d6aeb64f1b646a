"""nvfp4_block_scaled_11_b200 -- Python binding of libnvfp4 (NVFP4 ScaleSearch quantization, sm_100a).

Argument marshalling only: every function checks that its tensors are contiguous CUDA tensors,
allocates outputs with torch when the caller did not pass them, and calls the C ABI declared in
``include/nvfp4.h`` with raw device pointers and the current CUDA stream.  All computation happens
in the library's CUDA kernels; there is no CPU path.  A missing ``libnvfp4.so`` raises.

Element types: torch.float32, torch.bfloat16, torch.float16.
"""
from __future__ import annotations

import ctypes
import numbers
import os

import torch

__all__ = [
    "NVFP4Error", "lib", "status_str", "tensor_amax", "global_scale", "quantize", "quantize_ex",
    "dequantize", "quantize_dequantize", "hadamard16", "kv_mixed", "kv_mixed_dequantize", "DTYPE_CODE", "sf_mma_bytes", "quantize_mma", "quantize_mma_t", "kv_mixed_mma",
    "gemm_nt", "gemm_sf_offsets", "kv_gscale", "kv_append", "mxfp4_quantize", "mxfp4_dequantize",
    "msda_forward", "softmax_quantize_mma", "rows_divide", "attention_fp4", "search_policy", "kv_append_batch", "KvAppendBatch",
]

_SO = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libnvfp4.so")
_lib = None

DTYPE_CODE = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}
DTYPE_OF = {v: k for k, v in DTYPE_CODE.items()}

# C-ABI entry points and their argument types (include/nvfp4.h)
_P, _I64, _I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
_SIGS = {
    "nvfp4_status_str": (ctypes.c_char_p, [_I]),
    "nvfp4_version": (_I, []),
    "nvfp4_search_policy": (_I, [_I64, _I64, _P, _P]),
    "nvfp4_tensor_amax": (_I, [_P, _I64, _I, _P, _P]),
    "nvfp4_global_scale": (_I, [_P, _P, _P]),
    "nvfp4_quantize": (_I, [_P, _I64, _I, _I, _I, _I, _P, _P, _P, _P]),
    "nvfp4_quantize_ex": (_I, [_P, _I64, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P]),
    "nvfp4_dequantize": (_I, [_P, _P, _P, _I64, _I, _P, _P]),
    "nvfp4_dequantize_ex": (_I, [_P, _P, _P, _I64, _I, _P, _I, _P]),
    "nvfp4_quantize_dequantize": (_I, [_P, _I64, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "nvfp4_hadamard16": (_I, [_P, _I64, _I, _P, _I, _P]),
    "nvfp4_hadamard16_ex": (_I, [_P, _I64, _I, _P, _I, ctypes.c_uint32, _I, _P]),
    "nvfp4_kv_mixed": (_I, [_P, _I64, _I64, _I64, _I64, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "nvfp4_kv_mixed_dequantize": (_I, [_P, _I64, _I64, _I64, _I64, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P]),
    "nvfp4_msda_forward_nvfp4": (_I, [_P, _P, _P, _I64, _I64, _I64, _I64, _P, _I, _I, _I64, _P, _P, _P, _P]),
    "nvfp4_msda_forward": (_I, [_P, _I, _I64, _I64, _I64, _I64, _P, _I, _I, _I64, _P, _P, _P, _P]),
    "nvfp4_mxfp4_quantize": (_I, [_P, _I64, _I, _P, _P, _P]),
    "nvfp4_mxfp4_dequantize": (_I, [_P, _P, _I64, _I, _P, _P]),
    "nvfp4_kv_gscale": (_I, [_P, _I64, _I64, _I64, _I64, _I, _I, _I, _P, _P]),
    "nvfp4_kv_append": (_I, [_P, _I64, _I64, _I64, _I64, _I64, _I, _I, _I, _P, _P, _P, _I64, _I64, _I, _P]),
    "nvfp4_kv_append_batch": (_I, [_P, _I, _I, _I, _P]),
    "nvfp4_sf_mma_bytes": (_I64, [_I64, _I64, _I64]),
    "nvfp4_quantize_mma": (_I, [_P, _I64, _I64, _I64, _I, _I, _I, _P, _P, _P, _P, _P]),
    "nvfp4_quantize_mma_t": (_I, [_P, _I64, _I64, _I64, _I, _I, _I, _P, _P, _P, _P, _P]),
    "nvfp4_kv_mixed_mma": (_I, [_P, _I64, _I64, _I64, _I64, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "nvfp4_gemm_nt": (_I, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, ctypes.c_float, _P, _I, _P, _P]),
    "nvfp4_gemm_nt_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, ctypes.c_float, _P, _I, _P]),
    "nvfp4_softmax_quantize_mma": (_I, [_P, _I64, _I64, _I64, _I, _I64, _I, _I, _P, _P, _P, _P, _P, _P]),
    "nvfp4_rows_divide": (_I, [_P, _P, _I64, _I64, _P]),
    "nvfp4_attention_fused": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, ctypes.c_float, _I,
                                   _I64, _I, _I, _I, _P, ctypes.c_size_t, _P, _P, _P, _P, _P, _P, _P, _P]),
    "nvfp4_attention_fused_splits": (_I, [_I64, _I64, _I64, _P]),
    "nvfp4_attention_fused_workspace_bytes": (ctypes.c_size_t, [_I64, _I64, _I64, _I]),
    "nvfp4_gemm_sf_offsets": (_I, [_I64, _I64, _I64, _P]),
}


class NVFP4Error(RuntimeError):
    def __init__(self, status: int):
        super().__init__(status_str(status))
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded libnvfp4 (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_SO):
            raise RuntimeError(
                f"libnvfp4.so is not built ({_SO}); run `python -m nvfp4_block_scaled_11_b200.build`"
            )
        L = ctypes.CDLL(_SO)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def library_path() -> str:
    """Path of the loaded libnvfp4.so (for C programs that link it)."""
    lib()
    return _SO


def status_str(status: int) -> str:
    return lib().nvfp4_status_str(status).decode()


def _check(rc: int) -> None:
    if rc != 0:
        raise NVFP4Error(rc)


def search_policy(lane1_max: int | None = None, lanes_max: int | None = None) -> tuple[int, int]:
    """Launch policy of the ScaleSearch quantizers (windows of at most 32 offsets), bounds in threads
    (blocks x lanes per block): up to `lane1_max`, one offset per lane (16 or 32 lanes per block); up to
    `lanes_max`, a few offsets per lane (4 or 8 lanes per block); beyond, a thread per block.  All write
    the same bytes.  None keeps a bound; returns the previous bounds."""
    a, b = ctypes.c_int64(), ctypes.c_int64()
    _check(lib().nvfp4_search_policy(-1 if lane1_max is None else int(lane1_max),
                                     -1 if lanes_max is None else int(lanes_max), ctypes.byref(a), ctypes.byref(b)))
    return a.value, b.value


def _cuda(t: torch.Tensor, name: str) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _out(t: torch.Tensor, name: str, dtype, need: int) -> torch.Tensor:
    """A caller-provided buffer that a kernel reads or writes by size: a contiguous CUDA tensor of `dtype`
    (None: any dtype) with at least `need` elements, so that no launch reaches past its end."""
    _cuda(t, name)
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.numel() < need:
        raise ValueError(f"{name} holds {t.numel()} elements, {need} needed")
    return t


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _dt(t: torch.Tensor) -> int:
    try:
        return DTYPE_CODE[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}") from None


def tensor_amax(x: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """max |x| as a 1-element float32 device tensor (NaN / Inf propagate)."""
    _cuda(x, "x")
    out = torch.empty(1, dtype=torch.float32, device=x.device) if out is None else _out(out, "out", torch.float32, 1)
    _check(lib().nvfp4_tensor_amax(_ptr(x), x.numel(), _dt(x), _ptr(out), _stream(x)))
    return out


def global_scale(amax: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """g = amax / 2688 on the device."""
    _out(amax, "amax", torch.float32, 1)
    out = torch.empty(1, dtype=torch.float32, device=amax.device) if out is None else _out(out, "out", torch.float32, 1)
    _check(lib().nvfp4_global_scale(_ptr(amax), _ptr(out), _stream(amax)))
    return out


def _alloc_q(x, codes, scales, gscale):
    n = x.numel()
    dev = x.device
    codes = torch.empty(n // 2, dtype=torch.uint8, device=dev) if codes is None else _out(codes, "codes", torch.uint8, n // 2)
    scales = (torch.empty(n // 16, dtype=torch.uint8, device=dev) if scales is None
              else _out(scales, "scales", torch.uint8, n // 16))
    gscale = (torch.empty(1, dtype=torch.float32, device=dev) if gscale is None
              else _out(gscale, "gscale", torch.float32, 1))
    return codes, scales, gscale


def quantize(x: torch.Tensor, f_lo: int = -2, f_hi: int = 6, block: int = 16, codes=None, scales=None, gscale=None):
    """ScaleSearch quantize of x (blocks of 16 along the contiguous order).

    Returns (codes uint8[n/2], scales uint8[n/16], gscale float32[1])."""
    _cuda(x, "x")
    codes, scales, gscale = _alloc_q(x, codes, scales, gscale)
    _check(lib().nvfp4_quantize(_ptr(x), x.numel(), _dt(x), block, f_lo, f_hi, _ptr(codes), _ptr(scales),
                                _ptr(gscale), _stream(x)))
    return codes, scales, gscale


def quantize_ex(x: torch.Tensor, f_lo: int = -2, f_hi: int = 6, gscale_in: torch.Tensor | None = None,
                want_f: bool = True, want_sse: bool = True, block: int = 16, codes=None, scales=None, gscale=None,
                block_f=None, block_sse=None):
    """Quantize with optional external tensor scale and per-block outputs.

    Returns (codes, scales, gscale, block_f int8[n/16] or None, block_sse float32[n/16] or None)."""
    _cuda(x, "x")
    n = x.numel()
    keep = gscale
    if gscale_in is not None:
        _out(gscale_in, "gscale_in", torch.float32, 1)
    codes, scales, gscale = _alloc_q(x, codes, scales, gscale)
    if gscale_in is not None and keep is None:
        gscale = None  # g comes from gscale_in; no copy requested
    if want_f and block_f is None:
        block_f = torch.empty(n // 16, dtype=torch.int8, device=x.device)
    elif block_f is not None:
        _out(block_f, "block_f", torch.int8, n // 16)
    if want_sse and block_sse is None:
        block_sse = torch.empty(n // 16, dtype=torch.float32, device=x.device)
    elif block_sse is not None:
        _out(block_sse, "block_sse", torch.float32, n // 16)
    _check(lib().nvfp4_quantize_ex(_ptr(x), n, _dt(x), block, f_lo, f_hi, _ptr(gscale_in), _ptr(codes),
                                   _ptr(scales), _ptr(gscale), _ptr(block_f), _ptr(block_sse), _stream(x)))
    return codes, scales, gscale, block_f, block_sse


def quantize_dequantize(x: torch.Tensor, f_lo: int = -2, f_hi: int = 6, gscale_in: torch.Tensor | None = None,
                        codes=None, scales=None, gscale=None, out: torch.Tensor | None = None):
    """Fused round trip: quantize x with ScaleSearch and write its dequantized values (x's dtype) in the same
    pass.  Returns (out, codes, scales, gscale); out equals dequantize(codes, scales, g, x.dtype) bit for bit.
    out may be x itself (in-place simulated quantization)."""
    _cuda(x, "x")
    n = x.numel()
    if gscale_in is not None:
        _out(gscale_in, "gscale_in", torch.float32, 1)
    keep = gscale
    codes, scales, gscale = _alloc_q(x, codes, scales, gscale)
    if gscale_in is not None and keep is None:
        gscale = None
    out = torch.empty_like(x) if out is None else out
    _cuda(out, "out")
    if out.dtype != x.dtype or out.numel() != n:
        raise ValueError("out must have x's dtype and size")
    _check(lib().nvfp4_quantize_dequantize(_ptr(x), n, _dt(x), f_lo, f_hi, _ptr(gscale_in), _ptr(codes), _ptr(scales),
                                           _ptr(gscale), _ptr(out), _stream(x)))
    return out, codes, scales, gscale


def dequantize(codes: torch.Tensor, scales: torch.Tensor, gscale: torch.Tensor, out_dtype=torch.float32,
               out: torch.Tensor | None = None, ctas_per_sm: int = 0) -> torch.Tensor:
    """Dequantize n = 16 * scales.numel() elements to out_dtype.  ctas_per_sm > 0 bounds the launch
    footprint (to run beside another kernel on a second stream); 0 = default."""
    _cuda(scales, "scales")
    n = scales.numel() * 16
    _out(codes, "codes", torch.uint8, n // 2), _out(gscale, "gscale", torch.float32, 1)
    out = torch.empty(n, dtype=out_dtype, device=codes.device) if out is None else _out(out, "out", None, n)
    _check(lib().nvfp4_dequantize_ex(_ptr(codes), _ptr(scales), _ptr(gscale), n, DTYPE_CODE[out.dtype], _ptr(out),
                                     ctas_per_sm, _stream(codes)))
    return out


def hadamard16(x: torch.Tensor, out_dtype=None, out: torch.Tensor | None = None, signs: int = 0,
               inverse: bool = False) -> torch.Tensor:
    """FWHT-16 / 4 on every contiguous group of 16 elements; with `signs` (16-bit mask) the sign diagonal
    D goes first, (H/4) D x, or last for the inverse, D (H/4) x."""
    _cuda(x, "x")
    out_dtype = x.dtype if out_dtype is None else out_dtype
    out = torch.empty(x.shape, dtype=out_dtype, device=x.device) if out is None else _out(out, "out", None, x.numel())
    if signs == 0 and not inverse:
        _check(lib().nvfp4_hadamard16(_ptr(x), x.numel(), _dt(x), _ptr(out), DTYPE_CODE[out.dtype], _stream(x)))
    else:
        _check(lib().nvfp4_hadamard16_ex(_ptr(x), x.numel(), _dt(x), _ptr(out), DTYPE_CODE[out.dtype], signs,
                                         int(inverse), _stream(x)))
    return out


def kv_mixed(k: torch.Tensor, sink: int = 16, recent: int = 16, rotate: bool = True, f_lo: int = -2, f_hi: int = 6):
    """Mixed-precision KV layout of K[B,H,T,D] (BF16).

    Returns (sink bf16[B,H,sink,D], recent bf16[B,H,recent,D], codes uint8[B,H,Tm,D/2],
    scales uint8[B,H,Tm,D/16], gscale float32[1])."""
    _cuda(k, "k")
    if k.dtype != torch.bfloat16 or k.dim() != 4:
        raise TypeError("k must be a 4-D bfloat16 tensor [B,H,T,D]")
    B, H, T, D = k.shape
    Tm = T - sink - recent
    dev = k.device
    so = torch.empty((B, H, sink, D), dtype=torch.bfloat16, device=dev)
    ro = torch.empty((B, H, recent, D), dtype=torch.bfloat16, device=dev)
    codes = torch.empty((B, H, max(Tm, 0), D // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((B, H, max(Tm, 0), D // 16), dtype=torch.uint8, device=dev)
    gscale = torch.empty(1, dtype=torch.float32, device=dev)
    _check(lib().nvfp4_kv_mixed(_ptr(k), B, H, T, D, sink, recent, int(bool(rotate)), f_lo, f_hi, _ptr(so),
                                _ptr(ro), _ptr(codes), _ptr(scales), _ptr(gscale), _stream(k)))
    return so, ro, codes, scales, gscale


# ---- tensor-core consumer: scales in the MMA tile layout, NVFP4 x NVFP4 product ----
def sf_mma_bytes(rows: int, cols: int, batch: int = 1) -> int:
    """Bytes of the tile-layout scales of `batch` [rows, cols] matrices (padded to 128 rows x 4 blocks)."""
    nb = lib().nvfp4_sf_mma_bytes(rows, cols, batch)
    if nb < 0:
        raise NVFP4Error(int(nb))
    return int(nb)


def kv_mixed_dequantize(k: torch.Tensor, sink: int = 16, recent: int = 16, rotate: bool = True, f_lo: int = -2,
                        f_hi: int = 6, mid_out: torch.Tensor | None = None):
    """kv_mixed plus the middle's dequantized values (BF16 [B,H,Tm,D], rotated when `rotate`) in the same
    pass.  Returns (sink, recent, codes, scales, gscale, mid)."""
    _cuda(k, "k")
    if k.dtype != torch.bfloat16 or k.dim() != 4:
        raise TypeError("k must be a 4-D bfloat16 tensor [B,H,T,D]")
    B, H, T, D = k.shape
    Tm = T - sink - recent
    if Tm < 0:
        raise ValueError("T < sink + recent")
    dev = k.device
    so = torch.empty((B, H, sink, D), dtype=torch.bfloat16, device=dev)
    ro = torch.empty((B, H, recent, D), dtype=torch.bfloat16, device=dev)
    codes = torch.empty((B, H, Tm, D // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((B, H, Tm, D // 16), dtype=torch.uint8, device=dev)
    gscale = torch.empty(1, dtype=torch.float32, device=dev)
    mid = torch.empty((B, H, Tm, D), dtype=torch.bfloat16, device=dev) if mid_out is None else mid_out
    _cuda(mid, "mid_out")
    if mid.dtype != torch.bfloat16 or mid.numel() != B * H * Tm * D:
        raise ValueError("mid_out must be bfloat16 with B*H*Tm*D elements")
    _check(lib().nvfp4_kv_mixed_dequantize(_ptr(k), B, H, T, D, sink, recent, int(bool(rotate)), f_lo, f_hi, _ptr(so),
                                           _ptr(ro), _ptr(codes), _ptr(scales), _ptr(gscale), _ptr(mid), _stream(k)))
    return so, ro, codes, scales, gscale, mid


def quantize_mma(x: torch.Tensor, f_lo: int = -2, f_hi: int = 6, gscale_in: torch.Tensor | None = None,
                 codes: torch.Tensor | None = None, sf: torch.Tensor | None = None,
                 gscale: torch.Tensor | None = None):
    """Quantize x [rows, cols] or [batch, rows, cols] along cols with the scales in the tensor-core tile
    layout.  Returns (codes uint8[..., rows, cols/2] (x's rank), sf uint8[sf_mma_bytes], gscale float32[1])."""
    _cuda(x, "x")
    if x.dim() not in (2, 3):
        raise ValueError("x must be [rows, cols] or [batch, rows, cols]")
    batch, rows, cols = (1, *x.shape) if x.dim() == 2 else x.shape
    dev = x.device
    if codes is None:
        codes = torch.empty((*x.shape[:-1], cols // 2), dtype=torch.uint8, device=dev)
    if sf is None:
        sf = torch.empty(sf_mma_bytes(rows, cols, batch), dtype=torch.uint8, device=dev)
    if gscale is None:
        gscale = torch.empty(1, dtype=torch.float32, device=dev)
    _out(codes, "codes", torch.uint8, x.numel() // 2), _out(gscale, "gscale", torch.float32, 1)
    _out(sf, "sf", torch.uint8, sf_mma_bytes(rows, cols, batch))
    if gscale_in is not None:
        _out(gscale_in, "gscale_in", torch.float32, 1)
    _check(lib().nvfp4_quantize_mma(_ptr(x), batch, rows, cols, _dt(x), f_lo, f_hi, _ptr(gscale_in), _ptr(codes),
                                    _ptr(sf), _ptr(gscale), _stream(x)))
    return codes, sf, gscale


def quantize_mma_t(x: torch.Tensor, f_lo: int = -2, f_hi: int = 6, gscale_in: torch.Tensor | None = None,
                   codes: torch.Tensor | None = None, sf: torch.Tensor | None = None,
                   gscale: torch.Tensor | None = None):
    """Quantize x [rows, cols] or [batch, rows, cols] in blocks of 16 rows per column, written transposed:
    codes uint8[..., cols, rows/2], sf (tile layout of the [cols, rows] matrices), gscale float32[1]."""
    _cuda(x, "x")
    if x.dim() not in (2, 3):
        raise ValueError("x must be [rows, cols] or [batch, rows, cols]")
    batch, rows, cols = (1, *x.shape) if x.dim() == 2 else x.shape
    dev = x.device
    if codes is None:
        codes = torch.empty((*x.shape[:-2], cols, rows // 2), dtype=torch.uint8, device=dev)
    if sf is None:
        sf = torch.empty(sf_mma_bytes(cols, rows, batch), dtype=torch.uint8, device=dev)
    if gscale is None:
        gscale = torch.empty(1, dtype=torch.float32, device=dev)
    _out(codes, "codes", torch.uint8, x.numel() // 2), _out(gscale, "gscale", torch.float32, 1)
    _out(sf, "sf", torch.uint8, sf_mma_bytes(cols, rows, batch))
    if gscale_in is not None:
        _out(gscale_in, "gscale_in", torch.float32, 1)
    _check(lib().nvfp4_quantize_mma_t(_ptr(x), batch, rows, cols, _dt(x), f_lo, f_hi, _ptr(gscale_in), _ptr(codes),
                                      _ptr(sf), _ptr(gscale), _stream(x)))
    return codes, sf, gscale


def kv_mixed_mma(k: torch.Tensor, sink: int = 16, recent: int = 16, rotate: bool = True, f_lo: int = -2,
                 f_hi: int = 6, codes: torch.Tensor | None = None, sf: torch.Tensor | None = None,
                 gscale: torch.Tensor | None = None):
    """kv_mixed with the middle-token scales of every (batch, head) in the tensor-core tile layout.
    With sink = recent = 0 and rotate it is the rotated quantize of every token, fused (codes and scales
    as quantize_mma of the FWHT-16-rotated FP32 tensor).  codes / sf / gscale: optional preallocated outputs.

    Returns (sink, recent, codes uint8[B,H,Tm,D/2], sf uint8[sf_mma_bytes(Tm, D, B*H)], gscale)."""
    _cuda(k, "k")
    if k.dtype != torch.bfloat16 or k.dim() != 4:
        raise TypeError("k must be a 4-D bfloat16 tensor [B,H,T,D]")
    B, H, T, D = k.shape
    Tm = max(T - sink - recent, 0)
    dev = k.device
    so = torch.empty((B, H, sink, D), dtype=torch.bfloat16, device=dev)
    ro = torch.empty((B, H, recent, D), dtype=torch.bfloat16, device=dev)
    codes = torch.empty((B, H, Tm, D // 2), dtype=torch.uint8, device=dev) if codes is None else codes
    sf = torch.empty(max(sf_mma_bytes(Tm, D, B * H), 1), dtype=torch.uint8, device=dev) if sf is None else sf
    gscale = torch.empty(1, dtype=torch.float32, device=dev) if gscale is None else gscale
    for t, nm, need in ((codes, "codes", B * H * Tm * D // 2), (sf, "sf", sf_mma_bytes(Tm, D, B * H)),
                        (gscale, "gscale", 1)):
        _cuda(t, nm)
        if t.numel() < need:
            raise ValueError(f"{nm} holds {t.numel()} elements, {need} needed")
    _check(lib().nvfp4_kv_mixed_mma(_ptr(k), B, H, T, D, sink, recent, int(bool(rotate)), f_lo, f_hi, _ptr(so),
                                    _ptr(ro), _ptr(codes), _ptr(sf), _ptr(gscale), _stream(k)))
    return so, ro, codes, sf, gscale


def gemm_nt(a_codes: torch.Tensor, a_sf: torch.Tensor, a_gscale: torch.Tensor, b_codes: torch.Tensor,
            b_sf: torch.Tensor, b_gscale: torch.Tensor, alpha: float = 1.0, out_dtype=torch.float32,
            out: torch.Tensor | None = None, alpha_work: torch.Tensor | None = None) -> torch.Tensor:
    """D[l] = alpha * g_a * g_b * A[l] B[l]^T on the tensor cores (FP32 accumulation).

    a_codes: uint8 [M, K/2] or [batch, M, K/2] (quantize_mma output), b_codes: [.., N, K/2] likewise;
    returns D [M, N] or [batch, M, N] in out_dtype (float32 or bfloat16)."""
    for t, nm in ((a_codes, "a_codes"), (a_sf, "a_sf"), (a_gscale, "a_gscale"), (b_codes, "b_codes"),
                  (b_sf, "b_sf"), (b_gscale, "b_gscale")):
        _cuda(t, nm)
    squeeze = a_codes.dim() == 2
    a3 = a_codes if a_codes.dim() == 3 else a_codes.unsqueeze(0)
    b3 = b_codes if b_codes.dim() == 3 else b_codes.unsqueeze(0)
    batch, M, K2 = a3.shape
    if b3.shape[0] != batch or b3.shape[2] != K2:
        raise ValueError("a_codes and b_codes disagree on batch or K")
    N, K = b3.shape[1], 2 * K2
    dev = a_codes.device
    if a_codes.dtype != torch.uint8 or b_codes.dtype != torch.uint8:
        raise TypeError("a_codes and b_codes must be uint8")
    _out(a_sf, "a_sf", torch.uint8, sf_mma_bytes(M, K, batch) if M and K else 0)
    _out(b_sf, "b_sf", torch.uint8, sf_mma_bytes(N, K, batch) if N and K else 0)
    _out(a_gscale, "a_gscale", torch.float32, 1), _out(b_gscale, "b_gscale", torch.float32, 1)
    if out is None:
        out = torch.empty((batch, M, N), dtype=out_dtype, device=dev)
    _out(out, "out", None, batch * M * N)
    if out.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("out must be float32 or bfloat16")
    if alpha_work is None:
        alpha_work = torch.empty(1, dtype=torch.float32, device=dev)
    _out(alpha_work, "alpha_work", torch.float32, 1)
    _check(lib().nvfp4_gemm_nt(_ptr(a_codes), _ptr(a_sf), _ptr(a_gscale), _ptr(b_codes), _ptr(b_sf), _ptr(b_gscale),
                               batch, M, N, K, float(alpha), _ptr(out), DTYPE_CODE[out.dtype], _ptr(alpha_work),
                               _stream(a_codes)))
    return out[0] if squeeze and out.dim() == 3 else out


def gemm_sf_offsets(rows: int, K: int, batch: int = 1):
    """Host-side: byte offsets at which gemm_nt reads scale (l, r, c), as a numpy int64 array."""
    import numpy as np
    out = np.empty(batch * rows * (K // 16), np.int64)
    _check(lib().nvfp4_gemm_sf_offsets(rows, K, batch, out.ctypes.data))
    return out


# ---- incremental KV cache (decode) ----
def kv_gscale(k: torch.Tensor, sink: int = 16, recent: int = 16, rotate: bool = True,
              out: torch.Tensor | None = None) -> torch.Tensor:
    """Tensor scale over the (rotated) middle tokens of K[B,H,T,D] (BF16), as kv_mixed computes it."""
    _cuda(k, "k")
    if k.dtype != torch.bfloat16 or k.dim() != 4:
        raise TypeError("k must be a 4-D bfloat16 tensor [B,H,T,D]")
    B, H, T, D = k.shape
    out = torch.empty(1, dtype=torch.float32, device=k.device) if out is None else _out(out, "out", torch.float32, 1)
    _check(lib().nvfp4_kv_gscale(_ptr(k), B, H, T, D, sink, recent, int(bool(rotate)), _ptr(out), _stream(k)))
    return out


def kv_append(k_rows: torch.Tensor, first: int, n: int, gscale: torch.Tensor, codes: torch.Tensor,
              scales: torch.Tensor, t0: int, rotate: bool = True, f_lo: int = -2, f_hi: int = 6,
              tile_layout: bool = False) -> None:
    """Quantize tokens [first, first+n) of k_rows [..., T, D] (BF16, contiguous; leading dims = batch x
    heads) with the tensor scale gscale into rows [t0, t0+n) of codes [..., cap, D/2] and scales
    ([..., cap, D/16], or the tile layout of the per-head [cap, D] matrices when tile_layout)."""
    for t, nm in ((k_rows, "k_rows"), (gscale, "gscale"), (codes, "codes"), (scales, "scales")):
        _cuda(t, nm)
    if k_rows.dtype != torch.bfloat16:
        raise TypeError("k_rows must be bfloat16")
    T, D = k_rows.shape[-2], k_rows.shape[-1]
    BH = k_rows.numel() // max(T * D, 1)
    cap = codes.shape[-2]
    _out(gscale, "gscale", torch.float32, 1), _out(codes, "codes", torch.uint8, BH * cap * (D // 2))
    _out(scales, "scales", torch.uint8, sf_mma_bytes(cap, D, BH) if tile_layout else BH * cap * (D // 16))
    _check(lib().nvfp4_kv_append(_ptr(k_rows), BH, T, first, n, D, int(bool(rotate)), f_lo, f_hi, _ptr(gscale),
                                 _ptr(codes), _ptr(scales), cap, t0, 1 if tile_layout else 0, _stream(k_rows)))


class _KvAppendDesc(ctypes.Structure):
    """nvfp4_kv_append_desc (include/nvfp4.h)."""
    _fields_ = [("k_bf16", _P), ("gscale", _P), ("codes", _P), ("scales", _P), ("BH", _I64), ("T", _I64),
                ("first", _I64), ("n", _I64), ("D", _I64), ("cap", _I64), ("t0", _I64),
                ("rotate", ctypes.c_int32), ("scale_layout", ctypes.c_int32)]


KV_APPEND_BATCH_MAX = 64


class KvAppendBatch:
    """A prepared nvfp4_kv_append_batch over fixed caches: `caches` is a sequence of tuples
    (k_rows, gscale, codes, scales, rotate, tile_layout) with kv_append's meanings, validated once (at most
    64, every tensor on one device; the tensors are kept alive).  Each call sets only the rows: first, n and t0 (an int for every item,
    or one value per item; n = 0 skips an item) and launches once.  Outputs of different items must not
    overlap."""

    def __init__(self, caches, f_lo: int = -2, f_hi: int = 6):
        caches = list(caches)
        if len(caches) > KV_APPEND_BATCH_MAX:
            raise ValueError(f"at most {KV_APPEND_BATCH_MAX} items per batch")
        self._keep, self.f_lo, self.f_hi = caches, f_lo, f_hi
        self._descs = (_KvAppendDesc * max(len(caches), 1))()
        self._device = None
        for i, (k_rows, gscale, codes, scales, rotate, tile_layout) in enumerate(caches):
            for t, nm in ((k_rows, "k_rows"), (gscale, "gscale"), (codes, "codes"), (scales, "scales")):
                _cuda(t, nm)
                # one launch on one device's stream reads and writes every item: all on that device
                self._device = self._device or t.device
                if t.device != self._device:
                    raise ValueError(f"item {i}: {nm} is on {t.device}, the batch runs on {self._device}")
            if k_rows.dtype != torch.bfloat16:
                raise TypeError("k_rows must be bfloat16")
            T, D = k_rows.shape[-2], k_rows.shape[-1]
            BH = k_rows.numel() // max(T * D, 1)
            cap = codes.shape[-2]
            _out(gscale, "gscale", torch.float32, 1), _out(codes, "codes", torch.uint8, BH * cap * (D // 2))
            _out(scales, "scales", torch.uint8, sf_mma_bytes(cap, D, BH) if tile_layout else BH * cap * (D // 16))
            self._descs[i] = _KvAppendDesc(k_rows.data_ptr(), gscale.data_ptr(), codes.data_ptr(), scales.data_ptr(),
                                           BH, T, 0, 0, D, cap, 0, int(bool(rotate)), 1 if tile_layout else 0)
        self._count = len(caches)

    def __len__(self) -> int:
        return self._count

    def __call__(self, first, n, t0) -> None:
        if self._count == 0:
            return
        d = self._descs
        one = [isinstance(v, numbers.Integral) for v in (first, n, t0)]
        for i in range(self._count):
            d[i].first = int(first if one[0] else first[i])
            d[i].n = int(n if one[1] else n[i])
            d[i].t0 = int(t0 if one[2] else t0[i])
        _check(lib().nvfp4_kv_append_batch(ctypes.cast(d, _P), self._count, self.f_lo, self.f_hi,
                                           ctypes.c_void_p(torch.cuda.current_stream(self._device).cuda_stream)))


def kv_append_batch(items, f_lo: int = -2, f_hi: int = 6) -> None:
    """Several kv_append calls in one launch.  `items`: a sequence of tuples
    (k_rows, first, n, gscale, codes, scales, t0, rotate, tile_layout) with kv_append's meanings; all use
    the window [f_lo, f_hi] (at most 32 offsets).  Outputs of different items must not overlap."""
    items = list(items)
    if len(items) > KV_APPEND_BATCH_MAX:
        raise ValueError(f"at most {KV_APPEND_BATCH_MAX} items per batch")
    if not items:
        return
    b = KvAppendBatch([(it[0], it[3], it[4], it[5], it[7], it[8]) for it in items], f_lo, f_hi)
    b([it[1] for it in items], [it[2] for it in items], [it[6] for it in items])


# ---- MXFP4 (comparison format) ----
def mxfp4_quantize(x: torch.Tensor, codes: torch.Tensor | None = None, scales: torch.Tensor | None = None):
    """MXFP4 (32-element blocks, E8M0 power-of-two scales).  Returns (codes uint8[n/2], scales uint8[n/32])."""
    _cuda(x, "x")
    n = x.numel()
    codes = torch.empty(n // 2, dtype=torch.uint8, device=x.device) if codes is None else _out(codes, "codes", torch.uint8, n // 2)
    scales = (torch.empty(n // 32, dtype=torch.uint8, device=x.device) if scales is None
              else _out(scales, "scales", torch.uint8, n // 32))
    _check(lib().nvfp4_mxfp4_quantize(_ptr(x), n, _dt(x), _ptr(codes), _ptr(scales), _stream(x)))
    return codes, scales


def mxfp4_dequantize(codes: torch.Tensor, scales: torch.Tensor, out_dtype=torch.float32,
                     out: torch.Tensor | None = None) -> torch.Tensor:
    _cuda(scales, "scales")
    n = scales.numel() * 32
    _out(codes, "codes", torch.uint8, n // 2)
    out = torch.empty(n, dtype=out_dtype, device=codes.device) if out is None else _out(out, "out", None, n)
    _check(lib().nvfp4_mxfp4_dequantize(_ptr(codes), _ptr(scales), n, DTYPE_CODE[out.dtype], _ptr(out),
                                        _stream(codes)))
    return out


# ---- multi-scale deformable attention forward on NVFP4 (or full-precision) values ----
def msda_forward(value, shapes, loc: torch.Tensor, w: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """value: a tensor [bs, nkeys, heads, ch] (float32 / bfloat16 / float16), or the NVFP4 triple
    (codes uint8 [bs, nkeys, heads, ch/2], scales uint8 [bs, nkeys, heads, ch/16], gscale float32[1]);
    shapes: sequence of (H_l, W_l); loc [bs, nq, heads, L, P, 2] and w [bs, nq, heads, L, P] float32.
    Returns out [bs, nq, heads, ch] float32."""
    import numpy as np
    _cuda(loc, "loc"), _cuda(w, "w")
    sh = np.ascontiguousarray(np.asarray(shapes, np.int64).reshape(-1, 2))
    bs, nq, heads, L, P, _ = loc.shape
    if isinstance(value, (tuple, list)):
        codes, scales, gscale = value
        _, nkeys, _, ch2 = codes.shape
        ch = 2 * ch2
        _out(codes, "codes", torch.uint8, bs * nkeys * heads * ch2)
        _out(scales, "scales", torch.uint8, bs * nkeys * heads * (ch // 16)), _out(gscale, "gscale", torch.float32, 1)
    else:
        _cuda(value, "value")
        _, nkeys, _, ch = value.shape
        _out(value, "value", None, bs * nkeys * heads * ch)
    _out(loc, "loc", torch.float32, bs * nq * heads * L * P * 2), _out(w, "w", torch.float32, bs * nq * heads * L * P)
    if out is None:
        out = torch.empty((bs, nq, heads, ch), dtype=torch.float32, device=loc.device)
    _out(out, "out", torch.float32, bs * nq * heads * ch)
    shp = sh.ctypes.data
    if isinstance(value, (tuple, list)):
        _check(lib().nvfp4_msda_forward_nvfp4(_ptr(codes), _ptr(scales), _ptr(gscale), bs, nkeys, heads, ch, shp,
                                              L, P, nq, _ptr(loc), _ptr(w), _ptr(out), _stream(loc)))
    else:
        _check(lib().nvfp4_msda_forward(_ptr(value), _dt(value), bs, nkeys, heads, ch, shp, L, P, nq, _ptr(loc),
                                        _ptr(w), _ptr(out), _stream(loc)))
    return out


# ---- FP4 attention (ScaleSearchAttention numerics, unfused) ----
def softmax_quantize_mma(s: torch.Tensor, causal: bool = False, q_offset: int = 0, f_lo: int = -2, f_hi: int = 6,
                         codes=None, sf=None, g=None, m=None, l=None):
    """s float32 [batch, Tq, Tk] (or [Tq, Tk]).  Returns (codes [.., Tq, Tk/2], sf tile layout, gscale[1],
    row_max [batch*Tq], row_sum [batch*Tq]) for the softmax numerators P~ = exp(S - m); outputs may be given."""
    _cuda(s, "s")
    batch, Tq, Tk = (1, *s.shape) if s.dim() == 2 else s.shape
    dev = s.device
    if s.dtype != torch.float32:
        raise TypeError("s must be float32")
    codes = torch.empty((*s.shape[:-1], Tk // 2), dtype=torch.uint8, device=dev) if codes is None else codes
    sf = torch.empty(max(sf_mma_bytes(Tq, Tk, batch), 1), dtype=torch.uint8, device=dev) if sf is None else sf
    g = torch.empty(1, dtype=torch.float32, device=dev) if g is None else g
    m = torch.empty(batch * Tq, dtype=torch.float32, device=dev) if m is None else m
    l = torch.empty(batch * Tq, dtype=torch.float32, device=dev) if l is None else l
    _out(codes, "codes", torch.uint8, batch * Tq * (Tk // 2)), _out(sf, "sf", torch.uint8, sf_mma_bytes(Tq, Tk, batch))
    _out(g, "g", torch.float32, 1), _out(m, "m", torch.float32, batch * Tq), _out(l, "l", torch.float32, batch * Tq)
    _check(lib().nvfp4_softmax_quantize_mma(_ptr(s), batch, Tq, Tk, int(bool(causal)), q_offset, f_lo, f_hi,
                                            _ptr(codes), _ptr(sf), _ptr(g), _ptr(m), _ptr(l), _stream(s)))
    return codes, sf, g, m, l


def rows_divide(x: torch.Tensor, l: torch.Tensor) -> torch.Tensor:
    """In place: x[r, :] /= l[r] for x float32 [..., cols] viewed as rows."""
    _cuda(x, "x")
    if x.dtype != torch.float32:
        raise TypeError("x must be float32")
    cols = x.shape[-1]
    _out(l, "l", torch.float32, x.numel() // max(cols, 1))
    _check(lib().nvfp4_rows_divide(_ptr(x), _ptr(l), x.numel() // max(cols, 1), cols, _stream(x)))
    return x


def _prologue_operand(x: torch.Tensor, rotate: bool, signs: int, f_lo: int, f_hi: int):
    """Q or K [H, T, D] as an NVFP4 tensor-core operand, Hadamard-rotated along D when `rotate`.  BF16
    input without signs takes the fused path (rotation inside the amax and search kernels, no FP32 copy);
    the result is bit-identical to quantize_mma(hadamard16(x, float32))."""
    x = x.contiguous()
    if rotate and signs == 0 and x.dtype == torch.bfloat16:
        _, _, codes, sf, g = kv_mixed_mma(x[None], 0, 0, True, f_lo, f_hi)
        return codes[0], sf, g
    if rotate:
        x = hadamard16(x, out_dtype=torch.float32, signs=signs)
    return quantize_mma(x, f_lo, f_hi)


def attention_fused_splits(H: int, Tq: int, Tk: int) -> int:
    """The key-range count nvfp4_attention_fused_splits chooses for the current device."""
    s = ctypes.c_int(0)
    _check(lib().nvfp4_attention_fused_splits(H, Tq, Tk, ctypes.byref(s)))
    return s.value


def attention_fused_workspace(H: int, Tq: int, Tk: int, splits: int, device) -> torch.Tensor:
    """A workspace for nvfp4_attention_fused (uint8, nvfp4_attention_fused_workspace_bytes long)."""
    n = lib().nvfp4_attention_fused_workspace_bytes(H, Tq, Tk, splits)
    if n == 0:
        raise NVFP4Error(-2)
    return torch.empty(n, dtype=torch.uint8, device=device)


def attention_fused(qc, qsf, qg, kc, ksf, kg, vc_t, vsf_t, vg, causal: bool = False, q_offset: int = 0,
                    alpha: float = 1.0, f_lo: int = -2, f_hi: int = 6, verify: bool = False, out=None, m=None, l=None,
                    status=None, splits: int | None = None, workspace=None):
    """nvfp4_attention_fused on NVFP4 operands: q (codes [H, Tq, D/2], tile-layout scales, g), k likewise for
    [H, Tk, D], v transposed (codes [H, D, Tk/2] and the tile layout of [D, Tk] matrices, as quantize_mma_t
    gives them).  splits: key ranges per query tile (None: attention_fused_splits); workspace: a uint8 tensor
    of attention_fused_workspace's size (None: allocated here).  Returns (O [H, Tq, D] float32, row_max,
    row_sum), and with verify=True also the scores [H, Tq, Tk] and P~ (codes, tile-layout scales)."""
    for t_, nm in ((qc, "q codes"), (qsf, "q scales"), (qg, "q g"), (kc, "k codes"), (ksf, "k scales"), (kg, "k g"),
                   (vc_t, "v codes"), (vsf_t, "v scales"), (vg, "v g")):
        _cuda(t_, nm)
    H, Tq, D = qc.shape[0], qc.shape[1], 2 * qc.shape[2]
    Tk = kc.shape[1]
    dev = qc.device
    if splits is None:
        splits = attention_fused_splits(H, Tq, Tk)
    if workspace is None:
        workspace = attention_fused_workspace(H, Tq, Tk, splits, dev)
    _cuda(workspace, "workspace")
    out = torch.empty((H, Tq, D), dtype=torch.float32, device=dev) if out is None else out
    m = torch.empty(H * Tq, dtype=torch.float32, device=dev) if m is None else m
    l = torch.empty(H * Tq, dtype=torch.float32, device=dev) if l is None else l
    status = torch.zeros(1, dtype=torch.int32, device=dev) if status is None else status
    _out(out, "out", torch.float32, H * Tq * D), _out(m, "m", torch.float32, H * Tq)
    _out(l, "l", torch.float32, H * Tq), _out(status, "status", torch.int32, 1)
    s_out = p_codes = p_sf = None
    if verify:
        s_out = torch.zeros((H, Tq, Tk), dtype=torch.float32, device=dev)
        p_codes = torch.full((H, Tq, Tk // 2), 0xEE, dtype=torch.uint8, device=dev)   # every byte is written
        p_sf = torch.full((max(sf_mma_bytes(Tq, Tk, H), 1),), 0xEE, dtype=torch.uint8, device=dev)
    _check(lib().nvfp4_attention_fused(_ptr(qc), _ptr(qsf), _ptr(qg), _ptr(kc), _ptr(ksf), _ptr(kg), _ptr(vc_t),
                                       _ptr(vsf_t), _ptr(vg), H, Tq, Tk, D, float(alpha), int(bool(causal)), q_offset,
                                       f_lo, f_hi, int(splits), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                       _ptr(out), _ptr(m), _ptr(l), _ptr(s_out), _ptr(p_codes), _ptr(p_sf),
                                       _ptr(status), _stream(qc)))
    if verify:
        return out, m, l, s_out, p_codes, p_sf, status
    return out, m, l


def attention_fp4_fused(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False, rotate: bool = True,
                        scale: float | None = None, f_lo: int = -2, f_hi: int = 6, signs: int = 0):
    """attention_fp4 with the scores kept on chip: the same NVFP4 prologue (Q and K rotated and quantized into
    the tile layout, V quantized along the tokens), then nvfp4_attention_fused.  q [H, Tq, D], k and v
    [H, Tk, D] with D = 128, Tq % 128 == 0, Tk % 64 == 0.  Returns O [H, Tq, D] float32."""
    H, Tq, D = q.shape
    Tk = k.shape[1]
    scale = D ** -0.5 if scale is None else scale
    qc, qsf, qg = _prologue_operand(q, rotate, signs, f_lo, f_hi)
    kc, ksf, kg = _prologue_operand(k, rotate, signs, f_lo, f_hi)
    vc, vsf, vg = quantize_mma_t(v.contiguous(), f_lo, f_hi)
    o, _, _ = attention_fused(qc.view(H, Tq, D // 2), qsf, qg, kc.view(H, Tk, D // 2), ksf, kg,
                              vc.view(H, D, Tk // 2), vsf, vg, causal, Tk - Tq, scale, f_lo, f_hi)
    return o


def attention_fp4(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False, rotate: bool = True,
                  scale: float | None = None, f_lo: int = -2, f_hi: int = 6, signs: int = 0):
    """Attention with every product in NVFP4 on the tensor cores ("Search your block floating-point
    scales!", ScaleSearchAttention; unfused): q [H, Tq, D], k and v [H, Tk, D].
      rotate: Hadamard-16 along D on q and k (Q K^T unchanged, outliers spread), after the sign
        diagonal given by the 16-bit mask `signs` (the same for both, so Q K^T is still unchanged);
      S = scale * Q K^T (NVFP4 x NVFP4, FP32 accumulation);  P~ = exp(S - rowmax) quantized with ScaleSearch;
      O = (P~ V) / rowsum with V quantized along the tokens.  Causal: query i sees keys <= i + Tk - Tq.
    Returns O [H, Tq, D] float32."""
    H, Tq, D = q.shape
    Tk = k.shape[1]
    scale = D ** -0.5 if scale is None else scale
    qc, qsf, qg = _prologue_operand(q, rotate, signs, f_lo, f_hi)
    kc, ksf, kg = _prologue_operand(k, rotate, signs, f_lo, f_hi)
    s = gemm_nt(qc, qsf, qg, kc, ksf, kg, alpha=scale)
    pc, psf, pg, _, l = softmax_quantize_mma(s, causal, Tk - Tq, f_lo, f_hi)
    vc, vsf, vg = quantize_mma_t(v.contiguous(), f_lo, f_hi)
    o = gemm_nt(pc, psf, pg, vc, vsf, vg)
    return rows_divide(o, l)
