"""ctypes wrapper around the C oracle (``nvfp4_ref.c``).

TEST INFRASTRUCTURE ONLY.  This is the plain CPU definition of NVFP4 block quantization with
ScaleSearch that the CUDA library is checked against.  Only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline leg may import it; the library never does.

All array arguments are numpy arrays (contiguous); results come back as new numpy arrays.
Element types use the codes 0 = float32, 1 = bfloat16 (stored as uint16), 2 = float16.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_ref.c")
_SO = os.path.join(_HERE, "libnvfp4_ref.so")
CFLAGS = ["-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-Wall"]

F32, BF16, F16 = 0, 1, 2
_NP_OF = {F32: np.float32, BF16: np.uint16, F16: np.uint16}

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libnvfp4_ref.so`` with gcc (strict IEEE flags)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "nvfp4_ref.h"))
    ):
        subprocess.run(["gcc", *CFLAGS, "-o", _SO, _SRC, "-lm"], check=True)
    return _SO


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        P, I64, I, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
        sig = {
            "ref_e2m1_encode": (ctypes.c_uint8, [F]),
            "ref_e2m1_decode": (F, [ctypes.c_uint8]),
            "ref_e4m3_encode": (ctypes.c_uint8, [F]),
            "ref_e4m3_decode": (F, [ctypes.c_uint8]),
            "ref_e2m1_encode_n": (None, [P, I64, P]),
            "ref_e4m3_encode_n": (None, [P, I64, P]),
            "ref_f32_to_bf16_n": (None, [P, I64, P]),
            "ref_f32_to_f16_n": (None, [P, I64, P]),
            "ref_f16_to_f32_n": (None, [P, I64, P]),
            "ref_tensor_amax": (F, [P, I64, I]),
            "ref_global_scale": (F, [F]),
            "ref_search_block": (None, [P, F, I, I, P, P, P, P]),
            "ref_maxscale_block": (None, [P, F, P, P, P]),
            "ref_quantize": (I, [P, I64, I, I, I, P, P, P, P, P, P]),
            "ref_quantize_blocks": (None, [P, I, I64, I64, F, I, I, P, P, P, P]),
            "ref_dequantize": (I, [P, P, F, I64, I, P]),
            "ref_hadamard16": (I, [P, I64, I, P, I]),
            "ref_hadamard16_ex": (I, [P, I64, I, P, I, ctypes.c_uint32, I]),
            "ref_fwht16_f32": (None, [P]),
            "ref_kv_mixed": (I, [P, I64, I64, I64, I64, I, I, I, I, I, P, P, P, P, P]),
            "ref_exp_ss": (F, [F]),
            "ref_softmax_quantize": (I, [P, I64, I64, I64, I, I64, I, I, P, P, P, P]),
            "ref_msda_forward": (I, [P, P, P, P, P, I64, I64, I64, I64, I64, I64, I64, P]),
            "ref_mxfp4_quantize": (I, [P, I64, I, P, P]),
            "ref_mxfp4_dequantize": (I, [P, P, I64, I, P]),
            "ref_kv_append": (I, [P, I64, I64, I64, I64, I64, I, F, I, I, P, P, I64, I64]),
            "ref_sf_mma_bytes": (I64, [I64, I64]),
            "ref_sf_mma_offset": (I64, [I64, I64, I64]),
            "ref_scales_to_mma": (None, [P, I64, I64, I64, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _dtype_of(x: np.ndarray) -> int:
    if x.dtype == np.float32:
        return F32
    raise TypeError("pass float32 arrays, or uint16 arrays with an explicit dtype code")


# ---- scalar / array converters ----
def e2m1_encode(y: np.ndarray) -> np.ndarray:
    y = np.ascontiguousarray(y, np.float32)
    out = np.empty(y.shape, np.uint8)
    lib().ref_e2m1_encode_n(_p(y), y.size, _p(out))
    return out


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().ref_e4m3_encode_n(_p(v), v.size, _p(out))
    return out


def e2m1_decode(code: int) -> float:
    return float(lib().ref_e2m1_decode(code))


def e4m3_decode(code: int) -> float:
    return float(lib().ref_e4m3_decode(code))


def f32_to_bf16(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, np.float32)
    out = np.empty(v.shape, np.uint16)
    lib().ref_f32_to_bf16_n(_p(v), v.size, _p(out))
    return out


def f32_to_f16(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, np.float32)
    out = np.empty(v.shape, np.uint16)
    lib().ref_f32_to_f16_n(_p(v), v.size, _p(out))
    return out


def f16_to_f32(h: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(h, np.uint16)
    out = np.empty(h.shape, np.float32)
    lib().ref_f16_to_f32_n(_p(h), h.size, _p(out))
    return out


# ---- tensor steps ----
def tensor_amax(x: np.ndarray, dtype: int | None = None) -> np.float32:
    x = np.ascontiguousarray(x)
    dtype = _dtype_of(x) if dtype is None else dtype
    return np.float32(lib().ref_tensor_amax(_p(x), x.size, dtype))


def global_scale(amax) -> np.float32:
    return np.float32(lib().ref_global_scale(float(amax)))


def search_block(x16: np.ndarray, g, f_lo: int, f_hi: int):
    x16 = np.ascontiguousarray(x16, np.float32)
    assert x16.size == 16
    codes = np.zeros(8, np.uint8)
    sc = np.zeros(1, np.uint8)
    fs = np.zeros(1, np.int8)
    sse = np.zeros(1, np.float32)
    lib().ref_search_block(_p(x16), float(g), f_lo, f_hi, _p(codes), _p(sc), _p(fs), _p(sse))
    return codes, int(sc[0]), int(fs[0]), sse[0]


def maxscale_block(x16: np.ndarray, g):
    x16 = np.ascontiguousarray(x16, np.float32)
    codes = np.zeros(8, np.uint8)
    sc = np.zeros(1, np.uint8)
    sse = np.zeros(1, np.float32)
    lib().ref_maxscale_block(_p(x16), float(g), _p(codes), _p(sc), _p(sse))
    return codes, int(sc[0]), sse[0]


def quantize(x: np.ndarray, f_lo: int = -2, f_hi: int = 6, dtype: int | None = None, gscale_in=None):
    """Returns (codes[n/2], scales[n/16], g, block_f[n/16], block_sse[n/16])."""
    x = np.ascontiguousarray(x)
    dtype = _dtype_of(x) if dtype is None else dtype
    n = x.size
    nb = n // 16
    codes = np.empty(n // 2, np.uint8)
    scales = np.empty(nb, np.uint8)
    bf = np.empty(nb, np.int8)
    bs = np.empty(nb, np.float32)
    g = np.zeros(1, np.float32)
    gin = None if gscale_in is None else np.array([gscale_in], np.float32)
    rc = lib().ref_quantize(_p(x), n, dtype, f_lo, f_hi, _p(gin), _p(codes), _p(scales), _p(g), _p(bf), _p(bs))
    if rc != 0:
        raise ValueError(f"ref_quantize returned {rc}")
    return codes, scales, g[0], bf, bs


def quantize_blocks(x: np.ndarray, b0: int, b1: int, g, f_lo: int = -2, f_hi: int = 6, dtype: int | None = None):
    x = np.ascontiguousarray(x)
    dtype = _dtype_of(x) if dtype is None else dtype
    nb = b1 - b0
    codes = np.empty(nb * 8, np.uint8)
    scales = np.empty(nb, np.uint8)
    bf = np.empty(nb, np.int8)
    bs = np.empty(nb, np.float32)
    lib().ref_quantize_blocks(_p(x), dtype, b0, b1, float(g), f_lo, f_hi, _p(codes), _p(scales), _p(bf), _p(bs))
    return codes, scales, bf, bs


def dequantize(codes: np.ndarray, scales: np.ndarray, g, out_dtype: int = F32) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    n = scales.size * 16
    out = np.empty(n, _NP_OF[out_dtype])
    rc = lib().ref_dequantize(_p(codes), _p(scales), float(g), n, out_dtype, _p(out))
    if rc != 0:
        raise ValueError(f"ref_dequantize returned {rc}")
    return out


def hadamard16(x: np.ndarray, dtype: int | None = None, out_dtype: int = F32) -> np.ndarray:
    x = np.ascontiguousarray(x)
    dtype = _dtype_of(x) if dtype is None else dtype
    out = np.empty(x.size, _NP_OF[out_dtype])
    rc = lib().ref_hadamard16(_p(x), x.size, dtype, _p(out), out_dtype)
    if rc != 0:
        raise ValueError(f"ref_hadamard16 returned {rc}")
    return out


def hadamard16_ex(x: np.ndarray, signs: int, inverse: bool = False, dtype: int | None = None,
                  out_dtype: int = F32) -> np.ndarray:
    """(H16/4) D x, or D (H16/4) x when inverse; D negates element i of each group when bit i of signs is set."""
    x = np.ascontiguousarray(x)
    dtype = _dtype_of(x) if dtype is None else dtype
    out = np.empty(x.size, _NP_OF[out_dtype])
    rc = lib().ref_hadamard16_ex(_p(x), x.size, dtype, _p(out), out_dtype, signs, int(inverse))
    if rc != 0:
        raise ValueError(f"ref_hadamard16_ex returned {rc}")
    return out


def kv_mixed(k_bf16: np.ndarray, sink: int = 16, recent: int = 16, rotate: int = 1, f_lo: int = -2, f_hi: int = 6):
    """k_bf16: uint16 array [B,H,T,D].  Returns (sink[B,H,sink,D], recent[B,H,recent,D],
    codes[B,H,Tm,D/2], scales[B,H,Tm,D/16], g)."""
    k = np.ascontiguousarray(k_bf16, np.uint16)
    B, H, T, D = k.shape
    Tm = T - sink - recent
    so = np.empty((B, H, sink, D), np.uint16)
    ro = np.empty((B, H, recent, D), np.uint16)
    codes = np.empty((B, H, Tm, D // 2), np.uint8)
    scales = np.empty((B, H, Tm, D // 16), np.uint8)
    g = np.zeros(1, np.float32)
    rc = lib().ref_kv_mixed(_p(k), B, H, T, D, sink, recent, rotate, f_lo, f_hi, _p(so), _p(ro), _p(codes), _p(scales), _p(g))
    if rc != 0:
        raise ValueError(f"ref_kv_mixed returned {rc}")
    return so, ro, codes, scales, g[0]


# ---- tensor-core consumer: block-scale tile layout and the NVFP4 product ----
def sf_mma_bytes(rows: int, bpr: int) -> int:
    """Bytes of one [rows, bpr] scale matrix in the 128x4 tile layout (padded)."""
    return int(lib().ref_sf_mma_bytes(rows, bpr))


def sf_mma_offset(r: int, c: int, bpr: int) -> int:
    return int(lib().ref_sf_mma_offset(r, c, bpr))


def scales_to_mma(scales: np.ndarray, batch: int, rows: int, bpr: int) -> np.ndarray:
    """Row-major [batch, rows, bpr] scale bytes -> the tile layout (padding zero)."""
    lin = np.ascontiguousarray(scales, np.uint8).reshape(-1)
    if lin.size != batch * rows * bpr:
        raise ValueError("scales size does not match batch * rows * bpr")
    out = np.empty(batch * sf_mma_bytes(rows, bpr), np.uint8)
    lib().ref_scales_to_mma(_p(lin), batch, rows, bpr, _p(out))
    return out


def quantize_mma(x: np.ndarray, f_lo: int = -2, f_hi: int = 6, dtype: int | None = None, gscale_in=None):
    """Quantize x [batch, rows, cols] (or [rows, cols]) along cols; scales in the tile layout.

    Returns (codes [batch*rows*cols/2], sf_mma, g)."""
    if x.ndim == 2:
        x = x[None]
    batch, rows, cols = x.shape
    codes, scales, g, _, _ = quantize(x.reshape(-1), f_lo, f_hi, dtype, gscale_in)
    return codes, scales_to_mma(scales, batch, rows, cols // 16), g


_E2M1_TAB = None
_E4M3_TAB = None


def _tables():
    global _E2M1_TAB, _E4M3_TAB
    if _E2M1_TAB is None:
        _E2M1_TAB = np.array([e2m1_decode(c) for c in range(16)], np.float64)
        _E4M3_TAB = np.array([e4m3_decode(c) for c in range(256)], np.float64)
    return _E2M1_TAB, _E4M3_TAB


def block_values(codes: np.ndarray, scales: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """Exact real values E2M1(q) * E4M3(s) (without the tensor scale) of a [rows, cols] matrix, fp64."""
    t2, t4 = _tables()
    c = np.ascontiguousarray(codes, np.uint8).reshape(rows, cols // 2)
    q = np.empty((rows, cols), np.uint8)
    q[:, 0::2] = c & 15      # element 2k: low nibble
    q[:, 1::2] = c >> 4      # element 2k+1: high nibble
    sv = t4[np.ascontiguousarray(scales, np.uint8).reshape(rows, cols // 16)]
    return t2[q] * np.repeat(sv, 16, axis=1)


def gemm_nt(a_codes, a_scales, g_a, b_codes, b_scales, g_b, M: int, N: int, K: int, alpha: float = 1.0,
            batch: int = 1) -> np.ndarray:
    """D[l] = alpha * g_a * g_b * A[l] B[l]^T in fp64 from row-major codes and row-major (linear) scales.

    Each product of two E2M1 values and two E4M3 scales is exact in fp64; the sums are a library matmul."""
    A = np.ascontiguousarray(a_codes).reshape(batch, -1)
    As = np.ascontiguousarray(a_scales).reshape(batch, -1)
    B = np.ascontiguousarray(b_codes).reshape(batch, -1)
    Bs = np.ascontiguousarray(b_scales).reshape(batch, -1)
    out = np.empty((batch, M, N), np.float64)
    scale = float(alpha) * float(g_a) * float(g_b)
    for l in range(batch):
        av = block_values(A[l], As[l], M, K)
        bv = block_values(B[l], Bs[l], N, K)
        out[l] = (av @ bv.T) * scale
    return out


def kv_append(k_rows: np.ndarray, first: int, n: int, g, codes: np.ndarray, scales: np.ndarray, t0: int,
              rotate: int = 1, f_lo: int = -2, f_hi: int = 6) -> None:
    """Quantize tokens [first, first+n) of every (batch, head) of k_rows (uint16 BF16 [BH, T, D]) with the
    tensor scale g into rows [t0, t0+n) of codes [BH, cap, D/2] / scales [BH, cap, D/16], in place."""
    k = np.ascontiguousarray(k_rows, np.uint16)
    BH, T, D = k.shape
    cap = codes.shape[1]
    assert codes.flags.c_contiguous and scales.flags.c_contiguous
    rc = lib().ref_kv_append(_p(k), BH, T * D, first, n, D, rotate, float(g), f_lo, f_hi, _p(codes), _p(scales),
                             cap, t0)
    if rc != 0:
        raise ValueError(f"ref_kv_append returned {rc}")


# ---- MXFP4 (comparison format) ----
def mxfp4_quantize(x: np.ndarray, dtype: int | None = None):
    """(codes n/2, E8M0 scales n/32) of x (n % 32 == 0)."""
    x = np.ascontiguousarray(x).reshape(-1)
    dtype = _dtype_of(x) if dtype is None else dtype
    codes = np.empty(x.size // 2, np.uint8)
    scales = np.empty(x.size // 32, np.uint8)
    rc = lib().ref_mxfp4_quantize(_p(x), x.size, dtype, _p(codes), _p(scales))
    if rc != 0:
        raise ValueError(f"ref_mxfp4_quantize returned {rc}")
    return codes, scales


def mxfp4_dequantize(codes: np.ndarray, scales: np.ndarray, out_dtype: int = F32) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    n = scales.size * 32
    out = np.empty(n, _NP_OF[out_dtype])
    rc = lib().ref_mxfp4_dequantize(_p(codes), _p(scales), n, out_dtype, _p(out))
    if rc != 0:
        raise ValueError(f"ref_mxfp4_dequantize returned {rc}")
    return out


# ---- multi-scale deformable attention forward ----
def msda_forward(value: np.ndarray, shapes, loc: np.ndarray, w: np.ndarray) -> np.ndarray:
    """value float32 [bs, nkeys, heads, ch]; shapes [(H_l, W_l)]; loc float32 [bs, nq, heads, L, P, 2];
    w float32 [bs, nq, heads, L, P].  Returns float64 [bs, nq, heads, ch]."""
    value = np.ascontiguousarray(value, np.float32)
    loc = np.ascontiguousarray(loc, np.float32)
    w = np.ascontiguousarray(w, np.float32)
    bs, nkeys, heads, ch = value.shape
    _, nq, _, L, P, _ = loc.shape
    sh = np.ascontiguousarray(np.asarray(shapes, np.int64).reshape(L, 2))
    start = np.ascontiguousarray(np.concatenate([[0], np.cumsum(sh[:, 0] * sh[:, 1])[:-1]]).astype(np.int64))
    assert int((sh[:, 0] * sh[:, 1]).sum()) == nkeys
    out = np.empty((bs, nq, heads, ch), np.float64)
    lib().ref_msda_forward(_p(value), _p(sh), _p(start), _p(loc), _p(w), bs, nkeys, heads, ch, L, P, nq, _p(out))
    return out


def quantize_mma_t(x: np.ndarray, f_lo: int = -2, f_hi: int = 6, dtype: int | None = None, gscale_in=None):
    """x [batch, rows, cols] (or [rows, cols]) quantized in blocks of 16 rows per column: the tile-layout
    quantization of the transposed matrices.  Returns (codes [batch*cols*rows/2], sf_mma, g)."""
    if x.ndim == 2:
        x = x[None]
    return quantize_mma(np.ascontiguousarray(np.swapaxes(x, 1, 2)), f_lo, f_hi, dtype, gscale_in)


# ---- FP4 attention softmax ----
def exp_ss(x) -> np.float32:
    return np.float32(lib().ref_exp_ss(float(x)))


def softmax_quantize(s: np.ndarray, causal: bool = False, q_offset: int = 0, f_lo: int = -2, f_hi: int = 6):
    """s float32 [batch, Tq, Tk].  Returns (codes [batch,Tq,Tk/2], scales [batch,Tq,Tk/16] (row-major),
    row_max [batch,Tq], row_sum [batch,Tq], g) for P~ = exp(S - m) quantized with g = fl(1/2688)."""
    s = np.ascontiguousarray(s, np.float32)
    batch, Tq, Tk = s.shape
    codes = np.empty((batch, Tq, Tk // 2), np.uint8)
    scales = np.empty((batch, Tq, Tk // 16), np.uint8)
    m = np.empty((batch, Tq), np.float32)
    l = np.empty((batch, Tq), np.float32)
    rc = lib().ref_softmax_quantize(_p(s), batch, Tq, Tk, int(bool(causal)), q_offset, f_lo, f_hi, _p(codes),
                                    _p(scales), _p(m), _p(l))
    if rc != 0:
        raise ValueError(f"ref_softmax_quantize returned {rc}")
    return codes, scales, m, l, global_scale(1.0)
