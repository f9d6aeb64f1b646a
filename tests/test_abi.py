"""The C-ABI library loads and exports every symbol include/nvfp4.h declares; argument validation
rejects bad calls synchronously (these calls return before any CUDA work, so no GPU is needed)."""
import ctypes
import os
import re

import pytest

import nvfp4_block_scaled_11_b200 as nv
from nvfp4_block_scaled_11_b200 import build as nvbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "include", "nvfp4.h")


def _declared():
    src = open(HDR).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    nvbuild.build()
    return nv.lib()


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert len(names) >= 9
    for name in names:
        assert hasattr(L, name), name
        assert name in nv._SIGS, f"binding lacks {name}"


def test_status_strings(L):
    for code in (0, -1, -2, -3, -4, -5):
        assert nv.status_str(code).startswith("NVFP4")
    assert L.nvfp4_version() >= 100


V = ctypes.c_void_p


def test_quantize_argument_errors(L):
    fake = V(0x10000)  # 16-byte aligned, never dereferenced: validation fails first
    codes, scales, g = V(0x20000), V(0x30000), V(0x40000)
    # n not a multiple of 16
    assert L.nvfp4_quantize(fake, 17, 0, 16, -2, 6, codes, scales, g, None) == -2
    assert L.nvfp4_quantize(fake, -16, 0, 16, -2, 6, codes, scales, g, None) == -2
    # block != 16, bad dtype, bad window, missing gscale
    assert L.nvfp4_quantize(fake, 32, 0, 32, -2, 6, codes, scales, g, None) == -1
    assert L.nvfp4_quantize(fake, 32, 7, 16, -2, 6, codes, scales, g, None) == -1
    assert L.nvfp4_quantize(fake, 32, 0, 16, 3, 2, codes, scales, g, None) == -1
    assert L.nvfp4_quantize(fake, 32, 0, 16, -200, 6, codes, scales, g, None) == -1
    assert L.nvfp4_quantize(fake, 32, 0, 16, -2, 6, codes, scales, None, None) == -1
    assert L.nvfp4_quantize(None, 32, 0, 16, -2, 6, codes, scales, g, None) == -1
    # misaligned input / codes
    assert L.nvfp4_quantize(V(0x10008), 32, 0, 16, -2, 6, codes, scales, g, None) == -3
    assert L.nvfp4_quantize(fake, 32, 0, 16, -2, 6, V(0x20004), scales, g, None) == -3


def test_other_entry_point_errors(L):
    fake = V(0x10000)
    assert L.nvfp4_dequantize(fake, fake, fake, 24, 0, fake, None) == -2
    assert L.nvfp4_dequantize(fake, fake, None, 32, 0, fake, None) == -1
    assert L.nvfp4_dequantize(fake, fake, fake, 32, 9, fake, None) == -1
    assert L.nvfp4_dequantize(fake, fake, fake, 32, 0, V(0x10004), None) == -3
    assert L.nvfp4_hadamard16(fake, 20, 0, fake, 0, None) == -2
    assert L.nvfp4_hadamard16(fake, 32, 0, fake, 1, None) == -1  # in place across dtypes
    assert L.nvfp4_hadamard16_ex(fake, 32, 0, fake, 0, 0x10000, 0, None) == -1   # signs beyond 16 bits
    assert L.nvfp4_hadamard16_ex(fake, 32, 0, fake, 0, 0x00FF, 2, None) == -1     # inverse not 0/1
    assert L.nvfp4_hadamard16_ex(fake, 20, 0, fake, 0, 0x00FF, 1, None) == -2
    assert L.nvfp4_tensor_amax(fake, 10, 5, fake, None) == -1
    assert L.nvfp4_tensor_amax(V(0x10002), 10, 0, fake, None) == -3
    assert L.nvfp4_global_scale(None, fake, None) == -1
    # kv: T smaller than sink + recent, D not a multiple of 16
    assert L.nvfp4_kv_mixed(fake, 1, 1, 20, 128, 16, 16, 1, -2, 6, fake, fake, fake, fake, fake, None) == -2
    assert L.nvfp4_kv_mixed(fake, 1, 1, 64, 120, 16, 16, 1, -2, 6, fake, fake, fake, fake, fake, None) == -2
    assert L.nvfp4_kv_mixed(fake, 1, 1, 64, 128, 16, 16, 1, 5, 4, fake, fake, fake, fake, fake, None) == -1
    assert L.nvfp4_quantize_ex(fake, 32, 0, 16, -2, 6, None, fake, fake, None, None, None, None) == -1


def test_attention_fused_host_checks(L):
    """The fused attention's workspace size and its argument errors, all decided on the host before any
    launch (fake device pointers; no GPU needed)."""
    W = L.nvfp4_attention_fused_workspace_bytes
    # maxima only (one range), plus sums and accumulators (several), rounded to 256, then Q, K, V^T tiles
    assert W(2, 256, 512, 1) == (2 * 256 * 4 + 255) // 256 * 256 + (2 * 512 + 256) * 2 * 128 * 2
    assert W(2, 256, 512, 3) == (3 * 512 * 4 + 3 * 512 * 129 * 4 + 255) // 256 * 256 + (2 * 512 + 256) * 2 * 128 * 2
    for bad in ((-1, 128, 64, 1), (1, 128, 63, 1), (1, 128, 64, 0), (1, 128, 64, 65)):
        assert W(*bad) == 0, bad
    fake = V(0x10000)
    ws_ok = W(1, 128, 64, 1)

    def call(Tq=128, Tk=64, D=128, lo=-2, hi=6, splits=1, ws=fake, wsb=ws_ok, kc=fake, ksf=fake, out=fake, pc=None,
             psf=None):
        return L.nvfp4_attention_fused(fake, fake, fake, kc, ksf, fake, fake, fake, fake, 1, Tq, Tk, D,
                                       ctypes.c_float(1.0), 1, 0, lo, hi, splits, ws, wsb, out, fake, fake, None, pc,
                                       psf, None, None)
    assert call(Tq=100) == -2 and call(Tk=48) == -2 and call(D=64) == -2 and call(Tk=1 << 26) == -2
    assert call(lo=-2, hi=5) == -1 and call(lo=0, hi=-1) == -1          # 8 offsets; empty window
    assert call(splits=0) == -1 and call(splits=65) == -1
    assert call(ws=None) == -1 and call(wsb=ws_ok - 1) == -2             # no workspace; too small
    assert call(pc=fake) == -1                                           # codes without scales
    assert call(kc=V(0x10004)) == -3 and call(ksf=V(0x10002)) == -3 and call(out=V(0x10008)) == -3
    assert call(ws=V(0x10008)) == -3
    assert L.nvfp4_attention_fused(fake, fake, fake, fake, fake, fake, fake, fake, fake, 0, 128, 64, 128,
                                   ctypes.c_float(1.0), 1, 0, -2, 6, 1, None, 0, None, None, None, None, None, None,
                                   None, None) == 0                       # no heads: nothing to do


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(TypeError):
        nv.quantize(torch.zeros(32))


def test_size_products_that_overflow_are_rejected(L):
    """Sizes whose products do not fit in 64 bits come back as NVFP4_ERR_SIZE before anything runs."""
    fake, big = V(0x10000), 1 << 40
    assert L.nvfp4_quantize_mma(fake, big, big, 16 * big, 0, -2, 6, None, fake, fake, fake, None) == -2
    assert L.nvfp4_quantize_mma_t(fake, big, 16 * big, big, 0, -2, 6, None, fake, fake, fake, None) == -2
    assert L.nvfp4_sf_mma_bytes(big, 16 * big, big) == -2
    assert L.nvfp4_kv_mixed(fake, big, big, big, 128, 16, 16, 1, -2, 6, fake, fake, fake, fake, fake, None) == -2
    assert L.nvfp4_kv_gscale(fake, big, big, big, 128, 16, 16, 1, fake, None) == -2
    assert L.nvfp4_softmax_quantize_mma(fake, big, big, 16 * big, 1, 0, -2, 6, fake, fake, fake, fake, fake, None) == -2
    assert L.nvfp4_rows_divide(fake, fake, big, 4 * big, None) == -2
    assert L.nvfp4_kv_append(fake, big, big, 0, 16, 128, 1, -2, 6, fake, fake, fake, big, 0, 0, None) == -2
    assert L.nvfp4_gemm_nt(fake, fake, fake, fake, fake, fake, 1 << 30, 1 << 30, 1 << 30, 32, 1.0, fake, 0, fake,
                           None) == -2
    huge = 1 << 61
    assert L.nvfp4_quantize(fake, huge, 0, 16, -2, 6, fake, fake, fake, None) == -2
    assert L.nvfp4_dequantize(fake, fake, fake, huge, 0, fake, None) == -2
    assert L.nvfp4_hadamard16(fake, huge, 0, fake, 0, None) == -2
    assert L.nvfp4_tensor_amax(fake, huge, 0, fake, None) == -2
    assert L.nvfp4_mxfp4_quantize(fake, huge, 0, fake, fake, None) == -2


def test_search_policy_is_host_only_and_restorable():
    """The launch-policy call touches no device: its defaults, set / restore and argument errors."""
    default = nv.search_policy()
    assert default == (65536, 393216)
    try:
        assert nv.search_policy(10, 20) == default
        assert nv.search_policy(None, 30) == (10, 20)
        assert nv.search_policy() == (10, 30)
        with pytest.raises(nv.NVFP4Error):
            nv.search_policy(-5, None)
        assert nv.search_policy() == (10, 30)
    finally:
        nv.search_policy(*default)
    assert nv.search_policy() == default


def test_kv_append_batch_validates_on_the_host(L):
    """Argument errors of the batched KV append come back before any device call: too many items, a
    window wider than 32 offsets, an item with a bad head_dim or rows past the cache."""
    D = nv._KvAppendDesc
    fake = 1 << 20   # never dereferenced: every case fails validation first
    ok = D(fake, fake, fake, fake, 2, 32, 0, 16, 64, 64, 0, 1, 0)
    arr = (D * 65)(*([ok] * 65))
    assert L.nvfp4_kv_append_batch(ctypes.cast(arr, ctypes.c_void_p), 65, -2, 6, None) == -1
    assert L.nvfp4_kv_append_batch(ctypes.cast(arr, ctypes.c_void_p), 1, -16, 16, None) == -1
    assert L.nvfp4_kv_append_batch(None, 1, -2, 6, None) == -1
    assert L.nvfp4_kv_append_batch(None, 0, -2, 6, None) == 0
    bad_d = D(fake, fake, fake, fake, 2, 32, 0, 16, 60, 64, 0, 1, 0)
    past = D(fake, fake, fake, fake, 2, 32, 0, 16, 64, 64, 50, 1, 0)
    badrot = D(fake, fake, fake, fake, 2, 32, 0, 16, 64, 64, 0, 2, 0)
    for d, want in ((bad_d, -2), (past, -2), (badrot, -1)):
        arr2 = (D * 2)(ok, d)
        assert L.nvfp4_kv_append_batch(ctypes.cast(arr2, ctypes.c_void_p), 2, -2, 6, None) == want


def test_kv_append_batch_rejects_a_grid_too_large(L):
    """Each item stays below 2^32 blocks, but 64 such items need more CTAs than a grid holds: the call
    returns NVFP4_ERR_SIZE on the host (the fake pointers are never dereferenced)."""
    D = nv._KvAppendDesc
    fake = 1 << 20
    # BH = 1, D = 16: n rows are n blocks; 2^32 - 1 blocks per item, 64 items
    big = D(fake, fake, fake, fake, 1, (1 << 32) - 1, 0, (1 << 32) - 1, 16, (1 << 32) - 1, 0, 0, 0)
    arr = (D * 64)(*([big] * 64))
    for lo, hi in ((-2, 6), (-1, 1), (-8, 8), (-16, 15)):   # 4, 4, 8 and 8 lanes per block
        assert L.nvfp4_kv_append_batch(ctypes.cast(arr, ctypes.c_void_p), 64, lo, hi, None) == -2


def test_kv_append_desc_layout_matches_the_header(tmp_path):
    """The binding's ctypes mirror of nvfp4_kv_append_desc has the C struct's size and field offsets
    (a C program built against the header prints them)."""
    import subprocess
    fields = [f for f, _ in nv._KvAppendDesc._fields_]
    src = tmp_path / "layout.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "nvfp4.h"\nint main(void) {\n'
                   '  printf("%zu", sizeof(nvfp4_kv_append_desc));\n'
                   + "".join(f'  printf(" %zu", offsetof(nvfp4_kv_append_desc, {f}));\n' for f in fields)
                   + '  printf("\\n");\n  return 0;\n}\n')
    exe = tmp_path / "layout"
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    subprocess.run(["gcc", "-std=c99", "-I", inc, str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()]
    want = [ctypes.sizeof(nv._KvAppendDesc)] + [getattr(nv._KvAppendDesc, f).offset for f in fields]
    assert got == want


def _ctype_of(decl: str):
    """ctypes class the binding must use for one C parameter or return declaration."""
    d = " ".join(decl.replace("const", " ").split())
    if "*" in d:
        return ctypes.c_char_p if d.startswith("char") else ctypes.c_void_p
    base = d.rsplit(" ", 1)[0] if " " in d else d
    return {"int64_t": ctypes.c_int64, "int": ctypes.c_int, "int32_t": ctypes.c_int, "uint32_t": ctypes.c_uint32,
            "float": ctypes.c_float, "size_t": ctypes.c_size_t}[base]


def test_binding_signatures_match_the_header():
    """Every prototype's return type and parameter types (pointer, int64, int, uint32, float) equal the
    ctypes signature the binding installs, so no argument is passed with the wrong width."""
    src = re.sub(r"/\*.*?\*/", "", open(HDR).read(), flags=re.S)
    src = "\n".join(ln for ln in src.splitlines() if not ln.lstrip().startswith("#"))
    protos = re.findall(r"([A-Za-z_][\w\s\*]*?)\b(nvfp4_\w+)\s*\(([^)]*)\)\s*;", src)
    assert len(protos) == len(_declared())
    for ret, name, params in protos:
        ret = ret.strip().splitlines()[-1]      # the return type sits on the prototype's first line
        res, args = nv._SIGS[name]
        want_ret = ctypes.c_char_p if "char" in ret else _ctype_of(ret.strip() + " r")
        assert res is want_ret, name
        ps = [p.strip() for p in params.split(",")] if params.strip() not in ("", "void") else []
        assert [_ctype_of(p) for p in ps] == list(args), name
