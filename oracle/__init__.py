"""CPU oracle for rotated scalar quantization and the QJL sketch.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference leg may import this package.  The
product library (``kv_quantization_b200``) never imports it, and it never
imports the product library.

The arithmetic lives in ``rq_oracle.c`` (plain single-threaded C, built with
``-O2 -ffp-contract=off``, no fast-math); this module only compiles it and
marshals numpy arrays through ctypes.  Each wrapper names the C function it
calls; the C file cites the page passage each function follows.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

F16, BF16 = 0, 1
PACKED, INT8 = 0, 1


def build(force: bool = False) -> str:
    """Compile rq_oracle.c into liboracle.so next to it (gcc, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _ptr(a, ctype):
    return a.ctypes.data_as(C.POINTER(ctype)) if a is not None else None


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = C.CDLL(build())
            u8, u16, i8, f32, f64 = (C.POINTER(C.c_uint8), C.POINTER(C.c_uint16), C.POINTER(C.c_int8),
                                     C.POINTER(C.c_float), C.POINTER(C.c_double))
            i64, i32, u64 = C.c_int64, C.c_int, C.c_uint64
            sig = {
                "orc_lloyd_max": (i32, [i32, f64]),
                "orc_table_mse": (C.c_double, [i32, f64]),
                "orc_splitmix64": (u64, [u64, u64]),
                "orc_sign_diagonal": (None, [u64, i32, i8]),
                "orc_gauss": (C.c_double, [u64, u64]),
                "orc_projection": (None, [u64, i32, i32, i32, u16]),
                "orc_boundaries": (None, [f32, i32, f32]),
                "orc_quantize": (i32, [u16, i32, i64, i32, i32, i32, i8, f32, u8, u16, f32, f32]),
                "orc_rotate_f64": (i32, [u16, i32, i64, i32, i8, f64]),
                "orc_dequantize": (i32, [u8, u16, i64, i32, i32, i32, i8, f32, i32, u16, f32]),
                "orc_dequantize_f64": (i32, [u8, u16, i64, i32, i32, i32, i8, f32, f64]),
                "orc_residual": (i32, [u16, i32, u8, u16, i64, i32, i32, i32, i8, f32, u16, u16]),
                "orc_vec_norms": (i32, [u16, i32, i64, i32, u16]),
                "orc_sketch": (i32, [u16, i32, i64, i32, i32, u16, u8, f64]),
                "orc_score": (i32, [u16, i64, i32, i32, i32, u16, i32, u8, u16, i64,
                                    u8, u16, i32, i32, i8, f32, f64]),
                "orc_attention": (i32, [u16, i64, i32, i32, i32, u16, i32, u8, u16, i64,
                                        u8, u16, i32, i32, i8, f32,
                                        u8, u16, i32, i32, i8, f32, C.c_double, f64]),
                "orc_sub_blocks": (i32, [i32, C.POINTER(C.c_int), C.POINTER(C.c_int)]),
                "orc_unpack_codes": (None, [u8, i64, i32, i32, i32, u8]),
                "orc_pack_codes": (None, [u8, i64, i32, i32, i32, u8]),
                "orc_hadamard_matrix": (None, [i32, f64]),
                "orc_fwht_f32": (None, [f32, i64, i32]),
                "orc_fwht_f64": (None, [f64, i64, i32]),
                "orc_pairwise_sum": (C.c_float, [f32, i32]),
                "orc_f32_to_bf16": (C.c_uint16, [C.c_float]),
                "orc_f32_to_f16": (C.c_uint16, [C.c_float]),
                "orc_f16_to_f32": (C.c_float, [C.c_uint16]),
                "orc_bf16_to_f32": (C.c_float, [C.c_uint16]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


# ---------------------------------------------------------------- helpers

def _u16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def _signs_arr(signs):
    return None if signs is None else np.ascontiguousarray(signs, dtype=np.int8)


def code_bytes_per_block(d: int, bits: int, layout: int) -> int:
    return d if layout == INT8 else d * bits // 8


# ---------------------------------------------------------------- API

def lloyd_max(bits: int) -> np.ndarray:
    """orc_lloyd_max: float64 Lloyd-Max N(0,1) centroids, ascending."""
    c = np.zeros(1 << bits, np.float64)
    lib().orc_lloyd_max(bits, _ptr(c, C.c_double))
    return c


def table_mse(c: np.ndarray) -> float:
    c = np.ascontiguousarray(c, np.float64)
    return lib().orc_table_mse(len(c), _ptr(c, C.c_double))


def splitmix64(seed: int, k: int) -> int:
    return lib().orc_splitmix64(seed, k)


def sign_diagonal(seed: int, d: int) -> np.ndarray:
    s = np.zeros(d, np.int8)
    lib().orc_sign_diagonal(seed, d, _ptr(s, C.c_int8))
    return s


def gauss(seed: int, k: int) -> float:
    return lib().orc_gauss(seed, k)


def projection(seed: int, m: int, d: int, dtype: int = BF16) -> np.ndarray:
    """orc_projection: m x d JL matrix as 16-bit patterns (bf16 or fp16)."""
    S = np.zeros((m, d), np.uint16)
    lib().orc_projection(seed, m, d, dtype, _ptr(S, C.c_uint16))
    return S


def boundaries(c32: np.ndarray) -> np.ndarray:
    c32 = np.ascontiguousarray(c32, np.float32)
    t = np.zeros(len(c32) - 1, np.float32)
    lib().orc_boundaries(_ptr(c32, C.c_float), len(c32), _ptr(t, C.c_float))
    return t


def quantize(x16, dtype, d, bits, layout, signs, c32, want_y=False):
    """orc_quantize -> (codes uint8, norms uint16 fp16 bits, y fp32 | None, n32 fp32)."""
    x16 = _u16(x16).reshape(-1)
    nb = x16.size // d
    c32 = np.ascontiguousarray(c32, np.float32)
    codes = np.zeros(nb * code_bytes_per_block(d, bits, layout), np.uint8)
    norms = np.zeros(nb, np.uint16)
    y = np.zeros(nb * d, np.float32) if want_y else None
    n32 = np.zeros(nb, np.float32)
    s = _signs_arr(signs)
    lib().orc_quantize(_ptr(x16, C.c_uint16), dtype, nb, d, bits, layout, _ptr(s, C.c_int8),
                       _ptr(c32, C.c_float), _ptr(codes, C.c_uint8), _ptr(norms, C.c_uint16),
                       _ptr(y, C.c_float), _ptr(n32, C.c_float))
    return codes, norms, y, n32


def rotate_f64(x16, dtype, d, signs):
    x16 = _u16(x16).reshape(-1)
    y = np.zeros(x16.size, np.float64)
    s = _signs_arr(signs)
    lib().orc_rotate_f64(_ptr(x16, C.c_uint16), dtype, x16.size // d, d, _ptr(s, C.c_int8), _ptr(y, C.c_double))
    return y


def dequantize(codes, norms, d, bits, layout, signs, c32, out_dtype, want_f32=False):
    """orc_dequantize -> (out 16-bit patterns, fp32 reconstruction | None)."""
    codes = np.ascontiguousarray(codes, np.uint8)
    norms = _u16(norms)
    nb = norms.size
    c32 = np.ascontiguousarray(c32, np.float32)
    out = np.zeros(nb * d, np.uint16)
    xh = np.zeros(nb * d, np.float32) if want_f32 else None
    s = _signs_arr(signs)
    lib().orc_dequantize(_ptr(codes, C.c_uint8), _ptr(norms, C.c_uint16), nb, d, bits, layout,
                         _ptr(s, C.c_int8), _ptr(c32, C.c_float), out_dtype, _ptr(out, C.c_uint16),
                         _ptr(xh, C.c_float))
    return out, xh


def dequantize_f64(codes, norms, d, bits, layout, signs, c32):
    codes = np.ascontiguousarray(codes, np.uint8)
    norms = _u16(norms)
    c32 = np.ascontiguousarray(c32, np.float32)
    out = np.zeros(norms.size * d, np.float64)
    s = _signs_arr(signs)
    lib().orc_dequantize_f64(_ptr(codes, C.c_uint8), _ptr(norms, C.c_uint16), norms.size, d, bits, layout,
                             _ptr(s, C.c_int8), _ptr(c32, C.c_float), _ptr(out, C.c_double))
    return out


def residual(x16, dtype, codes, norms, d, bits, layout, signs, c32):
    """orc_residual -> (r as bf16 patterns, fp16 residual norms)."""
    x16 = _u16(x16).reshape(-1)
    codes = np.ascontiguousarray(codes, np.uint8)
    norms = _u16(norms)
    c32 = np.ascontiguousarray(c32, np.float32)
    r = np.zeros(x16.size, np.uint16)
    rn = np.zeros(norms.size, np.uint16)
    s = _signs_arr(signs)
    lib().orc_residual(_ptr(x16, C.c_uint16), dtype, _ptr(codes, C.c_uint8), _ptr(norms, C.c_uint16),
                       norms.size, d, bits, layout, _ptr(s, C.c_int8), _ptr(c32, C.c_float),
                       _ptr(r, C.c_uint16), _ptr(rn, C.c_uint16))
    return r, rn


def vec_norms(v16, dtype, d):
    v16 = _u16(v16).reshape(-1)
    n = np.zeros(v16.size // d, np.uint16)
    lib().orc_vec_norms(_ptr(v16, C.c_uint16), dtype, v16.size // d, d, _ptr(n, C.c_uint16))
    return n


def sketch(v16, dtype, d, m, S16, want_p=False):
    """orc_sketch -> (packed sign bytes [n][m/8], P/||v|| fp64 | None)."""
    v16 = _u16(v16).reshape(-1)
    S16 = _u16(S16).reshape(-1)
    n = v16.size // d
    signs = np.zeros(n * (m // 8), np.uint8)
    p = np.zeros(n * m, np.float64) if want_p else None
    lib().orc_sketch(_ptr(v16, C.c_uint16), dtype, n, d, m, _ptr(S16, C.c_uint16),
                     _ptr(signs, C.c_uint8), _ptr(p, C.c_double))
    return signs, p


def score(q16, G, nq, d, m, S16, sdtype, signs, sk_norms, T, codes=None, norms=None, bits=0,
          layout=PACKED, signs_diag=None, c32=None):
    """orc_score -> fp64 scores [G][nq][T]."""
    q16 = _u16(q16).reshape(-1)
    S16 = _u16(S16).reshape(-1)
    signs = np.ascontiguousarray(signs, np.uint8)
    sk_norms = _u16(sk_norms)
    out = np.zeros(G * nq * T, np.float64)
    cd = None if codes is None else np.ascontiguousarray(codes, np.uint8)
    nr = None if norms is None else _u16(norms)
    cc = None if c32 is None else np.ascontiguousarray(c32, np.float32)
    s = _signs_arr(signs_diag)
    lib().orc_score(_ptr(q16, C.c_uint16), G, nq, d, m, _ptr(S16, C.c_uint16), sdtype,
                    _ptr(signs, C.c_uint8), _ptr(sk_norms, C.c_uint16), T,
                    _ptr(cd, C.c_uint8), _ptr(nr, C.c_uint16), bits, layout,
                    _ptr(s, C.c_int8), _ptr(cc, C.c_float), _ptr(out, C.c_double))
    return out.reshape(G, nq, T)


def attention(q16, G, nq, d, m, S16, sdtype, signs, sk_norms, T, vcodes, vnorms, vbits, vlayout, vsigns_diag,
              vc32, softmax_scale, codes=None, norms=None, bits=0, layout=PACKED, signs_diag=None, c32=None):
    """orc_attention -> fp64 [G][nq][d]: softmax(scale * score) over the T
    keys of each group, applied to the fp64 reconstructions of the values."""
    q16 = _u16(q16).reshape(-1)
    S16 = _u16(S16).reshape(-1)
    signs = np.ascontiguousarray(signs, np.uint8)
    sk_norms = _u16(sk_norms)
    cd = None if codes is None else np.ascontiguousarray(codes, np.uint8)
    nr = None if norms is None else _u16(norms)
    cc = None if c32 is None else np.ascontiguousarray(c32, np.float32)
    s = _signs_arr(signs_diag)
    vcd = np.ascontiguousarray(vcodes, np.uint8)
    vnr = _u16(vnorms)
    vcc = np.ascontiguousarray(vc32, np.float32)
    vs = _signs_arr(vsigns_diag)
    out = np.zeros(G * nq * d, np.float64)
    rc = lib().orc_attention(_ptr(q16, C.c_uint16), G, nq, d, m, _ptr(S16, C.c_uint16), sdtype,
                             _ptr(signs, C.c_uint8), _ptr(sk_norms, C.c_uint16), T,
                             _ptr(cd, C.c_uint8), _ptr(nr, C.c_uint16), bits, layout,
                             _ptr(s, C.c_int8), _ptr(cc, C.c_float),
                             _ptr(vcd, C.c_uint8), _ptr(vnr, C.c_uint16), vbits, vlayout,
                             _ptr(vs, C.c_int8), _ptr(vcc, C.c_float), float(softmax_scale),
                             _ptr(out, C.c_double))
    if rc != 0:
        raise ValueError("orc_attention: empty key range")
    return out.reshape(G, nq, d)


def sub_blocks(d):
    """orc_sub_blocks -> [(offset, size), ...]: the power-of-two sub-blocks of a
    block of d values, largest first."""
    off = (C.c_int * 31)()
    sz = (C.c_int * 31)()
    n = lib().orc_sub_blocks(d, off, sz)
    return [(off[i], sz[i]) for i in range(n)]


def unpack_codes(codes, nblocks, d, bits, layout):
    codes = np.ascontiguousarray(codes, np.uint8)
    out = np.zeros(nblocks * d, np.uint8)
    lib().orc_unpack_codes(_ptr(codes, C.c_uint8), nblocks, d, bits, layout, _ptr(out, C.c_uint8))
    return out


def pack_codes(idx, d, bits, layout):
    idx = np.ascontiguousarray(idx, np.uint8).reshape(-1)
    nb = idx.size // d
    out = np.zeros(nb * code_bytes_per_block(d, bits, layout), np.uint8)
    lib().orc_pack_codes(_ptr(idx, C.c_uint8), nb, d, bits, layout, _ptr(out, C.c_uint8))
    return out


def hadamard_matrix(d):
    H = np.zeros((d, d), np.float64)
    lib().orc_hadamard_matrix(d, _ptr(H, C.c_double))
    return H


def fwht_f32(v):
    v = np.ascontiguousarray(v, np.float32).copy()
    d = v.shape[-1]
    lib().orc_fwht_f32(_ptr(v, C.c_float), v.size // d, d)
    return v


def fwht_f64(v):
    v = np.ascontiguousarray(v, np.float64).copy()
    d = v.shape[-1]
    lib().orc_fwht_f64(_ptr(v, C.c_double), v.size // d, d)
    return v


def pairwise_sum(v):
    v = np.ascontiguousarray(v, np.float32)
    return lib().orc_pairwise_sum(_ptr(v, C.c_float), v.size)


def f32_to_bf16(x: float) -> int:
    return lib().orc_f32_to_bf16(x)


def f32_to_f16(x: float) -> int:
    return lib().orc_f32_to_f16(x)


def f16_to_f32(h: int) -> float:
    return lib().orc_f16_to_f32(h)


def bf16_to_f32(h: int) -> float:
    return lib().orc_bf16_to_f32(h)


def f32_table(bits: int) -> np.ndarray:
    """Lloyd-Max table rounded to fp32, the form both sides consume."""
    return lloyd_max(bits).astype(np.float32)
