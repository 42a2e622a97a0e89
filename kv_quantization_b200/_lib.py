"""ctypes binding of librq (include/rq.h), argument marshalling only.

Every function here has the name of the C entry point it calls and forwards
its arguments unchanged: device buffers are torch CUDA tensors (passed by
data pointer), ``centroids`` is a host float32 array, ``stream`` defaults to
torch's current CUDA stream.  All arithmetic runs in librq's kernels; a
missing or unloadable librq.so raises immediately -- there is no fallback.
"""
from __future__ import annotations

import ctypes as C
import os
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librq.so")

RQ_F16, RQ_BF16 = 0, 1
RQ_CODES_PACKED, RQ_CODES_INT8 = 0, 1

_lock = threading.Lock()
_lib = None


class RQError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")
        self.status = status


def lib() -> C.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"librq.so not built ({LIB_PATH}); run python -m kv_quantization_b200.build")
            L = C.CDLL(LIB_PATH)
            vp, i64, i32, u64, sz = C.c_void_p, C.c_int64, C.c_int, C.c_uint64, C.c_size_t
            fp = C.POINTER(C.c_float)
            sig = {
                "rq_status_string": (C.c_char_p, [i32]),
                "rq_code_bytes": (i64, [i64, i32, i32, i32]),
                "rq_device_error": (i32, [i32]),
                "rq_last_launch": (C.c_char_p, []),
                "rq_probe_bounded_wait": (i32, [C.c_uint32, vp]),
                "rq_lloyd_max": (i32, [i32, fp]),
                "rq_quantize": (i32, [vp, i32, i64, i32, i32, i32, i32, u64, fp, vp, vp, vp]),
                "rq_dequantize": (i32, [vp, vp, i64, i32, i32, i32, i32, u64, fp, vp, i32, vp]),
                "rq_quantize_qjl": (i32, [vp, i32, i64, i32, i32, i32, i32, u64, fp, i32, vp, vp, vp, vp, vp, vp]),
                "qjl_make_projection": (i32, [u64, i32, i32, i32, vp, vp]),
                "qjl_sketch": (i32, [vp, i32, i64, i32, i32, vp, vp, vp, vp]),
                "qjl_score_workspace_bytes": (sz, [i64, i32, i32, i32]),
                "qjl_score": (i32, [vp, i64, i32, i32, i32, vp, i32, vp, vp, i64, vp, vp, i32, i32, i32, u64,
                                    fp, vp, vp, sz, vp]),
                "qjl_attention_workspace_bytes": (sz, [i64, i32, i32, i32, i64]),
                "qjl_attention": (i32, [vp, i64, i32, i32, i32, vp, i32, vp, vp, i64, vp, vp, i32, i32, i32, u64,
                                        vp, vp, vp, i32, i32, i32, u64, vp, C.c_float, vp, vp, sz, vp]),
                "qjl_score_noalloc": (i32, [vp, i64, i32, i32, i32, vp, i32, vp, vp, i64, vp, vp, i32, i32, i32,
                                            u64, fp, vp, vp]),
                "qjl_sketch_outlier_workspace_bytes": (sz, [i64, i32]),
                "qjl_sketch_outlier": (i32, [vp, i64, i32, i32, vp, i32, i32, vp, vp, vp, vp, vp, vp, sz, vp]),
                "qjl_score_outlier": (i32, [vp, i64, i32, i32, i32, vp, vp, vp, i64, i32, i32, vp, vp, vp, vp, vp, sz,
                                            vp]),
                "rq_beta_lloyd_max": (i32, [i32, i32, fp]),
                "rq_make_rotation": (i32, [i32, u64, fp]),
                "rq_quantize_dense": (i32, [vp, i32, i64, i32, vp, i32, i32, fp, vp, vp, vp]),
                "rq_dequantize_dense": (i32, [vp, vp, i64, i32, vp, i32, i32, fp, vp, i32, vp]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def exported_symbols():
    """Names this binding expects librq.so to export."""
    return ["rq_status_string", "rq_device_error", "rq_last_launch", "rq_probe_bounded_wait", "rq_code_bytes", "rq_lloyd_max", "rq_quantize", "rq_dequantize",
            "rq_quantize_qjl", "qjl_make_projection", "qjl_sketch", "qjl_score_workspace_bytes", "qjl_score",
            "qjl_score_noalloc", "qjl_attention_workspace_bytes", "qjl_attention", "rq_beta_lloyd_max",
            "rq_make_rotation", "rq_quantize_dense", "rq_dequantize_dense", "qjl_sketch_outlier_workspace_bytes",
            "qjl_sketch_outlier", "qjl_score_outlier"]


def status_string(status: int) -> str:
    return lib().rq_status_string(int(status)).decode()


def _check(fn, status):
    if status != 0:
        raise RQError(fn, status)


def _dev(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _table(centroids):
    c = np.ascontiguousarray(np.asarray(centroids, dtype=np.float32))
    return c, c.ctypes.data_as(C.POINTER(C.c_float))


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return RQ_BF16
    if t.dtype == torch.float16:
        return RQ_F16
    raise TypeError(f"expected a bfloat16 or float16 tensor, got {t.dtype}")


# ------------------------------------------------------------------ entry points

def rq_code_bytes(n: int, d: int, bits: int, layout: int) -> int:
    return lib().rq_code_bytes(n, d, bits, layout)


def rq_device_error(clear: bool = True) -> int:
    """RQ_OK, or RQ_EDEVICE when a kernel gave up a bounded wait since the last clear."""
    return lib().rq_device_error(int(clear))


def rq_last_launch() -> str:
    """Kernels enqueued by this thread's last librq call, comma-separated."""
    return lib().rq_last_launch().decode()


def rq_probe_bounded_wait(polls: int, stream=None):
    _check("rq_probe_bounded_wait", lib().rq_probe_bounded_wait(int(polls), _stream(stream)))


def rq_lloyd_max(bits: int) -> np.ndarray:
    out = np.zeros(1 << bits, np.float32)
    _check("rq_lloyd_max", lib().rq_lloyd_max(bits, out.ctypes.data_as(C.POINTER(C.c_float))))
    return out


def rq_quantize(x, d, bits, layout, use_signs, sign_seed, centroids, codes, norms, stream=None, n=None):
    c, cp = _table(centroids)
    _check("rq_quantize", lib().rq_quantize(_dev(x), _dtype_code(x), x.numel() if n is None else n, d, bits, layout,
                                            int(use_signs), sign_seed, cp, _dev(codes), _dev(norms), _stream(stream)))


def rq_dequantize(codes, norms, n, d, bits, layout, use_signs, sign_seed, centroids, out, stream=None):
    c, cp = _table(centroids)
    _check("rq_dequantize", lib().rq_dequantize(_dev(codes), _dev(norms), n, d, bits, layout, int(use_signs),
                                                sign_seed, cp, _dev(out), _dtype_code(out), _stream(stream)))


def qjl_sketch_outlier_workspace_bytes(n_vec: int, d: int) -> int:
    return lib().qjl_sketch_outlier_workspace_bytes(n_vec, d)


def qjl_sketch_outlier(keys, d, m, proj, m_o, n_out, signs, norms, out_idx, out_signs, out_norms, workspace,
                       stream=None, n_vec=None):
    nv = keys.numel() // d if n_vec is None else n_vec
    _check("qjl_sketch_outlier", lib().qjl_sketch_outlier(
        _dev(keys), nv, d, m, _dev(proj), m_o, n_out, _dev(signs), _dev(norms), _dev(out_idx), _dev(out_signs),
        _dev(out_norms), _dev(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def qjl_score_outlier(q, G, n_q, d, m, proj, signs, norms, T, m_o, n_out, out_idx, out_signs, out_norms, scores,
                      workspace, stream=None):
    _check("qjl_score_outlier", lib().qjl_score_outlier(
        _dev(q), G, n_q, d, m, _dev(proj), _dev(signs), _dev(norms), T, m_o, n_out, _dev(out_idx), _dev(out_signs),
        _dev(out_norms), _dev(scores), _dev(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))


def rq_beta_lloyd_max(d: int, bits: int) -> np.ndarray:
    """Lloyd-Max centroids (fp32, ascending) of one coordinate of a uniform unit vector in R^d."""
    out = np.zeros(1 << bits, np.float32)
    _check("rq_beta_lloyd_max", lib().rq_beta_lloyd_max(d, bits, out.ctypes.data_as(C.POINTER(C.c_float))))
    return out


def rq_make_rotation(d: int, seed: int) -> np.ndarray:
    """The seeded random orthogonal matrix Pi (d x d, fp32, row-major)."""
    out = np.zeros((d, d), np.float32)
    _check("rq_make_rotation", lib().rq_make_rotation(d, seed, out.ctypes.data_as(C.POINTER(C.c_float))))
    return out


def rq_quantize_dense(x, d, pi, bits, layout, centroids, codes, norms, stream=None, n=None):
    c, cp = _table(centroids)
    _check("rq_quantize_dense", lib().rq_quantize_dense(_dev(x), _dtype_code(x), x.numel() if n is None else n, d,
                                                        _dev(pi), bits, layout, cp, _dev(codes), _dev(norms),
                                                        _stream(stream)))


def rq_dequantize_dense(codes, norms, n, d, pi, bits, layout, centroids, out, stream=None):
    c, cp = _table(centroids)
    _check("rq_dequantize_dense", lib().rq_dequantize_dense(_dev(codes), _dev(norms), n, d, _dev(pi), bits, layout,
                                                            cp, _dev(out), _dtype_code(out), _stream(stream)))


def rq_quantize_qjl(x, d, bits, layout, use_signs, sign_seed, centroids, m, proj, codes, norms, qjl_signs,
                    qjl_norms, stream=None, n=None):
    c, cp = _table(centroids)
    _check("rq_quantize_qjl", lib().rq_quantize_qjl(
        _dev(x), _dtype_code(x), x.numel() if n is None else n, d, bits, layout, int(use_signs), sign_seed, cp,
        m, _dev(proj), _dev(codes), _dev(norms), _dev(qjl_signs), _dev(qjl_norms), _stream(stream)))


def qjl_make_projection(seed, m, d, proj, stream=None):
    _check("qjl_make_projection", lib().qjl_make_projection(seed, m, d, _dtype_code(proj), _dev(proj),
                                                            _stream(stream)))


def qjl_sketch(x, d, m, proj, signs, norms, stream=None, n_vec=None):
    nv = x.numel() // d if n_vec is None else n_vec
    _check("qjl_sketch", lib().qjl_sketch(_dev(x), _dtype_code(x), nv, d, m, _dev(proj), _dev(signs), _dev(norms),
                                          _stream(stream)))


def qjl_score_workspace_bytes(G, n_q, d, m) -> int:
    return lib().qjl_score_workspace_bytes(G, n_q, d, m)


def qjl_score(q, G, n_q, d, m, proj, signs, sk_norms, T, scores, workspace, codes=None, norms=None, bits=0,
              layout=RQ_CODES_PACKED, use_signs=0, sign_seed=0, centroids=None, stream=None):
    if centroids is None:
        cp = None
    else:
        c, cp = _table(centroids)
    _check("qjl_score", lib().qjl_score(
        _dev(q), G, n_q, d, m, _dev(proj), _dtype_code(proj), _dev(signs), _dev(sk_norms), T, _dev(codes),
        _dev(norms), bits, layout, int(use_signs), sign_seed, cp, _dev(scores), _dev(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def qjl_attention_workspace_bytes(G, n_q, d, m, T) -> int:
    return lib().qjl_attention_workspace_bytes(G, n_q, d, m, T)


def qjl_attention(q, G, n_q, d, m, proj, signs, sk_norms, T, v_codes, v_norms, v_bits, v_centroids, out, workspace,
                  softmax_scale, codes=None, norms=None, bits=0, layout=RQ_CODES_PACKED, use_signs=0, sign_seed=0,
                  centroids=None, v_layout=RQ_CODES_PACKED, v_use_signs=0, v_sign_seed=0, stream=None):
    """Softmax(softmax_scale * score) over the T compressed keys of each group,
    applied to the in-kernel reconstructions of the compressed values:
    out fp32 [G][n_q][d]."""
    cp = None
    if centroids is not None:
        c, cp = _table(centroids)
    vc, vcp = _table(v_centroids)
    _check("qjl_attention", lib().qjl_attention(
        _dev(q), G, n_q, d, m, _dev(proj), _dtype_code(proj), _dev(signs), _dev(sk_norms), T, _dev(codes),
        _dev(norms), bits, layout, int(use_signs), sign_seed, cp, _dev(v_codes), _dev(v_norms), v_bits, v_layout,
        int(v_use_signs), v_sign_seed, vcp, float(softmax_scale), _dev(out), _dev(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def qjl_score_noalloc(q, G, n_q, d, m, proj, signs, sk_norms, T, scores, codes=None, norms=None, bits=0,
                      layout=RQ_CODES_PACKED, use_signs=0, sign_seed=0, centroids=None, stream=None):
    """qjl_score with the library's own fixed 8 MiB device scratch instead of a
    caller workspace, for callers that cannot allocate device memory."""
    if centroids is None:
        cp = None
    else:
        c, cp = _table(centroids)
    _check("qjl_score_noalloc", lib().qjl_score_noalloc(
        _dev(q), G, n_q, d, m, _dev(proj), _dtype_code(proj), _dev(signs), _dev(sk_norms), T, _dev(codes),
        _dev(norms), bits, layout, int(use_signs), sign_seed, cp, _dev(scores), _stream(stream)))
