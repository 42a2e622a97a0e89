"""Host-side checks of librq: the library loads, exports every entry point of
include/rq.h, rejects bad arguments before touching the GPU, and its host
tables (Lloyd-Max levels, storage sizes) agree with the oracle and the pages."""
import os
import re
import subprocess

import numpy as np
import pytest

import oracle as O
import kv_quantization_b200 as rq
from kv_quantization_b200 import _lib as L
from tests.conftest import ROOT, read_golden

HEADER = os.path.join(ROOT, "include", "rq.h")


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:[\w\s\*]+?)\b(\w+)\s*\(", src, flags=re.M)) - {"if"})


def test_header_and_binding_agree():
    names = header_functions()
    assert names == sorted(L.exported_symbols()), names


def test_library_exports_every_header_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in header_functions():
        assert name in exported, name
    L.lib()  # loads


def test_status_strings():
    assert L.status_string(0) == "RQ_OK"
    for s in (-1, -2, -3, -4, -5):
        assert L.status_string(s).startswith("RQ_E")


@pytest.mark.parametrize("bits", range(1, 9))
def test_library_lloyd_max_equals_oracle(bits):
    got = L.rq_lloyd_max(bits)
    want = O.f32_table(bits)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_code_bytes():
    assert L.rq_code_bytes(131072, 128, 4, L.RQ_CODES_INT8) == 131072
    assert L.rq_code_bytes(4096 * 4096, 128, 3, L.RQ_CODES_PACKED) == 4096 * 4096 * 3 // 8
    assert L.rq_code_bytes(4096 * 4096, 128, 5, L.RQ_CODES_PACKED) == 4096 * 4096 * 5 // 8
    assert L.rq_code_bytes(100, 128, 4, L.RQ_CODES_PACKED) == -1
    assert L.rq_code_bytes(128, 96, 4, L.RQ_CODES_PACKED) == -1          # n not a multiple of d
    assert L.rq_code_bytes(96 * 5, 96, 4, L.RQ_CODES_PACKED) == 96 * 5 // 2  # block-diagonal size
    assert L.rq_code_bytes(100 * 4, 100, 4, L.RQ_CODES_PACKED) == -1     # not a multiple of 32


def test_k_side_ratio_from_library_layout():
    """Per-token bytes of a QJL key = m/8 sign bytes + one fp16 norm; the
    ratio against bf16 keys reproduces the README's 7.53x / 14.22x / 3.88x."""
    for hd, m, ratio in read_golden("qjl_k_side_ratio.txt"):
        hd, m = int(hd), int(m)
        per_token = m // 8 + np.dtype(np.float16).itemsize
        assert round(hd * 2 / per_token, 2) == float(ratio)


class FakeTensor:
    """Stand-in device buffer: validation must fail before any dereference."""

    def __init__(self, ptr, numel=1 << 20, dtype=None):
        import torch
        self._ptr, self._n = ptr, numel
        self.dtype = dtype or torch.bfloat16

    def data_ptr(self):
        return self._ptr

    def numel(self):
        return self._n

    def element_size(self):
        return 2


def _q(x, d=128, bits=4, layout=L.RQ_CODES_PACKED, cent=None, codes=None, norms=None, n=None):
    cent = O.f32_table(bits) if cent is None else cent
    codes = codes or FakeTensor(0x10000)
    norms = norms or FakeTensor(0x20000)
    L.rq_quantize(x, d, bits, layout, 1, 7, cent, codes, norms, stream=0, n=n)


@pytest.mark.parametrize("case, status", [
    (dict(d=100), -1), (dict(d=1024), -4), (dict(bits=9), -1), (dict(bits=0), -1), (dict(n=1000), -1),
    (dict(layout=5), -1), (dict(cent=np.array([0.0, 0.0] + [1.0] * 14, np.float32)), -1),
    (dict(cent=np.array([np.nan] * 16, np.float32)), -1),
])
def test_quantize_rejects_bad_arguments(case, status):
    with pytest.raises(L.RQError) as e:
        _q(FakeTensor(0x30000), **case)
    assert e.value.status == status


def test_quantize_rejects_null_and_misaligned():
    with pytest.raises(L.RQError) as e:
        _q(FakeTensor(0))
    assert e.value.status == -1
    with pytest.raises(L.RQError) as e:
        _q(FakeTensor(0x30008))
    assert e.value.status == -2


def test_zero_length_is_a_noop():
    _q(FakeTensor(0), n=0)    # nothing enqueued, nothing dereferenced


def test_qjl_rejects_bad_m():
    for m in (0, 4, 12, 520):
        with pytest.raises(L.RQError) as e:
            L.qjl_sketch(FakeTensor(0x40000), 128, m, FakeTensor(0x50000), FakeTensor(0x60000), FakeTensor(0x70000),
                         stream=0)
        assert e.value.status == -1
    with pytest.raises(L.RQError):
        L.qjl_make_projection(1, 256, 100, FakeTensor(0x50000), stream=0)


def test_score_workspace_size_and_check():
    assert L.qjl_score_workspace_bytes(8, 32, 256, 256) >= 8 * 32 * 512 * 4
    small = FakeTensor(0x90000, numel=16)
    with pytest.raises(L.RQError) as e:
        L.qjl_score(FakeTensor(0x40000), 8, 32, 256, 256, FakeTensor(0x50000), FakeTensor(0x60000),
                    FakeTensor(0x70000), 1000, FakeTensor(0x80000), small, stream=0)
    assert e.value.status == -3


def test_table_cache_miss_and_hit_paths():
    """Valid calls build (miss) and then reuse (hit) the per-call tables; with
    no GPU visible the call stops right after, at the device query."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is visible: the call would launch")
    for bits in (3, 4, 3, 4, 2, 5, 6, 7, 1, 8, 3):          # more configurations than cache slots
        with pytest.raises(L.RQError) as e:
            _q(FakeTensor(0x30000), bits=bits)
        assert e.value.status == -5


def test_probe_and_trace_validate_before_any_launch():
    """rq_probe_bounded_wait rejects a poll limit out of range without a GPU;
    a call that fails validation leaves the launch trace empty."""
    for polls in (0, (1 << 20) + 1):
        assert L.lib().rq_probe_bounded_wait(polls, None) == -1
        assert L.rq_last_launch() == ""
    assert L.lib().rq_quantize(None, 1, 128, 100, 4, 0, 0, 0, None, None, None, None) == -1
    assert L.rq_last_launch() == ""


def test_attention_validates_before_any_launch():
    """qjl_attention rejects shapes it does not take (RQ_EUNSUPPORTED), an
    empty key range and a bad scale (RQ_EINVAL), and an undersized workspace
    (RQ_ESIZE, or the device query without a GPU), all before any launch."""
    import torch
    vc = L.rq_lloyd_max(4)

    def call(nq=32, d=128, m=256, T=1000, scale=0.1, ws_numel=1 << 30, kw=None):
        return L.qjl_attention(FakeTensor(0x40000), 4, nq, d, m, FakeTensor(0x50000), FakeTensor(0x60000),
                               FakeTensor(0x70000), T, FakeTensor(0x80000), FakeTensor(0x90000), 4, vc,
                               FakeTensor(0xa0000), FakeTensor(0xb0000, numel=ws_numel), scale, stream=0,
                               **(kw or {}))
    for args, status in (((dict(nq=33),), -4), ((dict(d=64),), -4), ((dict(m=136),), -4),
                         ((dict(T=0),), -1), ((dict(scale=float("nan")),), -1), ((dict(scale=-1.0),), -1)):
        with pytest.raises(L.RQError) as e:
            call(**args[0])
        assert e.value.status == status, (args, e.value.status)
        assert L.rq_last_launch() == ""
    if not torch.cuda.is_available():
        with pytest.raises(L.RQError) as e:
            call(ws_numel=4)
        assert e.value.status == -5                           # stops at the device query


def test_block_diagonal_sizes_take_no_residual_sketch():
    """Blocks of a non-power-of-two size quantize and dequantize, but the fused
    residual sketch takes power-of-two blocks only: RQ_EUNSUPPORTED before any
    launch."""
    c = O.f32_table(3)
    with pytest.raises(L.RQError) as e:
        L.rq_quantize_qjl(FakeTensor(0x40000), 96, 3, L.RQ_CODES_PACKED, 1, 5, c, 128, FakeTensor(0x50000),
                          FakeTensor(0x60000), FakeTensor(0x70000), FakeTensor(0x80000), FakeTensor(0x90000),
                          stream=0, n=96 * 64)
    assert e.value.status == -4
    assert L.rq_last_launch() == ""


# ---------------------------------------------------------------- dense rotation (host tables)

@pytest.mark.parametrize("d,bits", [(3, 2), (16, 1), (128, 2), (128, 4), (512, 3)])
def test_beta_lloyd_max_matches_the_oracle(d, bits):
    from oracle import dense_rotation as D
    got = rq.rq_beta_lloyd_max(d, bits).astype(np.float64)
    want = D.beta_lloyd_max(d, bits)
    np.testing.assert_allclose(got, want.astype(np.float32).astype(np.float64), rtol=2e-7, atol=1e-9)
    assert np.all(got[1:] > got[:-1]) and np.array_equal(got, -got[::-1])


@pytest.mark.parametrize("d", [8, 64, 128])
def test_make_rotation_matches_the_oracle(d):
    from oracle import dense_rotation as D
    got = rq.rq_make_rotation(d, 21).astype(np.float64)
    np.testing.assert_allclose(got, D.rotation(21, d), atol=2e-7)


def test_dense_entry_points_validate_before_launch():
    import torch
    x = torch.zeros(256, dtype=torch.bfloat16)
    pi = torch.zeros(128, 128, dtype=torch.bfloat16)
    codes = torch.zeros(128, dtype=torch.uint8)
    norms = torch.zeros(2, dtype=torch.int16)
    c = rq.rq_beta_lloyd_max(128, 4)
    for d, want in ((64, "RQ_EUNSUPPORTED"), (100, "RQ_EUNSUPPORTED"), (0, "RQ_EINVAL")):
        with pytest.raises(rq.RQError, match=want):
            rq.rq_quantize_dense(x, d, pi, 4, rq.RQ_CODES_PACKED, c, codes, norms, stream=0)
    with pytest.raises(rq.RQError, match="RQ_EINVAL"):
        rq.rq_quantize_dense(x, 128, pi, 4, rq.RQ_CODES_PACKED, c, codes, norms, n=200, stream=0)
    with pytest.raises(rq.RQError, match="RQ_EINVAL"):
        rq.rq_dequantize_dense(codes, norms, 256, 128, pi, 9, rq.RQ_CODES_PACKED, c, x, stream=0)
    assert L.rq_last_launch() == ""
    with pytest.raises(rq.RQError, match="RQ_EINVAL"):
        rq.rq_beta_lloyd_max(2, 4)


def test_outlier_entry_points_validate_before_launch():
    import torch
    k = torch.zeros(64 * 128, dtype=torch.bfloat16)
    S = torch.zeros(256, 128, dtype=torch.bfloat16)
    b = torch.zeros(4096, dtype=torch.uint8)
    n = torch.zeros(64, dtype=torch.int16)
    ws = torch.zeros(64 * 128 * 2, dtype=torch.uint8)
    assert rq.qjl_sketch_outlier_workspace_bytes(64, 128) == 64 * 128 * 2
    for kw, want in ((dict(d=256), "RQ_EUNSUPPORTED"), (dict(d=100), "RQ_EINVAL"), (dict(n_out=0), "RQ_EINVAL"),
                     (dict(n_out=17), "RQ_EINVAL"), (dict(m_o=48), "RQ_EINVAL"), (dict(m_o=512), "RQ_EINVAL"),
                     (dict(n_vec=48), "RQ_EINVAL")):
        a = dict(d=128, m=256, m_o=128, n_out=8, n_vec=64)
        a.update(kw)
        with pytest.raises(rq.RQError, match=want):
            rq.qjl_sketch_outlier(k, a["d"], a["m"], S, a["m_o"], a["n_out"], b, n, b, b, n, ws, stream=0,
                                  n_vec=a["n_vec"])
    with pytest.raises(rq.RQError, match="RQ_ESIZE"):
        rq.qjl_sketch_outlier(k, 128, 256, S, 128, 8, b, n, b, b, n, ws[:100], stream=0)
    with pytest.raises(rq.RQError, match="RQ_EINVAL"):      # T not a multiple of the group
        rq.qjl_score_outlier(k, 1, 4, 128, 256, S, b, n, 48, 128, 8, b, b, n, torch.zeros(1), ws, stream=0)
    assert L.rq_last_launch() == ""
