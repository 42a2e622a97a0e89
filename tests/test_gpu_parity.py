"""GPU parity: librq (through its C ABI) against the CPU oracle.

Bars (from the arithmetic each side follows):
  * codes, norms, reconstructions, residual norms, the projection matrix:
    bit-exact (both sides compute in the same canonical fp32 order); any code
    mismatch must also sit within 1e-5 of a decision boundary and their count
    stay below 1e-6 of the elements;
  * sign bits: bit-exact except where |P_i| / ||v|| <= 1e-5 (the GPU
    accumulates in fp32, the oracle in fp64), count below 1e-6 of the bits
    (at these sizes: zero);
  * scores: |gpu - oracle| <= 1e-3 * ||q|| * (n16 + rn16) -- the error scale
    of a dot product of that size (the oracle is fp64 from the same inputs;
    the GPU rounds intermediates to fp32).
Inputs are the seeded recipes of kv_quantization_b200.synth at sizes the
oracle finishes in seconds, spanning several tiles with a ragged tail, plus
sampled checks at the full workload sizes.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from kv_quantization_b200 import _lib as L
from kv_quantization_b200 import synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(autouse=True)
def no_device_timeouts():
    """Every kernel's bounded waits completed (no RQ_EDEVICE recorded)."""
    yield
    torch.cuda.synchronize()
    assert L.rq_device_error(True) == 0


def u16(t):
    return synth.as_u16(t).reshape(-1)


def dt_code(dtype):
    return O.BF16 if dtype == torch.bfloat16 else O.F16


def run_quant(x, d, bits, layout, use_signs, seed, cent):
    n = x.numel()
    codes = torch.empty(L.rq_code_bytes(n, d, bits, layout), dtype=torch.uint8, device=DEV)
    norms = torch.empty(n // d, dtype=torch.int16, device=DEV)
    L.rq_quantize(x, d, bits, layout, use_signs, seed, cent, codes, norms)
    return codes, norms


def check_codes(g_codes, o_codes, x16, dtype, d, bits, layout, signs, cent):
    """Bit-exact codes, or mismatches confined to the 1e-5 boundary window."""
    if np.array_equal(g_codes, o_codes):
        return 0
    nb = x16.size // d
    gi = O.unpack_codes(g_codes, nb, d, bits, layout)
    oi = O.unpack_codes(o_codes, nb, d, bits, layout)
    bad = np.nonzero(gi != oi)[0]
    y64 = O.rotate_f64(x16, dtype, d, signs)
    t = O.boundaries(cent).astype(np.float64)
    near = np.min(np.abs(y64[bad][:, None] - t[None, :]), axis=1) <= 1e-5
    assert near.all(), f"{(~near).sum()} code mismatches outside the boundary window"
    assert bad.size < 1e-6 * x16.size, f"{bad.size} windowed mismatches"
    return bad.size


def check_signs(g, o, p_rel, n, m):
    if np.array_equal(g, o):
        return 0
    gb = np.unpackbits(g.reshape(n, m // 8), axis=1, bitorder="little")
    ob = np.unpackbits(o.reshape(n, m // 8), axis=1, bitorder="little")
    bad = np.nonzero((gb != ob).reshape(-1))[0]
    assert np.all(np.abs(p_rel[bad]) <= 1e-5), "sign mismatch outside the window"
    assert bad.size < max(1.0, 1e-6 * n * m), f"{bad.size} windowed sign mismatches"
    return bad.size


# ------------------------------------------------------------------ quantize / dequantize

def test_fp16_int8_256x512_full():
    """256 x 512 fp16 N(0, 0.02^2) seed 0, d = 128, 4-bit int8 codes, no signs."""
    x = synth.gaussian_matrix(256, 512, 0.02, seed=0, dtype=torch.float16, device=DEV)
    cent = L.rq_lloyd_max(4)
    codes, norms = run_quant(x, 128, 4, L.RQ_CODES_INT8, 0, 0, cent)
    out = torch.empty_like(x)
    L.rq_dequantize(codes, norms, x.numel(), 128, 4, L.RQ_CODES_INT8, 0, 0, cent, out)
    torch.cuda.synchronize()
    x16 = u16(x)
    oc, on, _, _ = O.quantize(x16, O.F16, 128, 4, O.INT8, None, cent)
    check_codes(codes.cpu().numpy(), oc, x16, O.F16, 128, 4, O.INT8, None, cent)
    assert np.array_equal(norms.cpu().numpy().view(np.uint16), on)
    oo, _ = O.dequantize(oc, on, 128, 4, O.INT8, None, cent, O.F16)
    assert np.array_equal(u16(out), oo)


CASES = [
    # d, bits, layout, dtype, signs
    (128, 4, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (128, 3, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (128, 5, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (128, 2, L.RQ_CODES_PACKED, torch.float16, 0),
    (128, 1, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (128, 8, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (128, 4, L.RQ_CODES_INT8, torch.float16, 1),
    (128, 6, L.RQ_CODES_PACKED, torch.bfloat16, 0),
    (64, 4, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (64, 3, L.RQ_CODES_INT8, torch.float16, 1),
    (256, 2, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (256, 6, L.RQ_CODES_INT8, torch.float16, 1),
    (512, 2, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (512, 7, L.RQ_CODES_PACKED, torch.float16, 0),
]


@pytest.mark.parametrize("d,bits,layout,dtype,signs", CASES)
def test_quant_dequant_parity(d, bits, layout, dtype, signs):
    nblocks = 3 * 128 + 7                                     # several tiles, ragged tail
    x = synth.student_t_outliers(1, nblocks * d, seed=100 + d + bits, dtype=dtype, device=DEV).reshape(-1)
    cent = L.rq_lloyd_max(bits)
    codes, norms = run_quant(x, d, bits, layout, signs, 1234 + bits, cent)
    out = torch.empty_like(x)
    L.rq_dequantize(codes, norms, x.numel(), d, bits, layout, signs, 1234 + bits, cent, out)
    torch.cuda.synchronize()
    x16 = u16(x)
    s = O.sign_diagonal(1234 + bits, d) if signs else None
    oc, on, _, _ = O.quantize(x16, dt_code(dtype), d, bits, layout, s, cent)
    nmis = check_codes(codes.cpu().numpy(), oc, x16, dt_code(dtype), d, bits, layout, s, cent)
    assert np.array_equal(norms.cpu().numpy().view(np.uint16), on)
    # dequantize parity on the oracle's codes (isolated from any code mismatch)
    oo, xh32 = O.dequantize(oc, on, d, bits, layout, s, cent, dt_code(dtype), want_f32=True)
    if nmis == 0:
        assert np.array_equal(u16(out), oo)
    out2 = torch.empty_like(x)
    L.rq_dequantize(torch.from_numpy(oc).to(DEV), torch.from_numpy(on.view(np.int16)).to(DEV), x.numel(), d, bits,
                    layout, signs, 1234 + bits, cent, out2)
    torch.cuda.synchronize()
    assert np.array_equal(u16(out2), oo)
    # reconstruction against the fp64 value: max abs error <= 1e-3 * block norm
    # (+ half an output ulp, the rounding the output dtype itself imposes)
    x64 = O.dequantize_f64(oc, on, d, bits, layout, s, cent)
    got = out2.float().cpu().numpy().astype(np.float64)
    nrm = np.repeat([O.f16_to_f32(int(h)) for h in on], d)
    ulp = np.abs(x64) * (2.0 ** -8 if dtype == torch.bfloat16 else 2.0 ** -11)
    assert np.all(np.abs(got - x64) <= 1e-3 * nrm + ulp + 1e-30)


def test_binary_search_fallback_table():
    """A table whose thresholds no 128-cell grid separates (two levels 1e-6
    apart) takes the binary-search path; codes still match exactly."""
    cent = L.rq_lloyd_max(4).copy()
    cent[8] = cent[7] + 1e-6
    x = synth.gaussian_matrix(64, 1024, 1.0, seed=5, dtype=torch.bfloat16, device=DEV)
    codes, norms = run_quant(x, 128, 4, L.RQ_CODES_PACKED, 1, 9, cent)
    torch.cuda.synchronize()
    x16 = u16(x)
    oc, on, _, _ = O.quantize(x16, O.BF16, 128, 4, O.PACKED, O.sign_diagonal(9, 128), cent)
    check_codes(codes.cpu().numpy(), oc, x16, O.BF16, 128, 4, O.PACKED, O.sign_diagonal(9, 128), cent)
    assert np.array_equal(norms.cpu().numpy().view(np.uint16), on)


def test_zero_and_tiny_blocks():
    x = torch.zeros(5 * 128, dtype=torch.bfloat16, device=DEV)
    x[128:256] = 1e-39            # squares underflow: n32 = 0, y = 0
    x[256] = 3.0                  # one-hot block
    cent = L.rq_lloyd_max(3)
    codes, norms = run_quant(x, 128, 3, L.RQ_CODES_PACKED, 1, 3, cent)
    out = torch.empty_like(x)
    L.rq_dequantize(codes, norms, x.numel(), 128, 3, L.RQ_CODES_PACKED, 1, 3, cent, out)
    torch.cuda.synchronize()
    x16 = u16(x)
    s = O.sign_diagonal(3, 128)
    oc, on, _, _ = O.quantize(x16, O.BF16, 128, 3, O.PACKED, s, cent)
    assert np.array_equal(codes.cpu().numpy(), oc)
    assert np.array_equal(norms.cpu().numpy().view(np.uint16), on)
    oo, _ = O.dequantize(oc, on, 128, 3, O.PACKED, s, cent, O.BF16)
    assert np.array_equal(u16(out), oo)


def test_weight_4096x4096_sampled_full_size():
    """4096 x 4096 bf16 Student-t with outliers at full size, bits 3/4/5, signs
    seed 1: 1500 sampled blocks against the oracle."""
    x = synth.student_t_outliers(4096, 4096, seed=1, device=DEV).reshape(-1)
    rng = np.random.default_rng(0)
    blocks = np.sort(rng.choice(x.numel() // 128, 1500, replace=False))
    xs = u16(x.view(-1, 128)[torch.from_numpy(blocks).to(DEV)])
    s = O.sign_diagonal(1, 128)
    for bits in (3, 4, 5):
        cent = L.rq_lloyd_max(bits)
        codes, norms = run_quant(x, 128, bits, L.RQ_CODES_PACKED, 1, 1, cent)
        out = torch.empty_like(x)
        L.rq_dequantize(codes, norms, x.numel(), 128, bits, L.RQ_CODES_PACKED, 1, 1, cent, out)
        torch.cuda.synchronize()
        cb = 128 * bits // 8
        gc = codes.view(-1, cb)[torch.from_numpy(blocks).to(DEV)].cpu().numpy().reshape(-1)
        oc, on, _, _ = O.quantize(xs, O.BF16, 128, bits, O.PACKED, s, cent)
        check_codes(gc, oc, xs, O.BF16, 128, bits, O.PACKED, s, cent)
        assert np.array_equal(norms.cpu().numpy().view(np.uint16)[blocks], on)
        oo, _ = O.dequantize(oc, on, 128, bits, O.PACKED, s, cent, O.BF16)
        assert np.array_equal(u16(out.view(-1, 128)[torch.from_numpy(blocks).to(DEV)]), oo)


LLAMA7B_LINEARS = [(4096, 4096)] * 4 + [(11008, 4096)] * 2 + [(4096, 11008)]   # q, k, v, o, gate, up, down


def test_llama7b_32_layers_one_call_sampled():
    """All linears of 32 Llama-7B-shaped layers (6.48e9 bf16 values, 50.6M
    blocks, 13 GB) quantized (4-bit, d = 128, seeded signs) and dequantized
    with one call each -- the largest input of the workloads -- and 2048
    blocks sampled over every layer and matrix checked against the oracle."""
    sizes = [r * c for r, c in LLAMA7B_LINEARS] * 32
    n = sum(sizes)
    x = torch.empty(n, dtype=torch.bfloat16, device=DEV)
    off = 0
    for i, (r, c) in enumerate(LLAMA7B_LINEARS * 32):
        x[off:off + r * c] = synth.llama_linear(r, c, seed=1000 + i, device=DEV).reshape(-1)
        off += r * c
    bits, seed = 4, 11
    cent = L.rq_lloyd_max(bits)
    codes, norms = run_quant(x, 128, bits, L.RQ_CODES_PACKED, 1, seed, cent)
    out = torch.empty_like(x)
    L.rq_dequantize(codes, norms, n, 128, bits, L.RQ_CODES_PACKED, 1, seed, cent, out)
    torch.cuda.synchronize()
    rng = np.random.default_rng(3)
    nb = n // 128
    blocks = np.unique(np.concatenate([rng.choice(nb, 2040, replace=False), [0, 1, nb - 2, nb - 1]]))
    idx = torch.from_numpy(blocks).to(DEV)
    xs = u16(x.view(-1, 128)[idx])
    s = O.sign_diagonal(seed, 128)
    gc = codes.view(-1, 64)[idx].cpu().numpy().reshape(-1)
    oc, on, _, _ = O.quantize(xs, O.BF16, 128, bits, O.PACKED, s, cent)
    check_codes(gc, oc, xs, O.BF16, 128, bits, O.PACKED, s, cent)
    assert np.array_equal(norms.view(torch.int16).cpu().numpy().view(np.uint16)[blocks], on)
    oo, _ = O.dequantize(oc, on, 128, bits, O.PACKED, s, cent, O.BF16)
    assert np.array_equal(u16(out.view(-1, 128)[idx]), oo)
    del x, out, codes, norms
    torch.cuda.empty_cache()


# ------------------------------------------------------------------ QJL

@pytest.mark.parametrize("m,d,dtype", [(128, 128, torch.bfloat16), (256, 128, torch.bfloat16),
                                       (256, 256, torch.float16), (512, 512, torch.bfloat16), (40, 64, torch.bfloat16)])
def test_projection_bit_exact(m, d, dtype):
    S = torch.empty(m, d, dtype=dtype, device=DEV)
    L.qjl_make_projection(77 + m, m, d, S)
    torch.cuda.synchronize()
    assert np.array_equal(u16(S), O.projection(77 + m, m, d, dt_code(dtype)).reshape(-1))


@pytest.mark.parametrize("d,m", [(128, 256), (128, 128), (256, 256), (512, 512), (64, 40)])
def test_sketch_keys(d, m):
    n = 2 * 301
    k = synth.kv_with_channels(1, 2, 301, d, seed=3, device=DEV).reshape(-1)
    S = torch.empty(m, d, dtype=torch.bfloat16, device=DEV)
    L.qjl_make_projection(3, m, d, S)
    signs = torch.empty(n * m // 8, dtype=torch.uint8, device=DEV)
    norms = torch.empty(n, dtype=torch.int16, device=DEV)
    L.qjl_sketch(k, d, m, S, signs, norms)
    torch.cuda.synchronize()
    k16 = u16(k)
    os_, p = O.sketch(k16, O.BF16, d, m, u16(S), want_p=True)
    check_signs(signs.cpu().numpy(), os_, p, n, m)
    assert np.array_equal(norms.cpu().numpy().view(np.uint16), O.vec_norms(k16, O.BF16, d))


QJL_CASES = [
    # d, bits, m, layout, dtype, signs
    (128, 4, 128, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (128, 3, 128, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (128, 5, 128, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (128, 1, 256, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (128, 2, 40, L.RQ_CODES_PACKED, torch.float16, 0),
    (128, 6, 64, L.RQ_CODES_INT8, torch.float16, 1),
    (256, 2, 256, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (256, 4, 72, L.RQ_CODES_PACKED, torch.float16, 1),
    (256, 3, 128, L.RQ_CODES_INT8, torch.bfloat16, 0),
    (512, 2, 512, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (512, 3, 72, L.RQ_CODES_PACKED, torch.float16, 0),
    (512, 4, 264, L.RQ_CODES_PACKED, torch.bfloat16, 1),
]


@pytest.mark.parametrize("d,bits,m,layout,dtype,signs", QJL_CASES)
def test_quantize_qjl_residual(d, bits, m, layout, dtype, signs):
    nblocks = 2 * 128 + 11
    x = synth.student_t_outliers(1, nblocks * d, seed=7 + d + m, dtype=dtype, device=DEV).reshape(-1)
    cent = L.rq_lloyd_max(bits)
    S = torch.empty(m, d, dtype=torch.bfloat16, device=DEV)
    L.qjl_make_projection(2, m, d, S)
    codes = torch.empty(L.rq_code_bytes(x.numel(), d, bits, layout), dtype=torch.uint8, device=DEV)
    norms = torch.empty(nblocks, dtype=torch.int16, device=DEV)
    qs = torch.empty(nblocks * m // 8, dtype=torch.uint8, device=DEV)
    qn = torch.empty(nblocks, dtype=torch.int16, device=DEV)
    L.rq_quantize_qjl(x, d, bits, layout, signs, 1, cent, m, S, codes, norms, qs, qn)
    torch.cuda.synchronize()
    x16 = u16(x)
    dt = dt_code(dtype)
    s = O.sign_diagonal(1, d) if signs else None
    oc, on, _, _ = O.quantize(x16, dt, d, bits, layout, s, cent)
    check_codes(codes.cpu().numpy(), oc, x16, dt, d, bits, layout, s, cent)
    assert np.array_equal(norms.cpu().numpy().view(np.uint16), on)
    r_bf, rn = O.residual(x16, dt, oc, on, d, bits, layout, s, cent)
    assert np.array_equal(qn.cpu().numpy().view(np.uint16), rn)
    osg, p = O.sketch(r_bf, O.BF16, d, m, u16(S), want_p=True)
    check_signs(qs.cpu().numpy(), osg, p, nblocks, m)


def _score_tol(q16, G, nq, d, sk_norms, norms=None):
    qf = (q16.astype(np.uint32) << 16).view(np.float32).astype(np.float64).reshape(G, nq, d)
    qn = np.linalg.norm(qf, axis=2)[:, :, None]
    kn = np.array([O.f16_to_f32(int(h)) for h in sk_norms.reshape(-1)]).reshape(G, 1, -1)
    if norms is not None:
        kn = kn + np.array([O.f16_to_f32(int(h)) for h in norms.reshape(-1)]).reshape(G, 1, -1)
    return 1e-3 * qn * kn


def test_score_pure_qjl():
    G, nq, T, d, m = 3, 32, 333, 128, 256
    k = synth.kv_with_channels(1, G, T, d, seed=4, device=DEV).reshape(-1)
    q = synth.normal((G, nq, d), seed=5, device=DEV)
    S = torch.empty(m, d, dtype=torch.bfloat16, device=DEV)
    L.qjl_make_projection(3, m, d, S)
    signs = torch.empty(G * T * m // 8, dtype=torch.uint8, device=DEV)
    kn = torch.empty(G * T, dtype=torch.int16, device=DEV)
    L.qjl_sketch(k, d, m, S, signs, kn)
    scores = torch.empty(G, nq, T, dtype=torch.float32, device=DEV)
    ws = torch.empty(L.qjl_score_workspace_bytes(G, nq, d, m) // 4, dtype=torch.float32, device=DEV)
    L.qjl_score(q, G, nq, d, m, S, signs, kn, T, scores, ws)
    torch.cuda.synchronize()
    q16 = u16(q)
    want = O.score(q16, G, nq, d, m, u16(S), O.BF16, signs.cpu().numpy(), kn.cpu().numpy().view(np.uint16), T)
    err = np.abs(scores.cpu().numpy().astype(np.float64) - want)
    assert np.all(err <= _score_tol(q16, G, nq, d, kn.cpu().numpy().view(np.uint16)))


def test_score_fp16_projection_ragged_queries():
    """Pure QJL score with the projection given in fp16 (the same matrix as the
    bf16 one the keys were sketched with, widened exactly) and 33 queries, so
    the query projection reads fp16 S and the second 32-query group is ragged."""
    G, nq, T, d, m = 2, 33, 200, 128, 128
    k = synth.kv_with_channels(1, G, T, d, seed=21, device=DEV).reshape(-1)
    q = synth.normal((G, nq, d), seed=22, device=DEV)
    S = torch.empty(m, d, dtype=torch.bfloat16, device=DEV)
    L.qjl_make_projection(12, m, d, S)
    signs = torch.empty(G * T * m // 8, dtype=torch.uint8, device=DEV)
    kn = torch.empty(G * T, dtype=torch.int16, device=DEV)
    L.qjl_sketch(k, d, m, S, signs, kn)
    S16 = S.to(torch.float16)
    scores = torch.empty(G, nq, T, dtype=torch.float32, device=DEV)
    ws = torch.empty(L.qjl_score_workspace_bytes(G, nq, d, m) // 4, dtype=torch.float32, device=DEV)
    L.qjl_score(q, G, nq, d, m, S16, signs, kn, T, scores, ws)
    torch.cuda.synchronize()
    q16 = u16(q)
    want = O.score(q16, G, nq, d, m, u16(S16), O.F16, signs.cpu().numpy(), kn.cpu().numpy().view(np.uint16), T)
    err = np.abs(scores.cpu().numpy().astype(np.float64) - want)
    assert np.all(err <= _score_tol(q16, G, nq, d, kn.cpu().numpy().view(np.uint16)))


@pytest.mark.parametrize("d", [256, 512])
def test_score_two_stage(d):
    """2-bit rotated Lloyd-Max keys + QJL (m = d) residual sketch, 32 queries."""
    G, nq, T, m, bits = 2, 32, 257, d, 2
    k = synth.normal((G, T, d), seed=6, device=DEV).reshape(-1)
    q = synth.normal((G, nq, d), seed=7, device=DEV)
    cent = L.rq_lloyd_max(bits)
    S = torch.empty(m, d, dtype=torch.bfloat16, device=DEV)
    L.qjl_make_projection(5, m, d, S)
    codes = torch.empty(L.rq_code_bytes(k.numel(), d, bits, L.RQ_CODES_PACKED), dtype=torch.uint8, device=DEV)
    norms = torch.empty(G * T, dtype=torch.int16, device=DEV)
    qs = torch.empty(G * T * m // 8, dtype=torch.uint8, device=DEV)
    qn = torch.empty(G * T, dtype=torch.int16, device=DEV)
    L.rq_quantize_qjl(k, d, bits, L.RQ_CODES_PACKED, 1, 4, cent, m, S, codes, norms, qs, qn)
    scores = torch.empty(G, nq, T, dtype=torch.float32, device=DEV)
    ws = torch.empty(L.qjl_score_workspace_bytes(G, nq, d, m) // 4, dtype=torch.float32, device=DEV)
    L.qjl_score(q, G, nq, d, m, S, qs, qn, T, scores, ws, codes=codes, norms=norms, bits=bits,
                layout=L.RQ_CODES_PACKED, use_signs=1, sign_seed=4, centroids=cent)
    torch.cuda.synchronize()
    q16 = u16(q)
    s = O.sign_diagonal(4, d)
    want = O.score(q16, G, nq, d, m, u16(S), O.BF16, qs.cpu().numpy(), qn.cpu().numpy().view(np.uint16), T,
                   codes=codes.cpu().numpy(), norms=norms.cpu().numpy().view(np.uint16), bits=bits,
                   layout=O.PACKED, signs_diag=s, c32=cent)
    err = np.abs(scores.cpu().numpy().astype(np.float64) - want)
    tol = _score_tol(q16, G, nq, d, qn.cpu().numpy().view(np.uint16), norms.cpu().numpy().view(np.uint16))
    assert np.all(err <= tol), float((err / tol).max())


@pytest.mark.parametrize("d,bits,m,nq,layout", [(128, 4, 128, 40, L.RQ_CODES_INT8), (64, 3, 72, 7, L.RQ_CODES_PACKED),
                                                 (128, 5, 256, 33, L.RQ_CODES_PACKED)])
def test_score_two_stage_shapes(d, bits, m, nq, layout):
    """Query counts that are not multiples of 32, m not a multiple of 64,
    int8 codes, and a ragged token tail."""
    G, T = 3, 131
    k = synth.normal((G, T, d), seed=16, device=DEV).reshape(-1)
    q = synth.normal((G, nq, d), seed=17, device=DEV)
    cent = L.rq_lloyd_max(bits)
    S = torch.empty(m, d, dtype=torch.bfloat16, device=DEV)
    L.qjl_make_projection(8, m, d, S)
    codes = torch.empty(L.rq_code_bytes(k.numel(), d, bits, layout), dtype=torch.uint8, device=DEV)
    norms = torch.empty(G * T, dtype=torch.int16, device=DEV)
    qs = torch.empty(G * T * m // 8, dtype=torch.uint8, device=DEV)
    qn = torch.empty(G * T, dtype=torch.int16, device=DEV)
    L.rq_quantize_qjl(k, d, bits, layout, 1, 9, cent, m, S, codes, norms, qs, qn)
    scores = torch.empty(G, nq, T, dtype=torch.float32, device=DEV)
    ws = torch.empty(L.qjl_score_workspace_bytes(G, nq, d, m) // 4 + 1, dtype=torch.float32, device=DEV)
    L.qjl_score(q, G, nq, d, m, S, qs, qn, T, scores, ws, codes=codes, norms=norms, bits=bits, layout=layout,
                use_signs=1, sign_seed=9, centroids=cent)
    torch.cuda.synchronize()
    q16 = u16(q)
    want = O.score(q16, G, nq, d, m, u16(S), O.BF16, qs.cpu().numpy(), qn.cpu().numpy().view(np.uint16), T,
                   codes=codes.cpu().numpy(), norms=norms.cpu().numpy().view(np.uint16), bits=bits,
                   layout=layout, signs_diag=O.sign_diagonal(9, d), c32=cent)
    err = np.abs(scores.cpu().numpy().astype(np.float64) - want)
    tol = _score_tol(q16, G, nq, d, qn.cpu().numpy().view(np.uint16), norms.cpu().numpy().view(np.uint16))
    assert np.all(err <= tol), float((err / tol).max())
