"""GPU parity: librq (through its C ABI) against the CPU oracle, on inputs
the oracle finishes in seconds that still span several tiles with a ragged
tail (the bars are listed in tests/gpu_checks.py).  Every case also names the
kernel the dispatch must have chosen for it (rq_last_launch), so that each
kernel the library can launch is compared with the oracle somewhere.
"""
import numpy as np
import pytest
import torch

import oracle as O
from kv_quantization_b200 import _lib as L
from kv_quantization_b200 import synth
from tests.gpu_checks import (DEV, check_codes, check_scores, check_signs, dt_code, score_tol, u16)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def no_device_timeouts():
    """Every kernel's bounded waits completed (no RQ_EDEVICE recorded)."""
    yield
    torch.cuda.synchronize()
    assert L.rq_device_error(True) == 0


def run_quant(x, d, bits, layout, use_signs, seed, cent):
    n = x.numel()
    codes = torch.empty(L.rq_code_bytes(n, d, bits, layout), dtype=torch.uint8, device=DEV)
    norms = torch.empty(n // d, dtype=torch.int16, device=DEV)
    L.rq_quantize(x, d, bits, layout, use_signs, seed, cent, codes, norms)
    return codes, norms


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


def quant_kernels(d, bits, layout):
    """Kernels the dispatch picks for rq_quantize / rq_dequantize: the d = 128
    one-block-per-thread kernels when a saturating search grid of at most 128
    cells exists (the Lloyd-Max tables of 1-5 bits), the general-d kernels
    otherwise; 1-4-bit packed d = 128 codes take the pair-table dequantize."""
    q = "quantize_v5_kernel" if d == 128 and bits <= 5 else "quantize_v2_kernel"
    if d != 128:
        dq = "dequantize_v2_kernel"
    elif layout == L.RQ_CODES_PACKED and bits <= 4:
        dq = "dequantize_v5p_kernel"
    else:
        dq = "dequantize_v5_kernel"
    return q, dq


CASES = [
    # d, bits, layout, dtype, signs
    (128, 4, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (128, 3, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (128, 5, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (128, 2, L.RQ_CODES_PACKED, torch.float16, 0),
    (128, 1, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (128, 8, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (128, 7, L.RQ_CODES_INT8, torch.float16, 1),
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
    kq, kdq = quant_kernels(d, bits, layout)
    codes, norms = run_quant(x, d, bits, layout, signs, 1234 + bits, cent)
    assert L.rq_last_launch() == kq
    out = torch.empty_like(x)
    L.rq_dequantize(codes, norms, x.numel(), d, bits, layout, signs, 1234 + bits, cent, out)
    assert L.rq_last_launch() == kdq
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
    """A table whose thresholds no 128-cell grid separates (levels 6, 7, 8
    within 2e-6, so two decision thresholds lie 1e-6 apart) takes the
    branch-free binary search; codes still match exactly."""
    cent = L.rq_lloyd_max(4).copy()
    cent[7] = cent[6] + 1e-6
    cent[8] = cent[6] + 2e-6
    assert np.all(np.diff(cent) > 0)
    x = synth.gaussian_matrix(64, 1024, 1.0, seed=5, dtype=torch.bfloat16, device=DEV)
    codes, norms = run_quant(x, 128, 4, L.RQ_CODES_PACKED, 1, 9, cent)
    assert L.rq_last_launch() == "quantize_v2_kernel"
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
        # the reconstruction of the library's own codes (equal to the oracle's
        # except for windowed mismatches, which the check above bounds)
        oo, _ = O.dequantize(gc, on, 128, bits, O.PACKED, s, cent, O.BF16)
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
    assert L.rq_last_launch() == "projection_kernel"
    torch.cuda.synchronize()
    assert np.array_equal(u16(S), O.projection(77 + m, m, d, dt_code(dtype)).reshape(-1))


# Key sketch: d = 128 with m <= 256 takes the warp-specialised TMA kernel; the
# tensor-core fallback covers the shapes whose S and tile fit in shared memory;
# the CUDA-core kernel the rest.
SKETCH_CASES = [
    # d, m, kernel
    (128, 256, "sketch_v3_kernel"),
    (128, 128, "sketch_v3_kernel"),
    (128, 72, "sketch_v3_kernel"),
    (128, 512, "qjl_mma_kernel<sketch>"),
    (256, 256, "qjl_mma_kernel<sketch>"),
    (256, 264, "sketch_kernel"),
    (512, 32, "qjl_mma_kernel<sketch>"),
    (512, 512, "sketch_kernel"),
    (64, 40, "qjl_mma_kernel<sketch>"),
]


@pytest.mark.parametrize("d,m,kernel", SKETCH_CASES)
def test_sketch_keys(d, m, kernel):
    n = 2 * 301
    k = synth.kv_with_channels(1, 2, 301, d, seed=3, device=DEV).reshape(-1)
    S = torch.empty(m, d, dtype=torch.bfloat16, device=DEV)
    L.qjl_make_projection(3, m, d, S)
    signs = torch.empty(n * m // 8, dtype=torch.uint8, device=DEV)
    norms = torch.empty(n, dtype=torch.int16, device=DEV)
    L.qjl_sketch(k, d, m, S, signs, norms)
    assert L.rq_last_launch() == kernel
    torch.cuda.synchronize()
    k16 = u16(k)
    os_, p = O.sketch(k16, O.BF16, d, m, u16(S), want_p=True)
    check_signs(signs.cpu().numpy(), os_, p, n, m)
    assert np.array_equal(norms.cpu().numpy().view(np.uint16), O.vec_norms(k16, O.BF16, d))


# Fused quantize + residual sketch: one kernel per head dim when a saturating
# search grid exists (bits <= 5) and S's tiles fit; then the pipelined
# fallback for d = 128 / 256 (6-8-bit tables); then the unpipelined
# tensor-core kernel (any d whose S fits in shared memory); then CUDA cores.
QJL_CASES = [
    # d, bits, m, layout, dtype, signs, kernel
    (128, 4, 128, L.RQ_CODES_PACKED, torch.bfloat16, 1, "qjl_v6_quant_kernel"),
    (128, 3, 128, L.RQ_CODES_PACKED, torch.bfloat16, 1, "qjl_v6_quant_kernel"),
    (128, 5, 128, L.RQ_CODES_PACKED, torch.bfloat16, 1, "qjl_v6_quant_kernel"),
    (128, 1, 256, L.RQ_CODES_PACKED, torch.bfloat16, 1, "qjl_v6_quant_kernel"),
    (128, 2, 40, L.RQ_CODES_PACKED, torch.float16, 0, "qjl_v6_quant_kernel"),
    (128, 5, 64, L.RQ_CODES_INT8, torch.float16, 1, "qjl_v6_quant_kernel"),
    (128, 6, 64, L.RQ_CODES_INT8, torch.float16, 1, "qjl_v3_quant_kernel"),
    (256, 2, 256, L.RQ_CODES_PACKED, torch.bfloat16, 1, "qjl_v7_quant_kernel"),
    (256, 4, 72, L.RQ_CODES_PACKED, torch.float16, 1, "qjl_v7_quant_kernel"),
    (256, 3, 128, L.RQ_CODES_INT8, torch.bfloat16, 0, "qjl_v7_quant_kernel"),
    (512, 2, 512, L.RQ_CODES_PACKED, torch.bfloat16, 1, "qjl_v8_quant_kernel"),
    (512, 3, 72, L.RQ_CODES_PACKED, torch.float16, 0, "qjl_v8_quant_kernel"),
    (128, 7, 128, L.RQ_CODES_PACKED, torch.bfloat16, 1, "qjl_v3_quant_kernel"),
    (128, 8, 256, L.RQ_CODES_INT8, torch.float16, 0, "qjl_v3_quant_kernel"),
    (256, 8, 64, L.RQ_CODES_PACKED, torch.bfloat16, 1, "qjl_v3_quant_kernel"),
    (64, 3, 72, L.RQ_CODES_PACKED, torch.bfloat16, 1, "qjl_mma_kernel<fused>"),
    (64, 8, 128, L.RQ_CODES_INT8, torch.float16, 1, "qjl_mma_kernel<fused>"),
    (128, 4, 264, L.RQ_CODES_PACKED, torch.bfloat16, 1, "qjl_mma_kernel<fused>"),
    (512, 8, 16, L.RQ_CODES_PACKED, torch.bfloat16, 1, "qjl_mma_kernel<fused>"),
    (512, 4, 264, L.RQ_CODES_PACKED, torch.bfloat16, 1, "quantize_kernel"),
    (256, 2, 512, L.RQ_CODES_PACKED, torch.float16, 1, "quantize_kernel"),
]


def run_fused(x, d, bits, layout, signs, seed, cent, m, S):
    nblocks = x.numel() // d
    codes = torch.empty(L.rq_code_bytes(x.numel(), d, bits, layout), dtype=torch.uint8, device=DEV)
    norms = torch.empty(nblocks, dtype=torch.int16, device=DEV)
    qs = torch.empty(nblocks * m // 8, dtype=torch.uint8, device=DEV)
    qn = torch.empty(nblocks, dtype=torch.int16, device=DEV)
    L.rq_quantize_qjl(x, d, bits, layout, signs, seed, cent, m, S, codes, norms, qs, qn)
    return codes, norms, qs, qn


def check_fused(x16, dt, d, bits, layout, signs, seed, cent, m, S16, codes, norms, qs, qn, full_blocks=None):
    """Codes, norms, residual norms bit-exact; residual sign bits windowed."""
    nb = x16.size // d
    s = O.sign_diagonal(seed, d) if signs else None
    oc, on, _, _ = O.quantize(x16, dt, d, bits, layout, s, cent)
    check_codes(codes, oc, x16, dt, d, bits, layout, s, cent)
    assert np.array_equal(norms, on)
    r_bf, rn = O.residual(x16, dt, oc, on, d, bits, layout, s, cent)
    assert np.array_equal(qn, rn)
    osg, p = O.sketch(r_bf, O.BF16, d, m, S16, want_p=True)
    check_signs(qs, osg, p, nb, m, full_bits=None if full_blocks is None else full_blocks * m)


@pytest.mark.parametrize("d,bits,m,layout,dtype,signs,kernel", QJL_CASES)
def test_quantize_qjl_residual(d, bits, m, layout, dtype, signs, kernel):
    nblocks = 2 * 128 + 11
    x = synth.student_t_outliers(1, nblocks * d, seed=7 + d + m, dtype=dtype, device=DEV).reshape(-1)
    cent = L.rq_lloyd_max(bits)
    S = torch.empty(m, d, dtype=torch.bfloat16, device=DEV)
    L.qjl_make_projection(2, m, d, S)
    codes, norms, qs, qn = run_fused(x, d, bits, layout, signs, 1, cent, m, S)
    assert L.rq_last_launch() == kernel
    torch.cuda.synchronize()
    check_fused(u16(x), dt_code(dtype), d, bits, layout, signs, 1, cent, m, u16(S), codes.cpu().numpy(),
                norms.cpu().numpy().view(np.uint16), qs.cpu().numpy(), qn.cpu().numpy().view(np.uint16))


# ------------------------------------------------------------------ scores

def make_two_stage(G, T, d, bits, m, layout, seed, sseed, pseed):
    k = synth.normal((G, T, d), seed=seed, device=DEV).reshape(-1)
    cent = L.rq_lloyd_max(bits)
    S = torch.empty(m, d, dtype=torch.bfloat16, device=DEV)
    L.qjl_make_projection(pseed, m, d, S)
    codes, norms, qs, qn = run_fused(k, d, bits, layout, 1, sseed, cent, m, S)
    return k, cent, S, codes, norms, qs, qn


def score_kernels(nq, d=128, m=256, bits=0, layout=L.RQ_CODES_PACKED):
    """Kernels qjl_score launches: queries on M (score_v5) when n_q <= 128 and
    every token's sign bytes (and code bytes, for two-stage keys) are a
    multiple of 16; the 128-token tensor-core kernel (score_v4) for the other
    n_q <= 128 shapes; the CUDA-core score above 128 queries."""
    if nq > 128:
        return "score_prologue_kernel,score_kernel"
    pw = 8 if layout == L.RQ_CODES_INT8 else bits
    if (m // 8) % 16 == 0 and (bits == 0 or (d * pw // 8) % 16 == 0):
        return "score_v2_prologue,score_v5_kernel"
    return "score_v2_prologue,score_v4_kernel"


@pytest.mark.parametrize("nq", [32, 160])
def test_score_pure_qjl(nq):
    G, T, d, m = 3, 333, 128, 256
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
    assert L.rq_last_launch() == score_kernels(nq)
    torch.cuda.synchronize()
    q16 = u16(q)
    kn16 = kn.cpu().numpy().view(np.uint16)
    want = O.score(q16, G, nq, d, m, u16(S), O.BF16, signs.cpu().numpy(), kn16, T)
    check_scores(scores.cpu().numpy(), want, score_tol(q16, G, nq, d, kn16), f"pure d={d} m={m} nq={nq}")


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
    kn16 = kn.cpu().numpy().view(np.uint16)
    want = O.score(q16, G, nq, d, m, u16(S16), O.F16, signs.cpu().numpy(), kn16, T)
    check_scores(scores.cpu().numpy(), want, score_tol(q16, G, nq, d, kn16), "pure fp16 S nq=33")


@pytest.mark.parametrize("d", [256, 512])
def test_score_two_stage(d):
    """2-bit rotated Lloyd-Max keys + QJL (m = d) residual sketch, 32 queries."""
    G, nq, T, m, bits = 2, 32, 257, d, 2
    k, cent, S, codes, norms, qs, qn = make_two_stage(G, T, d, bits, m, L.RQ_CODES_PACKED, 6, 4, 5)
    q = synth.normal((G, nq, d), seed=7, device=DEV)
    scores = torch.empty(G, nq, T, dtype=torch.float32, device=DEV)
    ws = torch.empty(L.qjl_score_workspace_bytes(G, nq, d, m) // 4, dtype=torch.float32, device=DEV)
    L.qjl_score(q, G, nq, d, m, S, qs, qn, T, scores, ws, codes=codes, norms=norms, bits=bits,
                layout=L.RQ_CODES_PACKED, use_signs=1, sign_seed=4, centroids=cent)
    assert L.rq_last_launch() == score_kernels(nq, d, m, bits)
    torch.cuda.synchronize()
    q16 = u16(q)
    n16 = norms.cpu().numpy().view(np.uint16)
    want = O.score(q16, G, nq, d, m, u16(S), O.BF16, qs.cpu().numpy(), qn.cpu().numpy().view(np.uint16), T,
                   codes=codes.cpu().numpy(), norms=n16, bits=bits, layout=O.PACKED,
                   signs_diag=O.sign_diagonal(4, d), c32=cent)
    check_scores(scores.cpu().numpy(), want, score_tol(q16, G, nq, d, n16), f"two-stage d={d}")


@pytest.mark.parametrize("d,bits,m,nq,layout", [(128, 4, 128, 40, L.RQ_CODES_INT8), (64, 3, 72, 7, L.RQ_CODES_PACKED),
                                                 (128, 5, 256, 33, L.RQ_CODES_PACKED),
                                                 (128, 3, 128, 100, L.RQ_CODES_PACKED),
                                                 (64, 2, 128, 64, L.RQ_CODES_INT8),
                                                 (128, 4, 128, 136, L.RQ_CODES_PACKED),
                                                 (256, 2, 256, 129, L.RQ_CODES_PACKED)])
def test_score_two_stage_shapes(d, bits, m, nq, layout):
    """Query counts that are not multiples of 32 (and above 128: the CUDA-core
    score), m not a multiple of 64, int8 codes, and a ragged token tail."""
    G, T = 3, 131
    k, cent, S, codes, norms, qs, qn = make_two_stage(G, T, d, bits, m, layout, 16, 9, 8)
    q = synth.normal((G, nq, d), seed=17, device=DEV)
    scores = torch.empty(G, nq, T, dtype=torch.float32, device=DEV)
    ws = torch.empty(L.qjl_score_workspace_bytes(G, nq, d, m) // 4 + 1, dtype=torch.float32, device=DEV)
    L.qjl_score(q, G, nq, d, m, S, qs, qn, T, scores, ws, codes=codes, norms=norms, bits=bits, layout=layout,
                use_signs=1, sign_seed=9, centroids=cent)
    assert L.rq_last_launch() == score_kernels(nq, d, m, bits, layout)
    torch.cuda.synchronize()
    q16 = u16(q)
    n16 = norms.cpu().numpy().view(np.uint16)
    want = O.score(q16, G, nq, d, m, u16(S), O.BF16, qs.cpu().numpy(), qn.cpu().numpy().view(np.uint16), T,
                   codes=codes.cpu().numpy(), norms=n16, bits=bits, layout=layout,
                   signs_diag=O.sign_diagonal(9, d), c32=cent)
    check_scores(scores.cpu().numpy(), want, score_tol(q16, G, nq, d, n16), f"two-stage d={d} b={bits} nq={nq}")


@pytest.mark.parametrize("two,nq,T", [(False, 24, 1000), (True, 40, 2052), (False, 64, 516)])
def test_score_tma_store_shapes(two, nq, T):
    """T % 4 == 0 takes the score kernel's TMA-store epilogue: ragged last
    boxes (T not a multiple of 32) and query counts that end inside a
    16-row box are clipped by the tensor map, never written past a group."""
    G, d, bits = 3, 128, 2
    m = 128 if two else 256
    q = synth.normal((G, nq, d), seed=31, device=DEV)
    scores = torch.full((G, nq, T), float("nan"), dtype=torch.float32, device=DEV)
    ws = torch.empty(L.qjl_score_workspace_bytes(G, nq, d, m) // 4, dtype=torch.float32, device=DEV)
    q16 = u16(q)
    if two:
        k, cent, S, codes, norms, qs, qn = make_two_stage(G, T, d, bits, m, L.RQ_CODES_PACKED, 32, 33, 34)
        L.qjl_score(q, G, nq, d, m, S, qs, qn, T, scores, ws, codes=codes, norms=norms, bits=bits,
                    layout=L.RQ_CODES_PACKED, use_signs=1, sign_seed=33, centroids=cent)
        n16 = norms.cpu().numpy().view(np.uint16)
        want = O.score(q16, G, nq, d, m, u16(S), O.BF16, qs.cpu().numpy(), qn.cpu().numpy().view(np.uint16), T,
                       codes=codes.cpu().numpy(), norms=n16, bits=bits, layout=O.PACKED,
                       signs_diag=O.sign_diagonal(33, d), c32=cent)
        tol = score_tol(q16, G, nq, d, n16)
    else:
        k = synth.kv_with_channels(1, G, T, d, seed=35, device=DEV).reshape(-1)
        S = torch.empty(m, d, dtype=torch.bfloat16, device=DEV)
        L.qjl_make_projection(36, m, d, S)
        signs = torch.empty(G * T * m // 8, dtype=torch.uint8, device=DEV)
        kn = torch.empty(G * T, dtype=torch.int16, device=DEV)
        L.qjl_sketch(k, d, m, S, signs, kn)
        L.qjl_score(q, G, nq, d, m, S, signs, kn, T, scores, ws)
        kn16 = kn.cpu().numpy().view(np.uint16)
        want = O.score(q16, G, nq, d, m, u16(S), O.BF16, signs.cpu().numpy(), kn16, T)
        tol = score_tol(q16, G, nq, d, kn16)
    assert L.rq_last_launch() == "score_v2_prologue,score_v5_kernel"
    torch.cuda.synchronize()
    got = scores.cpu().numpy()
    assert not np.isnan(got).any()
    check_scores(got, want, tol, f"tma store two={two} nq={nq} T={T}")


BD_CASES = [
    # d, bits, layout, dtype, signs
    (96, 4, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (96, 3, L.RQ_CODES_PACKED, torch.float16, 0),
    (160, 2, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (192, 5, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (320, 8, L.RQ_CODES_INT8, torch.float16, 1),
    (448, 4, L.RQ_CODES_INT8, torch.bfloat16, 1),
    (480, 1, L.RQ_CODES_PACKED, torch.bfloat16, 1),
    (224, 7, L.RQ_CODES_PACKED, torch.float16, 1),
]


@pytest.mark.parametrize("d,bits,layout,dtype,signs", BD_CASES)
def test_block_diagonal_quant_dequant_parity(d, bits, layout, dtype, signs):
    """Blocks of a non-power-of-two size (block-diagonal transform): codes,
    norms and reconstructions bit-exact against the oracle, over enough blocks
    that every CTA's warps loop several times, with zero blocks mixed in."""
    nb = 8 * 148 * 6 + 37
    x = synth.kv_with_channels(1, 1, nb, d, seed=d + bits, device=DEV).reshape(-1).to(dtype)
    x[5 * d:6 * d] = 0
    cent = L.rq_lloyd_max(bits)
    codes = torch.empty(L.rq_code_bytes(x.numel(), d, bits, layout), dtype=torch.uint8, device=DEV)
    norms = torch.empty(nb, dtype=torch.int16, device=DEV)
    L.rq_quantize(x, d, bits, layout, signs, 17, cent, codes, norms)
    assert L.rq_last_launch() == "quantize_bd_kernel"
    out = torch.empty_like(x)
    L.rq_dequantize(codes, norms, x.numel(), d, bits, layout, signs, 17, cent, out)
    assert L.rq_last_launch() == "dequantize_bd_kernel"
    torch.cuda.synchronize()
    x16 = u16(x)
    s = O.sign_diagonal(17, d) if signs else None
    oc, on, _, _ = O.quantize(x16, dt_code(dtype), d, bits, O.INT8 if layout == L.RQ_CODES_INT8 else O.PACKED, s, cent)
    assert np.array_equal(norms.cpu().numpy().view(np.uint16), on)
    assert np.array_equal(codes.cpu().numpy(), oc)
    oo, _ = O.dequantize(oc, on, d, bits, O.INT8 if layout == L.RQ_CODES_INT8 else O.PACKED, s, cent, dt_code(dtype))
    assert np.array_equal(u16(out), oo)
