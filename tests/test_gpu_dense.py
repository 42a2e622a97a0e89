"""rq_quantize_dense / rq_dequantize_dense on the GPU against the dense-rotation
oracle (TurboQuant README, "Algorithm in one paragraph").

Bars (from the arithmetic: the rotation is a 16-bit tensor-core GEMM with
fp32 accumulation, the oracle sums the same 16-bit operands in fp64):
- norms: bit-exact (both take the canonical fp32 pairwise norm);
- codes: equal, except one level apart where the oracle's z lies within
  DELTA = 2^-15 of the boundary between the two levels.  |z| <= 1 and the
  fp32 accumulation of 128 exact products errs by at most 128 * 2^-23 *
  sum_i |Pi_ji x_i| / ||x|| <= 128 * 2^-23 = 2^-16 (Cauchy-Schwarz, rows of
  Pi of norm ~1), plus one rounding of the scale: 2^-15 covers both;
- reconstructions: within one unit in the last place of the output dtype at
  the oracle's value, plus n16 * 2^-15 for the fp32 accumulation.
"""
import numpy as np
import pytest
import torch

import oracle as O
from oracle import dense_rotation as D
from kv_quantization_b200 import _lib as L
from kv_quantization_b200 import synth
from tests.gpu_checks import DEV, dt_code, report, u16

pytestmark = pytest.mark.gpu

d = 128
DELTA = 2.0 ** -15
_PI = {}
_CB = {}


def rotation16(seed, dtype):
    key = (seed, dtype)
    if key not in _PI:
        _PI[key] = D.to16(D.rotation(seed, d), dt_code(dtype))
    return _PI[key]


def codebook(bits):
    if bits not in _CB:
        _CB[bits] = (D.beta_lloyd_max(d, bits) if bits <= 4 else O.lloyd_max(bits) / np.sqrt(d)).astype(np.float32)
    return _CB[bits]


def dev16(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16).copy()).to(DEV).view(dtype)


def check_dense_codes(g, o, z, c32, nb, bits, layout):
    gi = O.unpack_codes(g, nb, d, bits, layout).reshape(nb, d).astype(np.int64)
    oi = O.unpack_codes(o, nb, d, bits, layout).reshape(nb, d).astype(np.int64)
    bad = gi != oi
    if not bad.any():
        return 0
    assert np.all(np.abs(gi - oi)[bad] == 1), "codes differ by more than one level"
    t = D.boundaries32(c32).astype(np.float64)
    between = t[np.minimum(gi, oi)[bad]]                 # the boundary separating the two levels
    assert np.all(np.abs(z[bad] - between) <= DELTA), np.max(np.abs(z[bad] - between))
    assert bad.mean() < 0.01
    return int(bad.sum())


def ulp16(v, dtype):
    e = np.floor(np.log2(np.maximum(np.abs(v), 1e-30)))
    return np.exp2(e - (7 if dtype == torch.bfloat16 else 10))


def run_quantize(x, bits, layout, pi_dev, c32):
    nb = x.numel() // d
    codes = torch.empty(L.rq_code_bytes(x.numel(), d, bits, layout), dtype=torch.uint8, device=DEV)
    norms = torch.empty(nb, dtype=torch.int16, device=DEV)
    L.rq_quantize_dense(x, d, pi_dev, bits, layout, c32, codes, norms)
    torch.cuda.synchronize()
    assert "quantize_dense_kernel" in L.rq_last_launch()
    return codes.cpu().numpy(), norms.cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("bits,layout", [(2, L.RQ_CODES_PACKED), (3, L.RQ_CODES_PACKED), (4, L.RQ_CODES_PACKED),
                                         (4, L.RQ_CODES_INT8), (8, L.RQ_CODES_PACKED)])
def test_dense_quantize_matches_oracle(dtype, bits, layout):
    nb = 128 * 5 + 37                                   # several tiles and a ragged last tile
    x = synth.kv_with_channels(1, 1, nb, d, seed=bits + 7 * layout, dtype=dtype, device=DEV).reshape(-1)
    pi16 = rotation16(3, dtype)
    c32 = codebook(bits)
    g_codes, g_norms = run_quantize(x, bits, layout, dev16(pi16, dtype), c32)
    o_codes, o_norms, z, _ = D.quantize(u16(x), dt_code(dtype), d, pi16, bits, layout, c32)
    np.testing.assert_array_equal(g_norms, o_norms)
    nbad = check_dense_codes(g_codes, o_codes, z, c32, nb, bits, layout)
    report("dense_quantize", dtype=str(dtype), bits=bits, layout=layout, blocks=nb, boundary_codes=nbad)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("bits,layout", [(2, L.RQ_CODES_PACKED), (4, L.RQ_CODES_PACKED), (4, L.RQ_CODES_INT8),
                                         (5, L.RQ_CODES_PACKED), (8, L.RQ_CODES_PACKED)])
def test_dense_dequantize_matches_oracle(dtype, bits, layout):
    nb = 128 * 3 + 101
    rng = np.random.default_rng(bits)
    idx = rng.integers(0, 1 << bits, nb * d).astype(np.uint8)
    codes = O.pack_codes(idx, d, bits, layout)
    norms = np.float16(rng.random(nb) * 20 + 0.1).view(np.uint16)
    norms[5] = 0                                        # a zero block
    pi16 = rotation16(4, dtype)
    c32 = codebook(bits)
    out = torch.empty(nb * d, dtype=dtype, device=DEV)
    L.rq_dequantize_dense(torch.from_numpy(codes).to(DEV), torch.from_numpy(norms.view(np.int16)).to(DEV), nb * d, d,
                          dev16(pi16, dtype), bits, layout, c32, out)
    torch.cuda.synchronize()
    assert "dequantize_dense_kernel" in L.rq_last_launch()
    _, v = D.dequantize(codes, norms, nb, d, pi16, bits, layout, D.to16(c32, dt_code(dtype)), dt_code(dtype),
                        dt_code(dtype))
    g = out.float().cpu().numpy().astype(np.float64).reshape(nb, d)
    n16 = norms.view(np.float16).astype(np.float64)[:, None]
    tol = ulp16(v, dtype) + n16 * 2.0 ** -15
    err = np.abs(g - v)
    assert np.all(err <= tol), (np.max(err - tol), np.unravel_index(np.argmax(err - tol), err.shape))
    assert np.all(g[5] == 0)
    report("dense_dequantize", dtype=str(dtype), bits=bits, layout=layout, blocks=nb,
           max_err_over_tol=float(np.max(err / tol)))


def test_dense_zero_blocks_and_empty_call():
    # ||x|| = 0: z = 0 for every coordinate, code = #{t_k < 0} = K/2 - 1 (the
    # middle boundary of a symmetric table is exactly 0)
    nb, bits = 130, 4
    x = torch.zeros(nb * d, dtype=torch.bfloat16, device=DEV)
    x[128 * d:129 * d] = 1.0                            # one non-zero block in the last tile
    pi16 = rotation16(3, torch.bfloat16)
    c32 = codebook(bits)
    g_codes, g_norms = run_quantize(x, bits, L.RQ_CODES_PACKED, dev16(pi16, torch.bfloat16), c32)
    idx = O.unpack_codes(g_codes, nb, d, bits, L.RQ_CODES_PACKED).reshape(nb, d)
    assert np.all(idx[:128] == 7) and np.all(idx[129] == 7) and np.all(g_norms[:128] == 0)
    o_codes, o_norms, z, _ = D.quantize(u16(x), O.BF16, d, pi16, bits, L.RQ_CODES_PACKED, c32)
    np.testing.assert_array_equal(g_norms, o_norms)
    check_dense_codes(g_codes, o_codes, z, c32, nb, bits, L.RQ_CODES_PACKED)
    empty = torch.empty(0, dtype=torch.bfloat16, device=DEV)
    L.rq_quantize_dense(empty, d, dev16(pi16, torch.bfloat16), bits, L.RQ_CODES_PACKED, c32,
                        torch.empty(16, dtype=torch.uint8, device=DEV), torch.empty(16, dtype=torch.int16, device=DEV))


def test_dense_round_trip_error_is_the_codebook_error():
    # x^ = ||x|| Pi^T c[code(Pi x / ||x||)]: with Pi orthogonal the relative
    # squared error is the codebook's mean squared error times d (plus the
    # 16-bit roundings), about 0.0095 for the 4-bit Beta table at d = 128
    nb, bits = 4096, 4
    x = synth.normal((nb, d), seed=31, device=DEV).reshape(-1)
    pi_dev = dev16(rotation16(5, torch.bfloat16), torch.bfloat16)
    c32 = codebook(bits)
    codes = torch.empty(nb * d // 2, dtype=torch.uint8, device=DEV)
    norms = torch.empty(nb, dtype=torch.int16, device=DEV)
    out = torch.empty_like(x)
    L.rq_quantize_dense(x, d, pi_dev, bits, L.RQ_CODES_PACKED, c32, codes, norms)
    L.rq_dequantize_dense(codes, norms, x.numel(), d, pi_dev, bits, L.RQ_CODES_PACKED, c32, out)
    xv, ov = x.float().reshape(nb, d), out.float().reshape(nb, d)
    rel = ((ov - xv).pow(2).sum(1) / xv.pow(2).sum(1)).mean().item()
    assert 0.0085 < rel < 0.0110, rel


def test_dense_full_size_sampled():
    # the benchmark's V-cache workload (4 x 8 x 32768 blocks of 128, bf16, 4
    # bits packed): every block on the GPU, 2048 sampled blocks through the oracle
    nb, bits = 4 * 8 * 32768, 4
    x = synth.kv_with_channels(4, 8, 32768, d, seed=13, device=DEV).reshape(-1)
    pi16 = rotation16(6, torch.bfloat16)
    c32 = codebook(bits)
    g_codes, g_norms = run_quantize(x, bits, L.RQ_CODES_PACKED, dev16(pi16, torch.bfloat16), c32)
    rows = np.sort(np.random.default_rng(0).choice(nb, 2048, replace=False))
    rows[-1] = nb - 1
    xs = u16(x).reshape(nb, d)[rows]
    o_codes, o_norms, z, _ = D.quantize(xs, O.BF16, d, pi16, bits, L.RQ_CODES_PACKED, c32)
    np.testing.assert_array_equal(g_norms[rows], o_norms)
    gs = g_codes.reshape(nb, d * bits // 8)[rows].reshape(-1)
    nbad = check_dense_codes(gs, o_codes, z, c32, len(rows), bits, L.RQ_CODES_PACKED)
    report("dense_full_size", blocks=nb, sampled=len(rows), boundary_codes=nbad)
