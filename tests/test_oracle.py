"""Pins of the CPU oracle against facts fixed outside it.

Every check here ties the oracle to something other than itself: values printed
on the pages or in the literature (tests/golden/, each file cites its source),
closed forms, library routines (scipy, numpy, torch conversions), invariants and
brute force on tiny inputs.  A plausible mistake anywhere in the oracle -- a
dropped term, a wrong sign or index, a transposed operand -- fails one of them.
"""
import math

import numpy as np
import pytest
import scipy.linalg
from scipy import integrate, stats

import oracle as O
from tests.conftest import read_golden

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def rand_u16(rng, shape, std, dtype):
    """Random 16-bit patterns (host numpy only, for oracle-only tests)."""
    import torch
    x = torch.from_numpy((rng.standard_normal(shape) * std).astype(np.float32))
    x = x.to(torch.bfloat16 if dtype == O.BF16 else torch.float16)
    return x.view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------------ Lloyd-Max

@pytest.mark.parametrize("bits", [1, 2, 3])
def test_lloyd_max_matches_max_1960(bits):
    want = {int(r[0]): [float(v) for v in r[1:]] for r in read_golden("lloyd_max_n01.txt")}[bits]
    c = O.lloyd_max(bits)
    K = 1 << bits
    assert np.all(np.diff(c) > 0)
    # the printed table carries 3-4 decimals (1.344, 2.152 in the original)
    assert np.allclose(c[K // 2:], want, rtol=0, atol=1.2e-4)
    assert np.allclose(c[: K // 2], -np.array(want[::-1]), rtol=0, atol=1.2e-4)


def test_lloyd_max_one_bit_closed_form():
    c = O.lloyd_max(1)
    assert abs(c[1] - math.sqrt(2 / math.pi)) < 1e-14


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6])
def test_lloyd_max_fixed_point_by_quadrature(bits):
    """Independent check with scipy: each level is the conditional mean of its
    cell (centroid condition) and the table MSE equals the integral."""
    c = O.lloyd_max(bits)
    t = np.concatenate([[-np.inf], 0.5 * (c[1:] + c[:-1]), [np.inf]])
    worst = 0.0
    mse = 0.0
    for i, ci in enumerate(c):
        p = stats.norm.cdf(t[i + 1]) - stats.norm.cdf(t[i])
        m1 = integrate.quad(lambda z: z * stats.norm.pdf(z), t[i], t[i + 1], epsabs=1e-15)[0]
        worst = max(worst, abs(m1 / p - ci))
        mse += integrate.quad(lambda z: (z - ci) ** 2 * stats.norm.pdf(z), t[i], t[i + 1], epsabs=1e-15)[0]
    assert worst < 1e-9
    assert abs(O.table_mse(c) - mse) < 1e-10


def test_lloyd_max_distortion_matches_turbopress_table():
    rows = {r[0]: float(r[1]) for r in read_golden("turbopress_single_layer.txt")}
    for bits in (2, 3, 4):
        assert abs(math.sqrt(O.table_mse(O.lloyd_max(bits))) - rows[f"nearest{bits}"]) < 1.5e-3


# ------------------------------------------------------------------ 16-bit formats

def test_half_and_bfloat_rounding_match_library():
    import torch
    rng = np.random.default_rng(1)
    x = np.concatenate([
        (rng.standard_normal(20000) * 10.0 ** rng.uniform(-9, 5, 20000)).astype(np.float32),
        np.array([0.0, -0.0, 65504, 65519.99, 65520, 6.1e-5, 5.96e-8, 2.98e-8, 2.9802322e-8,
                  1e-30, 3.4e38, -3.39e38, np.inf, -np.inf], np.float32)])
    with np.errstate(over="ignore"):
        want16 = x.astype(np.float16).view(np.uint16)
    wantbf = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got16 = np.array([O.f32_to_f16(float(v)) for v in x], np.uint16)
    gotbf = np.array([O.f32_to_bf16(float(v)) for v in x], np.uint16)
    assert np.array_equal(got16, want16)
    assert np.array_equal(gotbf, wantbf)
    back = np.array([O.f16_to_f32(int(h)) for h in want16], np.float32)
    assert np.array_equal(back, want16.view(np.float16).astype(np.float32))


# ------------------------------------------------------------------ RNG

def test_splitmix64_reference_vector():
    for seed, k, out in read_golden("splitmix64.txt"):
        assert O.splitmix64(int(seed), int(k)) == int(out)


def test_sign_diagonal_bits():
    s = O.sign_diagonal(99, 256)
    for j in range(256):
        w = O.splitmix64(99, j // 64)
        assert s[j] == (-1 if (w >> (j % 64)) & 1 else 1)
    assert abs(int(s.sum())) < 60   # balanced Rademacher


def test_gaussian_is_standard_normal():
    z = np.array([O.gauss(5, k) for k in range(200000)])
    assert abs(z.mean()) < 0.01 and abs(z.var() - 1.0) < 0.015
    assert stats.kstest(z, "norm").pvalue > 1e-3


def test_projection_entries_are_rounded_gauss():
    import torch
    S = O.projection(3, 16, 32, O.BF16)
    z = np.array([O.gauss(3, k) for k in range(16 * 32)], np.float64).astype(np.float32)
    want = torch.from_numpy(z).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(S.reshape(-1), want)
    S16 = O.projection(3, 16, 32, O.F16)
    assert np.array_equal(S16.reshape(-1), z.astype(np.float16).view(np.uint16))


# ------------------------------------------------------------------ Hadamard

@pytest.mark.parametrize("d", [2, 4, 8, 64, 128, 256, 512])
def test_hadamard_is_sylvester(d):
    H = O.hadamard_matrix(d)
    assert np.array_equal(H, scipy.linalg.hadamard(d).astype(np.float64))
    assert np.array_equal(H @ H.T, d * np.eye(d))


@pytest.mark.parametrize("d", [2, 4, 16, 128, 512])
def test_fwht_equals_matrix_product(d):
    rng = np.random.default_rng(d)
    v = rng.standard_normal((5, d))
    H = scipy.linalg.hadamard(d).astype(np.float64)
    got = O.fwht_f64(v)
    assert np.allclose(got, v @ H.T, atol=1e-12 * d)
    # fp32 canonical transform stays within a few ulps of the fp64 one
    g32 = O.fwht_f32(v.astype(np.float32))
    assert np.max(np.abs(g32 - v.astype(np.float32).astype(np.float64) @ H.T)) < 1e-5 * math.sqrt(d) * np.abs(v).max() * 4
    # rotation preserves norms (orthonormal H / sqrt(d)); H is its own inverse up to d
    assert np.allclose(np.linalg.norm(got, axis=1), math.sqrt(d) * np.linalg.norm(v, axis=1))
    assert np.allclose(O.fwht_f64(got), d * v)


def test_fwht_by_hand_d2_d4():
    assert np.array_equal(O.fwht_f64(np.array([3.0, 5.0])), [8.0, -2.0])
    assert np.array_equal(O.fwht_f64(np.array([1.0, 2.0, 3.0, 4.0])), [10.0, -2.0, -4.0, 0.0])


def test_pairwise_sum():
    v = np.arange(1, 129, dtype=np.float32)
    assert O.pairwise_sum(v) == 128 * 129 / 2
    rng = np.random.default_rng(0)
    w = rng.standard_normal(512).astype(np.float32) ** 2
    assert abs(O.pairwise_sum(w) - math.fsum(w.astype(np.float64))) < 1e-6 * w.sum()


# ------------------------------------------------------------------ packing

def test_packing_golden():
    for row in read_golden("packing.txt"):
        bits = int(row[0])
        codes = np.array([int(v) for v in row[1].split(",")], np.uint8)
        want = np.array([int(v, 16) for v in row[3].split(",")], np.uint8)
        got = O.pack_codes(codes, 8, bits, O.PACKED)
        assert np.array_equal(got, want), (bits, got, want)
        assert np.array_equal(O.unpack_codes(got, 1, 8, bits, O.PACKED), codes)


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6, 7, 8])
def test_pack_roundtrip(bits):
    rng = np.random.default_rng(bits)
    idx = rng.integers(0, 1 << bits, 16 * 128, dtype=np.uint8)
    for layout in (O.PACKED, O.INT8):
        p = O.pack_codes(idx, 128, bits, layout)
        assert p.size == 16 * O.code_bytes_per_block(128, bits, layout)
        assert np.array_equal(O.unpack_codes(p, 16, 128, bits, layout), idx)


# ------------------------------------------------------------------ quantizer

def _brute_codes(y64, c):
    return np.argmin(np.abs(y64[:, None] - c[None, :].astype(np.float64)), axis=1)


@pytest.mark.parametrize("d", [2, 4, 8, 128])
@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5])
def test_quantize_is_nearest_centroid(d, bits):
    rng = np.random.default_rng(100 * d + bits)
    x = rand_u16(rng, 4096 if d < 128 else 64 * 128, 0.02, O.BF16)
    c = O.f32_table(bits)
    s = O.sign_diagonal(11, d)
    codes, norms, y, n32 = O.quantize(x, O.BF16, d, bits, O.INT8, s, c, want_y=True)
    y64 = O.rotate_f64(x, O.BF16, d, s)
    t = O.boundaries(c).astype(np.float64)
    window = np.min(np.abs(y64[:, None] - t[None, :]), axis=1) <= 1e-5
    brute = _brute_codes(y64, c)
    mism = codes != brute
    assert not np.any(mism & ~window)
    # fp32 canonical y stays within the window of the fp64 value
    assert np.max(np.abs(y - y64)) < 1e-5
    # norms: fp16 of the exact L2 norm, within one fp16 ulp
    xf = np.array([O.bf16_to_f32(int(h)) for h in x], np.float64).reshape(-1, d)
    nex = np.linalg.norm(xf, axis=1)
    nf = np.array([O.f16_to_f32(int(h)) for h in norms])
    assert np.all(np.abs(nf - nex) <= np.spacing(nex.astype(np.float16)).astype(np.float64) * 1.0 + 1e-12)


def test_quantize_zero_block_and_signs_off():
    c = O.f32_table(4)
    x = np.zeros(128, np.uint16)
    codes, norms, y, _ = O.quantize(x, O.BF16, 128, 4, O.INT8, None, c, want_y=True)
    assert norms[0] == 0 and np.all(y == 0)
    assert np.all(codes == 7)  # #{t_k < 0} for the symmetric 16-level table
    out, _ = O.dequantize(codes, norms, 128, 4, O.INT8, None, c, O.BF16)
    assert np.all((out & 0x7fff) == 0)   # +-0: the sign of H c survives the zero scale


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_code_idempotence_and_constructed_blocks(bits):
    rng = np.random.default_rng(bits)
    d = 128
    c = O.f32_table(bits)
    s = O.sign_diagonal(3, d)
    x = rand_u16(rng, 256 * d, 1.0, O.F16)
    codes, norms, _, _ = O.quantize(x, O.F16, d, bits, O.PACKED, s, c)
    xh, _ = O.dequantize(codes, norms, d, bits, O.PACKED, s, c, O.F16)
    codes2, _, _, _ = O.quantize(xh, O.F16, d, bits, O.PACKED, s, c)
    i1 = O.unpack_codes(codes, 256, d, bits, O.PACKED)
    i2 = O.unpack_codes(codes2, 256, d, bits, O.PACKED)
    assert np.mean(i1 != i2) < 1e-3
    # blocks built as x = D H^-1 (3 c_idx) rotate back to y = alpha * c_idx with
    # alpha = sqrt(d) / ||c_idx||, so their codes are the brute-force nearest
    # levels to alpha * c_idx, and their norm is 3 ||c_idx|| / sqrt(d)
    H = scipy.linalg.hadamard(d).astype(np.float64)
    idx = rng.integers(0, 1 << bits, (8, d))
    import torch
    for b in range(8):
        cv = c[idx[b]].astype(np.float64)
        xb = (s * (H.T @ (3.0 * cv))) / d
        x16 = torch.from_numpy(xb.astype(np.float32)).to(torch.float16)
        codes_b, norms_b, _, _ = O.quantize(x16.view(torch.int16).numpy().view(np.uint16), O.F16, d, bits,
                                            O.INT8, s, c)
        alpha = math.sqrt(d) / np.linalg.norm(cv)
        want = _brute_codes(alpha * cv, c)
        # fp16 rounding of the constructed input moves y by < 2e-3: only
        # coordinates that close to a decision boundary may differ
        near = np.min(np.abs((alpha * cv)[:, None] - O.boundaries(c)[None, :]), axis=1) < 2e-3
        assert not np.any((codes_b != want) & ~near)
        want_norm = 3.0 * np.linalg.norm(cv) / math.sqrt(d)
        assert abs(O.f16_to_f32(int(norms_b[0])) - want_norm) < 2e-3 * want_norm


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_reconstruction_rel_rmse_matches_turbopress(bits):
    """Isotropic blocks: relative RMSE of <q, x^> vs <q, x> equals sqrt(MSE_b),
    the turbopress single-layer nearest-rounding figure."""
    rows = {r[0]: float(r[1]) for r in read_golden("turbopress_single_layer.txt")}
    rng = np.random.default_rng(7 + bits)
    d = 1024
    n = 48
    c = O.f32_table(bits)
    s = O.sign_diagonal(0, d)
    x = rand_u16(rng, n * d, 1.0, O.F16)
    codes, norms, _, _ = O.quantize(x, O.F16, d, bits, O.PACKED, s, c)
    xh = O.dequantize_f64(codes, norms, d, bits, O.PACKED, s, c).reshape(n, d)
    xf = x.view(np.float16).astype(np.float64).reshape(n, d)
    q = rng.standard_normal((64, d))
    err = (xh - xf) @ q.T
    ref = xf @ q.T
    rel = math.sqrt(np.mean(err ** 2) / np.mean(ref ** 2))
    assert abs(rel - rows[f"nearest{bits}"]) < 0.012, rel


def test_dequantize_f32_vs_f64():
    rng = np.random.default_rng(5)
    d, bits = 256, 5
    c = O.f32_table(bits)
    s = O.sign_diagonal(1, d)
    x = rand_u16(rng, 64 * d, 0.02, O.BF16)
    codes, norms, _, _ = O.quantize(x, O.BF16, d, bits, O.PACKED, s, c)
    out, xh32 = O.dequantize(codes, norms, d, bits, O.PACKED, s, c, O.BF16, want_f32=True)
    xh64 = O.dequantize_f64(codes, norms, d, bits, O.PACKED, s, c)
    nb = np.array([O.f16_to_f32(int(h)) for h in norms]).repeat(d)
    assert np.max(np.abs(xh32 - xh64) / nb) < 1e-6
    outf = np.array([O.bf16_to_f32(int(h)) for h in out])
    assert np.array_equal(outf.astype(np.float32), np.array([O.bf16_to_f32(O.f32_to_bf16(float(v))) for v in xh32], np.float32))


# ------------------------------------------------------------------ QJL

def test_sign_bits_follow_decode_convention():
    """Bit i of byte i//8 = (P_i >= 0); decoding with ((byte >> j) & 1) * 2 - 1
    (qjl_apply.py `_qjl_decode_keys`) gives back sign(S v)."""
    rng = np.random.default_rng(2)
    d, m = 64, 40
    v = rand_u16(rng, 7 * d, 1.0, O.BF16)
    S = O.projection(9, m, d, O.BF16)
    packed, p = O.sketch(v, O.BF16, d, m, S, want_p=True)
    bit_idx = np.arange(8, dtype=np.uint8)
    unpacked = ((packed.reshape(7, m // 8)[:, :, None] >> bit_idx) & 1).reshape(7, m)
    sgn = unpacked.astype(np.float64) * 2 - 1
    Sf = np.array([O.bf16_to_f32(int(h)) for h in S.reshape(-1)]).reshape(m, d)
    vf = np.array([O.bf16_to_f32(int(h)) for h in v]).reshape(7, d)
    P = vf @ Sf.T
    assert np.array_equal(sgn, np.where(P >= 0, 1.0, -1.0))
    assert np.allclose(p.reshape(7, m), P / np.linalg.norm(vf, axis=1, keepdims=True))


def test_k_side_ratio_accounting():
    for hd, m, ratio in read_golden("qjl_k_side_ratio.txt"):
        hd, m = int(hd), int(m)
        sketch_bytes = O.sketch(np.zeros(hd, np.uint16), O.BF16, hd, m, np.zeros(m * hd, np.uint16))[0].size
        norm_bytes = O.vec_norms(np.zeros(hd, np.uint16), O.BF16, hd).nbytes
        assert round(hd * 2 / (sketch_bytes + norm_bytes), 2) == float(ratio)


def test_qjl_estimator_unbiased_and_variance():
    """Monte-Carlo over projection seeds: mean -> <q, r>, variance ->
    (1/m) [(pi/2) ||r||^2 ||q||^2 - <q, r>^2] (the sign-estimator variance; the
    turbopress findings give the same sqrt(pi/2)||r|| ||x|| / sqrt(k) scale)."""
    import torch
    rng = np.random.default_rng(3)
    d, m, trials = 32, 32, 6000
    r = torch.from_numpy(rng.standard_normal(d).astype(np.float32)).to(torch.bfloat16)
    q = torch.from_numpy((0.6 * r.float().numpy() + 0.8 * rng.standard_normal(d)).astype(np.float32)).to(torch.bfloat16)
    r16 = r.view(torch.int16).numpy().view(np.uint16)
    q16 = q.view(torch.int16).numpy().view(np.uint16)
    rn = O.vec_norms(r16, O.BF16, d)
    rf, qf = r.double().numpy(), q.double().numpy()
    est = np.empty(trials)
    for k in range(trials):
        S = O.projection(1000 + k, m, d, O.BF16)
        sg, _ = O.sketch(r16, O.BF16, d, m, S)
        est[k] = O.score(q16, 1, 1, d, m, S, O.BF16, sg, rn, 1)[0, 0, 0]
    true = float(qf @ rf) * O.f16_to_f32(int(rn[0])) / np.linalg.norm(rf)
    var_th = ((math.pi / 2) * np.dot(rf, rf) * np.dot(qf, qf) - np.dot(qf, rf) ** 2) / m
    se = math.sqrt(var_th / trials)
    assert abs(est.mean() - true) < 4 * se + 0.004 * abs(true), (est.mean(), true, se)
    assert abs(est.var() / var_th - 1.0) < 0.08


def test_two_stage_rel_rmse_matches_turbopress():
    """2-bit rotated Lloyd-Max + QJL (m = d) on the residual: relative RMSE
    of the inner-product estimate ~ sqrt((pi/2) * MSE_2b) = 0.43 (turbopress
    single-layer table, row "2b + QJL k=d")."""
    rows = {r[0]: float(r[1]) for r in read_golden("turbopress_single_layer.txt")}
    rng = np.random.default_rng(4)
    d, n, nq, bits = 128, 96, 16, 2
    m = d
    c = O.f32_table(bits)
    s = O.sign_diagonal(4, d)
    x = rand_u16(rng, n * d, 1.0, O.BF16)
    codes, norms, _, _ = O.quantize(x, O.BF16, d, bits, O.PACKED, s, c)
    r_bf, rn = O.residual(x, O.BF16, codes, norms, d, bits, O.PACKED, s, c)
    q = rand_u16(rng, nq * d, 1.0, O.BF16)
    errs, refs = [], []
    for k in range(6):
        S = O.projection(50 + k, m, d, O.BF16)
        sg, _ = O.sketch(r_bf, O.BF16, d, m, S)
        est = O.score(q, 1, nq, d, m, S, O.BF16, sg, rn, n, codes=codes, norms=norms, bits=bits,
                      layout=O.PACKED, signs_diag=s, c32=c)[0]
        xf = x.view(np.uint16).astype(np.uint32) << 16
        xf = xf.view(np.float32).astype(np.float64).reshape(n, d)
        qf = (q.astype(np.uint32) << 16).view(np.float32).astype(np.float64).reshape(nq, d)
        ref = qf @ xf.T
        errs.append(est - ref)
        refs.append(ref)
    rel = math.sqrt(np.mean(np.square(errs)) / np.mean(np.square(refs)))
    assert abs(rel - rows["nearest2+qjl_k=d"]) < 0.03, rel


def test_score_first_stage_equals_dot_with_reconstruction():
    """With no sign bits contributing (zero sketch norm), the score is exactly
    <q, x^> where x^ is the fp64 reconstruction: this fixes q~ = H D q."""
    rng = np.random.default_rng(6)
    d, n, nq, bits, m = 64, 10, 3, 3, 8
    c = O.f32_table(bits)
    s = O.sign_diagonal(8, d)
    x = rand_u16(rng, n * d, 1.0, O.BF16)
    q = rand_u16(rng, nq * d, 1.0, O.BF16)
    codes, norms, _, _ = O.quantize(x, O.BF16, d, bits, O.PACKED, s, c)
    S = O.projection(1, m, d, O.BF16)
    sc = O.score(q, 1, nq, d, m, S, O.BF16, np.zeros(n * m // 8, np.uint8), np.zeros(n, np.uint16), n,
                 codes=codes, norms=norms, bits=bits, layout=O.PACKED, signs_diag=s, c32=c)[0]
    xh = O.dequantize_f64(codes, norms, d, bits, O.PACKED, s, c).reshape(n, d)
    qf = (q.astype(np.uint32) << 16).view(np.float32).astype(np.float64).reshape(nq, d)
    assert np.allclose(sc, qf @ xh.T, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ attention over compressed K/V

def _attn_case(rng, G, T, nq, d, m, kbits, vbits, two_stage=True):
    """Keys (two-stage or pure QJL) and 4-bit values of G groups, compressed
    by the oracle; returns the arguments of O.attention and the pieces a pin
    needs."""
    kc, vc = O.f32_table(kbits), O.f32_table(vbits)
    ks, vs = O.sign_diagonal(21, d), O.sign_diagonal(22, d)
    S = O.projection(23, m, d, O.BF16)
    k = rand_u16(rng, G * T * d, 1.0, O.BF16)
    v = rand_u16(rng, G * T * d, 1.0, O.BF16)
    q = rand_u16(rng, G * nq * d, 1.0, O.BF16)
    if two_stage:
        codes, norms, _, _ = O.quantize(k, O.BF16, d, kbits, O.PACKED, ks, kc)
        r, rn = O.residual(k, O.BF16, codes, norms, d, kbits, O.PACKED, ks, kc)
        sg, _ = O.sketch(r, O.BF16, d, m, S)
        kw = dict(codes=codes, norms=norms, bits=kbits, layout=O.PACKED, signs_diag=ks, c32=kc)
    else:
        sg, _ = O.sketch(k, O.BF16, d, m, S)
        rn = O.vec_norms(k, O.BF16, d)
        kw = {}
    vcodes, vnorms, _, _ = O.quantize(v, O.BF16, d, vbits, O.PACKED, vs, vc)
    return dict(q=q, S=S, sg=sg, rn=rn, kw=kw, vcodes=vcodes, vnorms=vnorms, vs=vs, vc=vc)


def _attn(c, G, nq, d, m, T, vbits, scale, **over):
    a = dict(c)
    a.update(over)
    return O.attention(a["q"], G, nq, d, m, a["S"], O.BF16, a["sg"], a["rn"], T, a["vcodes"], a["vnorms"], vbits,
                       O.PACKED, a["vs"], a["vc"], scale, **a["kw"])


@pytest.mark.parametrize("two_stage", [True, False])
def test_attention_matches_scipy_softmax_of_scores(two_stage):
    """softmax(scale * score) @ V with scipy's softmax and numpy's product over
    the oracle's own (pinned) scores and fp64 reconstructions: fixes the
    scale, the per-group key/value offsets and the normalisation."""
    from scipy.special import softmax
    rng = np.random.default_rng(30)
    G, T, nq, d, m, vbits = 3, 37, 5, 64, 64, 4
    c = _attn_case(rng, G, T, nq, d, m, 2, vbits, two_stage)
    scale = 1.0 / math.sqrt(d)
    got = _attn(c, G, nq, d, m, T, vbits, scale)
    sc = O.score(c["q"], G, nq, d, m, c["S"], O.BF16, c["sg"], c["rn"], T, **c["kw"])
    vh = O.dequantize_f64(c["vcodes"], c["vnorms"], d, vbits, O.PACKED, c["vs"], c["vc"]).reshape(G, T, d)
    want = np.einsum("gqt,gtd->gqd", softmax(scale * sc, axis=-1), vh)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def test_attention_single_key_returns_its_value():
    rng = np.random.default_rng(31)
    G, T, nq, d, m, vbits = 2, 1, 3, 128, 128, 4
    c = _attn_case(rng, G, T, nq, d, m, 3, vbits)
    got = _attn(c, G, nq, d, m, T, vbits, 0.125)
    vh = O.dequantize_f64(c["vcodes"], c["vnorms"], d, vbits, O.PACKED, c["vs"], c["vc"]).reshape(G, 1, d)
    assert np.array_equal(got, np.broadcast_to(vh, (G, nq, d)))


def test_attention_equal_keys_average_the_values():
    """Every key of a group identical: the weights are uniform whatever the
    scores, so the output is the plain mean of the reconstructed values."""
    rng = np.random.default_rng(32)
    G, T, nq, d, m, vbits = 2, 20, 4, 64, 64, 3
    c = _attn_case(rng, G, T, nq, d, m, 2, vbits)
    mb = m // 8
    for key in ("sg", "rn"):
        arr = c[key].reshape(G, T, -1)
        c[key] = np.ascontiguousarray(np.repeat(arr[:, :1], T, axis=1)).reshape(-1)
    cb = O.code_bytes_per_block(d, 2, O.PACKED)
    c["kw"]["codes"] = np.ascontiguousarray(np.repeat(c["kw"]["codes"].reshape(G, T, cb)[:, :1], T, axis=1)).reshape(-1)
    c["kw"]["norms"] = np.ascontiguousarray(np.repeat(c["kw"]["norms"].reshape(G, T)[:, :1], T, axis=1)).reshape(-1)
    assert c["sg"].size == G * T * mb
    got = _attn(c, G, nq, d, m, T, vbits, 0.3)
    vh = O.dequantize_f64(c["vcodes"], c["vnorms"], d, vbits, O.PACKED, c["vs"], c["vc"]).reshape(G, T, d)
    want = np.broadcast_to(vh.mean(axis=1)[:, None, :], (G, nq, d))
    assert np.allclose(got, want, rtol=1e-13, atol=1e-13)


def test_attention_token_permutation_invariant_and_hard_limit():
    """Permuting the tokens (keys and values together) leaves the output
    unchanged; a very large scale selects the value of the top-scoring key
    (and the max subtraction keeps it finite)."""
    rng = np.random.default_rng(33)
    G, T, nq, d, m, vbits, kbits = 1, 29, 4, 64, 64, 4, 2
    c = _attn_case(rng, G, T, nq, d, m, kbits, vbits)
    base = _attn(c, G, nq, d, m, T, vbits, 0.2)
    perm = rng.permutation(T)
    mb, cb, vcb = m // 8, O.code_bytes_per_block(d, kbits, O.PACKED), O.code_bytes_per_block(d, vbits, O.PACKED)
    p = dict(c)
    p["sg"] = np.ascontiguousarray(c["sg"].reshape(T, mb)[perm]).reshape(-1)
    p["rn"] = np.ascontiguousarray(c["rn"][perm])
    p["vcodes"] = np.ascontiguousarray(c["vcodes"].reshape(T, vcb)[perm]).reshape(-1)
    p["vnorms"] = np.ascontiguousarray(c["vnorms"][perm])
    p["kw"] = dict(c["kw"])
    p["kw"]["codes"] = np.ascontiguousarray(c["kw"]["codes"].reshape(T, cb)[perm]).reshape(-1)
    p["kw"]["norms"] = np.ascontiguousarray(c["kw"]["norms"][perm])
    assert np.allclose(_attn(p, G, nq, d, m, T, vbits, 0.2), base, rtol=1e-12, atol=1e-12)
    sc = O.score(c["q"], G, nq, d, m, c["S"], O.BF16, c["sg"], c["rn"], T, **c["kw"])[0]
    top = np.argsort(sc, axis=1)
    gap = sc[np.arange(nq), top[:, -1]] - sc[np.arange(nq), top[:, -2]]
    scale = 800.0 / gap.min()
    hard = _attn(c, G, nq, d, m, T, vbits, scale)[0]
    vh = O.dequantize_f64(c["vcodes"], c["vnorms"], d, vbits, O.PACKED, c["vs"], c["vc"]).reshape(T, d)
    assert np.all(np.isfinite(hard))
    assert np.allclose(hard, vh[top[:, -1]], rtol=0, atol=1e-12)


# ------------------------------------------------------------------ non-power-of-two blocks

def test_sub_blocks_follow_the_printed_decomposition():
    for row in read_golden("block_diagonal_sizes.txt"):
        d, want = int(row[0]), [int(v) for v in row[1:]]
        assert [b for _, b in O.sub_blocks(d)] == want
    for d in (96, 160, 192, 224, 320, 448, 480, 128, 512):
        sb = O.sub_blocks(d)
        sizes = [b for _, b in sb]
        assert sum(sizes) == d and sizes == sorted(sizes, reverse=True)
        assert all(b & (b - 1) == 0 for b in sizes) and len(set(sizes)) == len(sizes)
        assert [o for o, _ in sb] == [sum(sizes[:i]) for i in range(len(sizes))]


def _rotation_matrix(d, signs):
    """sqrt(d) blockdiag(H_b / sqrt(b)) D from scipy's Sylvester Hadamard."""
    blocks = [scipy.linalg.hadamard(b) / math.sqrt(b) for _, b in O.sub_blocks(d)]
    return math.sqrt(d) * scipy.linalg.block_diag(*blocks) @ np.diag(signs.astype(np.float64))


@pytest.mark.parametrize("d", [96, 192, 320, 448])
def test_block_diagonal_rotation_matches_scipy(d):
    """y = sqrt(d) R x / ||x|| with R = blockdiag(H_b / sqrt(b)) D orthogonal:
    the fp64 rotation against scipy's Hadamard, ||y|| = sqrt(d), and the fp32
    canonical coordinates within a few ulps of it."""
    rng = np.random.default_rng(d)
    n = 7
    x = rand_u16(rng, n * d, 1.0, O.BF16)
    s = O.sign_diagonal(11, d)
    R = _rotation_matrix(d, s)
    assert np.allclose(R @ R.T, d * np.eye(d), atol=1e-9)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64).reshape(n, d)
    want = (xf @ R.T) / np.linalg.norm(xf, axis=1, keepdims=True)
    y64 = O.rotate_f64(x, O.BF16, d, s).reshape(n, d)
    assert np.allclose(y64, want, rtol=1e-12, atol=1e-12)
    assert np.allclose(np.linalg.norm(y64, axis=1), math.sqrt(d), rtol=1e-12)
    _, _, y32, _ = O.quantize(x, O.BF16, d, 4, O.PACKED, s, O.f32_table(4), want_y=True)
    assert np.abs(y32.reshape(n, d) - y64).max() <= 1e-5 * np.abs(y64).max()


@pytest.mark.parametrize("d,bits", [(96, 4), (160, 3), (448, 2)])
def test_block_diagonal_codes_are_nearest_and_reconstruct(d, bits):
    """Codes are the nearest centroid of the fp32 coordinates (brute force), and
    the fp64 reconstruction is ||x||16 R^T c / sqrt(d) (scipy); the fp32 one
    stays within 1e-6 of it relative to the block norm."""
    rng = np.random.default_rng(d + bits)
    n = 9
    x = rand_u16(rng, n * d, 1.0, O.BF16)
    s = O.sign_diagonal(12, d)
    c = O.f32_table(bits)
    codes, norms, y32, _ = O.quantize(x, O.BF16, d, bits, O.PACKED, s, c, want_y=True)
    idx = O.unpack_codes(codes, n, d, bits, O.PACKED).reshape(n, d).astype(np.int64)
    y = y32.reshape(n, d).astype(np.float64)
    dist = np.abs(y[..., None] - c.astype(np.float64)[None, None, :])
    best = dist.min(-1, keepdims=True)
    assert np.all(dist[np.arange(n)[:, None], np.arange(d)[None, :], idx] <= best[..., 0] + 1e-12)
    R = _rotation_matrix(d, s)
    n16 = np.array([O.f16_to_f32(int(h)) for h in norms], np.float64)
    want = (c.astype(np.float64)[idx] @ R) * (n16[:, None] / d)
    xh64 = O.dequantize_f64(codes, norms, d, bits, O.PACKED, s, c).reshape(n, d)
    assert np.allclose(xh64, want, rtol=1e-12, atol=1e-12)
    _, xh32 = O.dequantize(codes, norms, d, bits, O.PACKED, s, c, O.BF16, want_f32=True)
    assert np.abs(xh32.reshape(n, d) - xh64).max() <= 1e-6 * n16.max()
