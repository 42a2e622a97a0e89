"""Pins of the dense-rotation oracle (TurboQuant README, "Algorithm in one
paragraph": random orthogonal rotation by QR with sign fix, Lloyd-Max
centroids of the Beta coordinate law), each against something other than the
oracle itself: closed forms, an independent quadrature, the Gaussian limit,
exact special cases of the rotation."""
import math

import numpy as np
import pytest
from scipy import integrate
from scipy.special import gammaln

import oracle as O
from oracle import dense_rotation as D


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_beta_codebook_d3_is_the_uniform_quantizer(bits):
    # d = 3: (1 - t^2)^0, the uniform law on [-1, 1]; its Lloyd-Max quantizer
    # is the uniform one with levels -1 + (2k + 1) / K
    K = 1 << bits
    want = np.array([-1.0 + (2 * k + 1) / K for k in range(K)])
    np.testing.assert_allclose(D.beta_lloyd_max(3, bits), want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("d", [4, 16, 128, 1000])
def test_beta_codebook_one_bit_is_mean_abs(d):
    # one bit: the centroids are +-E|T| = Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2))
    e = math.exp(gammaln(d / 2.0) - 0.5 * math.log(math.pi) - gammaln((d + 1) / 2.0))
    np.testing.assert_allclose(D.beta_lloyd_max(d, 1), [-e, e], rtol=1e-12)


def test_beta_density_integrates_to_one_and_matches_the_tail():
    for d in (3, 5, 64, 300):
        tot, _ = integrate.quad(lambda t: float(D.beta_density(t, d)), -1, 1, epsabs=1e-13, limit=200)
        assert abs(tot - 1.0) < 1e-10
        for t in (0.0, 0.05, 0.2, 0.5):
            tail, _ = integrate.quad(lambda u: float(D.beta_density(u, d)), t, 1, epsabs=1e-14, limit=200)
            assert abs(float(D.beta_upper_tail(t, d)) - tail) < 1e-11, (d, t)


@pytest.mark.parametrize("d,bits", [(16, 2), (128, 3), (128, 4), (512, 4)])
def test_beta_codebook_is_a_lloyd_fixed_point(d, bits):
    # every centroid is its cell's conditional mean by independent quadrature
    c = D.beta_lloyd_max(d, bits)
    t = np.concatenate([[-1.0], 0.5 * (c[:-1] + c[1:]), [1.0]])
    f = lambda u: float(D.beta_density(u, d))
    for k in range(len(c)):
        m0, _ = integrate.quad(f, t[k], t[k + 1], epsabs=0, epsrel=1e-13, limit=200)
        m1, _ = integrate.quad(lambda u: u * f(u), t[k], t[k + 1], epsabs=0, epsrel=1e-13, limit=200)
        assert abs(m1 / m0 - c[k]) < 1e-9 * max(1.0, abs(c[k])), (k, m1 / m0, c[k])


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_beta_codebook_tends_to_the_gaussian_table(bits):
    # sqrt(d) T -> N(0, 1): the scaled Beta codebook approaches the N(0,1)
    # Lloyd-Max table (pinned against its printed values elsewhere) as O(1/d)
    g = O.lloyd_max(bits)
    err = [np.max(np.abs(D.beta_lloyd_max(d, bits) * math.sqrt(d) - g)) for d in (256, 4096)]
    assert err[1] < 2e-3
    assert err[1] < err[0] / 8


@pytest.mark.parametrize("d", [8, 64, 128])
def test_rotation_is_orthogonal_with_positive_r(d):
    Pi = D.rotation(11, d)
    np.testing.assert_allclose(Pi.T @ Pi, np.eye(d), atol=1e-12)
    # G = Pi R with R upper triangular and a positive diagonal (the sign fix)
    G = D.gaussian_matrix(11, d)
    R = Pi.T @ G
    assert np.max(np.abs(np.tril(R, -1))) < 1e-10
    assert np.all(np.diag(R) > 0)
    # G's entries are the projection stream's Box-Muller normals
    assert G[0, 1] == O.gauss(11, 1) and G[1, 0] == O.gauss(11, d)


def _perm_matrix(d, seed):
    rng = np.random.default_rng(seed)
    p = rng.permutation(d)
    s = np.where(rng.random(d) < 0.5, -1.0, 1.0)
    P = np.zeros((d, d))
    P[np.arange(d), p] = s                          # (P x)_j = s_j x_{p(j)}
    return P, p, s


@pytest.mark.parametrize("dtype", [O.BF16, O.F16])
def test_quantize_with_a_signed_permutation(dtype):
    # Pi a signed permutation (exact in 16 bits): z_j = s_j x_{p(j)} / ||x||,
    # the code is the count of boundaries below z_j
    d, bits, nb = 64, 3, 50
    rng = np.random.default_rng(1)
    x = rng.standard_normal((nb, d))
    x16 = D.to16(x, dtype)
    P, p, s = _perm_matrix(d, 2)
    c32 = (D.beta_lloyd_max(d, bits)).astype(np.float32)
    codes, norms, z, n32 = D.quantize(x16, dtype, d, D.to16(P, dtype), bits, O.PACKED, c32)
    xv = D.from16(x16, dtype)
    zz = s[None, :] * xv[:, p] / n32[:, None].astype(np.float64)
    np.testing.assert_array_equal(z, zz)
    t = (np.float32(0.5) * (c32[:-1] + c32[1:])).astype(np.float64)
    want = np.array([[int(np.sum(t < v)) for v in row] for row in zz], np.uint8)
    np.testing.assert_array_equal(O.unpack_codes(codes, nb, d, bits, O.PACKED).reshape(nb, d), want)
    np.testing.assert_allclose(n32, np.linalg.norm(xv, axis=1), rtol=1e-6)


def test_dequantize_with_a_signed_permutation():
    d, bits, nb = 32, 4, 20
    rng = np.random.default_rng(3)
    idx = rng.integers(0, 1 << bits, (nb, d)).astype(np.uint8)
    codes = O.pack_codes(idx.reshape(-1), d, bits, O.PACKED)
    norms = np.float16(rng.random(nb) * 4 + 0.5).view(np.uint16)
    P, p, s = _perm_matrix(d, 4)
    cop = D.to16(D.beta_lloyd_max(d, bits), O.BF16)
    out16, v = D.dequantize(codes, norms, nb, d, D.to16(P, O.BF16), bits, O.PACKED, cop, O.BF16, O.BF16)
    c = D.from16(cop, O.BF16)[idx]
    # (P^T c)_i: entry P[j, p(j)] = s_j sends s_j c_j to coordinate p(j)
    want = np.zeros((nb, d))
    want[:, p] = s[None, :] * c
    np.testing.assert_array_equal(v, norms.view(np.float16).astype(np.float64)[:, None] * want)


def test_hadamard_rotation_reduces_to_the_walsh_hadamard_path():
    # Pi = H D / sqrt(d) in fp16 with the N(0,1) table divided by sqrt(d): the
    # codes of the Walsh-Hadamard oracle, except where z sits on a boundary
    d, bits, nb = 128, 3, 200
    rng = np.random.default_rng(5)
    x16 = D.to16(rng.standard_normal((nb, d)), O.F16)
    sgn = O.sign_diagonal(9, d).astype(np.float64)
    H = O.hadamard_matrix(d).astype(np.float64)
    Pi16 = D.to16(H * sgn[None, :] / math.sqrt(d), O.F16)
    g32 = O.f32_table(bits)
    dense_c = (g32.astype(np.float64) / math.sqrt(d)).astype(np.float32)
    codes_d, _, z, _ = D.quantize(x16, O.F16, d, Pi16, bits, O.PACKED, dense_c)
    codes_w, _, _, _ = O.quantize(x16, O.F16, d, bits, O.PACKED, O.sign_diagonal(9, d), g32)
    a = O.unpack_codes(codes_d, nb, d, bits, O.PACKED).astype(int)
    b = O.unpack_codes(codes_w, nb, d, bits, O.PACKED).astype(int)
    assert np.all(np.abs(a - b) <= 1)
    assert np.mean(a == b) > 0.995
