"""CPU oracle for quantization with a dense random orthogonal rotation and a
Beta-distribution Lloyd-Max codebook.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg may import this module; it never imports the
product library.  Plain numpy / scipy, float64 unless stated.

Source followed: eliza "scripts/quantization" README, section "TurboQuant",
"Algorithm in one paragraph":
  (1) store ||x||;
  (2) rotate the unit vector x / ||x|| by a fixed random orthogonal matrix Pi,
      drawn by the QR decomposition of a Gaussian matrix with the sign fix;
      each rotated coordinate then follows the law of one coordinate of a
      uniform point on the unit sphere (a Beta law on [-1, 1], close to
      N(0, 1/d) for large d);
  (3) bucketize each coordinate against the Lloyd-Max centroids of that law
      at b bits;
  (4) bit-pack the indices;
  inverse: centroid lookup, x^ = ||x|| Pi^T c.

Readings where the page leaves a step open (listed in the design notes too):
  - The coordinate law.  A coordinate t of a uniform unit vector in R^d has
    density f_d(t) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) (1 - t^2)^((d-3)/2)
    on [-1, 1] (t^2 ~ Beta(1/2, (d-1)/2)); that is the "Beta distribution"
    the page names.
  - Sign fix: Pi = Q diag(sign(diag(R))) for G = Q R (a Haar-distributed
    orthogonal matrix; its determinant may be -1).
  - G[i][j] = gauss(seed, i*d + j), the same Box-Muller-over-SplitMix64
    stream the projection matrix uses, kept in float64.
  - Operand precision.  The rotation runs as a 16-bit GEMM: Pi and the
    centroid operand of the inverse are the caller's 16-bit copies, and the
    oracle takes those same 16-bit values (exactly, in float64).
  - Norm: the same fp32 pairwise norm as the Walsh-Hadamard path; stored fp16.
  - Code = #{k : t_k < z}, t_k = fl32(0.5 fl32(c_k + c_k+1)), z = (Pi x)_j / n32;
    the GPU takes z in fp32 from an fp32 accumulation, so the tests accept
    either neighbour when z lies within the accumulation bound of a t_k.
  - Reconstruction x^ = n16 * (Pi^T c), rounded once to the output dtype.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import betaincc, gammaln

from . import F16, gauss, pack_codes, unpack_codes


# ---------------------------------------------------------------- the law

def beta_density(t, d: int):
    """f_d(t): density of one coordinate of a uniform unit vector in R^d."""
    t = np.asarray(t, np.float64)
    logc = gammaln(d / 2.0) - 0.5 * math.log(math.pi) - gammaln((d - 1) / 2.0)
    with np.errstate(divide="ignore"):
        return np.where(np.abs(t) < 1.0, np.exp(logc + (d - 3) / 2.0 * np.log1p(-t * t)), 0.0)


def beta_upper_tail(t, d: int):
    """P(T > t) for t >= 0: half the upper regularized incomplete beta of t^2."""
    t = np.asarray(t, np.float64)
    return 0.5 * betaincc(0.5, (d - 1) / 2.0, np.minimum(t * t, 1.0))


def beta_first_moment(a, b, d: int):
    """Integral of t f_d(t) over [a, b] in closed form:
    d/dt (1 - t^2)^((d-1)/2) = -(d-1) t (1 - t^2)^((d-3)/2)."""
    logc = gammaln(d / 2.0) - 0.5 * math.log(math.pi) - gammaln((d - 1) / 2.0)
    k = (d - 1) / 2.0
    g = lambda t: np.power(np.maximum(1.0 - np.minimum(np.asarray(t, np.float64) ** 2, 1.0), 0.0), k)
    return math.exp(logc) * (g(a) - g(b)) / (2.0 * k)


def beta_lloyd_max(d: int, bits: int, max_iters: int = 200000) -> np.ndarray:
    """Lloyd-Max centroids of f_d at `bits` bits (ascending, float64, exactly
    symmetric): boundaries at midpoints, centroids at the cells' conditional
    means, iterated from a uniform start until no centroid moves by more than
    a few ulps.  Only the upper half is iterated (the middle boundary is 0); a
    cell's mass is a difference of upper tails, so tail cells keep their
    relative precision."""
    K = 1 << bits
    h = K // 2
    c = (np.arange(h) + 0.5) / h * min(1.0, 3.0 / math.sqrt(d))      # upper-half start
    for _ in range(max_iters):
        t = np.concatenate([[0.0], 0.5 * (c[:-1] + c[1:]), [1.0]])
        mass = beta_upper_tail(t[:-1], d) - beta_upper_tail(t[1:], d)
        new = beta_first_moment(t[:-1], t[1:], d) / mass
        done = np.max(np.abs(new - c)) <= 8.0 * np.finfo(np.float64).eps * np.max(np.abs(new))
        c = new
        if done:                                         # moves of a few ulps: the float64 limit
            break
    return np.concatenate([-c[::-1], c])


# ---------------------------------------------------------------- Pi

def gaussian_matrix(seed: int, d: int) -> np.ndarray:
    G = np.empty((d, d), np.float64)
    for i in range(d):
        for j in range(d):
            G[i, j] = gauss(seed, i * d + j)
    return G


def rotation(seed: int, d: int) -> np.ndarray:
    """Pi = Q diag(sign(diag R)), G = Q R (numpy's Householder QR)."""
    G = gaussian_matrix(seed, d)
    Q, R = np.linalg.qr(G)
    s = np.sign(np.diag(R))
    s[s == 0] = 1.0
    return Q * s[None, :]


def to16(a: np.ndarray, dtype: int) -> np.ndarray:
    """float64 -> float32 -> 16-bit patterns (round to nearest even)."""
    f = np.asarray(a, np.float32).reshape(-1)
    if dtype == F16:
        return f.astype(np.float16).view(np.uint16).reshape(np.shape(a))
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    return r.reshape(np.shape(a))


def from16(h: np.ndarray, dtype: int) -> np.ndarray:
    h = np.asarray(h, np.uint16)
    if dtype == F16:
        return h.view(np.float16).astype(np.float64)
    return (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- quantize

def norm_f32(x: np.ndarray) -> np.ndarray:
    """Pairwise fp32 norm of each row (leaves (2k, 2k+1), recursive halving)."""
    s = (x.astype(np.float32) * x.astype(np.float32)).astype(np.float32)
    while s.shape[1] > 1:
        s = (s[:, 0::2] + s[:, 1::2]).astype(np.float32)
    return np.sqrt(s[:, 0]).astype(np.float32)


def norm_to_f16(n32: np.ndarray) -> np.ndarray:
    return np.minimum(n32.astype(np.float32), np.float32(65504.0)).astype(np.float16).view(np.uint16)


def boundaries32(c32: np.ndarray) -> np.ndarray:
    c32 = np.asarray(c32, np.float32)
    return (np.float32(0.5) * (c32[:-1] + c32[1:]).astype(np.float32)).astype(np.float32)


def quantize(x16, dtype: int, d: int, Pi16, bits: int, layout: int, c32):
    """-> (codes uint8, norms fp16 bits, z float64 [nb, d], n32 fp32)."""
    x = from16(np.asarray(x16, np.uint16).reshape(-1, d), dtype)
    Pi = from16(np.asarray(Pi16, np.uint16).reshape(d, d), dtype)
    n32 = norm_f32(x)
    y = x @ Pi.T                                          # y[b, j] = sum_i Pi[j, i] x[b, i]
    with np.errstate(divide="ignore", invalid="ignore"):
        z = np.where(n32[:, None] > 0, y / n32[:, None].astype(np.float64), 0.0)
    t = boundaries32(c32).astype(np.float64)
    idx = np.searchsorted(t, z, side="left").astype(np.uint8)   # #{k : t_k < z}
    codes = pack_codes(idx.reshape(-1), d, bits, layout)
    return codes, norm_to_f16(n32), z, n32


def dequantize(codes, norms16, nblocks: int, d: int, Pi16, bits: int, layout: int, cop16, out_dtype: int,
               op_dtype: int):
    """x^ = n16 * Pi^T c with c the 16-bit centroid operand `cop16` (patterns in
    op_dtype); returns (out 16-bit patterns, float64 value before rounding)."""
    idx = unpack_codes(codes, nblocks, d, bits, layout).reshape(nblocks, d)
    c = from16(cop16, op_dtype)[idx]
    Pi = from16(np.asarray(Pi16, np.uint16).reshape(d, d), op_dtype)
    n16 = np.asarray(norms16, np.uint16).view(np.float16).astype(np.float64)
    v = n16[:, None] * (c @ Pi)                            # (Pi^T c)_i = sum_j Pi[j, i] c_j
    return to16(v, out_dtype), v
