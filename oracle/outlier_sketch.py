"""CPU oracle for the QJL key sketch with a per-group outlier sketch.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg may import this module; it never imports the
product library.  Plain numpy, float64 unless stated.

Sources followed:
  - eliza "scripts/quantization" README, section "QJL", "Algorithm in one
    paragraph": a 1-bit JL sketch of each key plus its norm; outlier
    coordinates (a few indices with disproportionately large norms) get a
    top-k sketch per group of group_size consecutive tokens, with its own JL
    projection of dimension dim_outlier; the query goes through the same
    projection and the score is the unbiased estimator;
  - the same README's knobs: group size 32, outlier count 8 per group;
  - qjl_apply.py, `attach_qjl_to_cache`'s key hook: per group, the norm of
    every coordinate over the group's tokens, the top `outlier_count`
    coordinates of it as uint8 indices, one projection matrix passed to the
    quantizer together with `outlier_sketch_dim`, and per-token full-key
    norms.

Readings where the pages leave a step open (listed in the design notes too):
  - The key splits into k_in (k with the group's outlier coordinates O set to
    zero) and k_out (k on O, zero elsewhere).  The main sketch is
    sign(S k_in) with ||k_in||; the outlier sketch is sign(S_o k_out) with
    ||k_out||, where S_o = the first m_o rows of the one projection S (the
    quantizer receives a single matrix and the outlier dimension).
  - Score = sqrt(pi/2)/m ||k_in|| <S q, sign(S k_in)>
          + sqrt(pi/2)/m_o ||k_out|| <S_o q_O, sign(S_o k_out)>,
    q_O the query on O (zero elsewhere): each term is the QJL estimator of
    <q, k_in> and of <q_O, k_out> = <q, k_out>, so the sum is unbiased for
    <q, k>, and restricting the query to O in the outlier term is what makes
    the per-group index table part of the score.
  - Group ranking: per coordinate the fp32 sum of squares over the group's 32
    tokens in token order; the top k by that sum, ties to the lower index;
    stored in that order (largest first).
  - Norms: ||k_in|| the canonical fp32 pairwise norm of the masked key;
    ||k_out|| the fp32 sum of squares of the k outlier values in stored order,
    correctly rounded square root; both stored fp16.  Sign bit = (P >= 0).
"""
from __future__ import annotations

import math

import numpy as np

GROUP = 32


def f32_to_f16_bits(v):
    return np.minimum(np.asarray(v, np.float32), np.float32(65504.0)).astype(np.float16).view(np.uint16)


def outlier_indices(keys: np.ndarray, n_out: int) -> np.ndarray:
    """keys float (exact 16-bit values) [G][T][d] -> uint8 [G][T/32][n_out]."""
    G, T, d = keys.shape
    k32 = keys.astype(np.float32).reshape(G, T // GROUP, GROUP, d)
    s = np.zeros((G, T // GROUP, d), np.float32)
    for t in range(GROUP):                                   # token order, fp32
        s = (s + (k32[:, :, t, :] * k32[:, :, t, :]).astype(np.float32)).astype(np.float32)
    # descending sum, ties to the lower index: a stable sort on (-s)
    order = np.argsort(-s.astype(np.float64), axis=-1, kind="stable")
    return order[..., :n_out].astype(np.uint8)


def pairwise_norm_f32(x: np.ndarray) -> np.ndarray:
    s = (x.astype(np.float32) * x.astype(np.float32)).astype(np.float32)
    while s.shape[-1] > 1:
        s = (s[..., 0::2] + s[..., 1::2]).astype(np.float32)
    return np.sqrt(s[..., 0]).astype(np.float32)


def split(keys: np.ndarray, idx: np.ndarray):
    """(k_in, k_out) float64 [G][T][d] for the group index table idx."""
    G, T, d = keys.shape
    mask = np.zeros((G, T // GROUP, d), bool)
    gi, ji = np.meshgrid(np.arange(G), np.arange(T // GROUP), indexing="ij")
    for r in range(idx.shape[-1]):
        mask[gi, ji, idx[..., r]] = True
    mask = np.repeat(mask, GROUP, axis=1)
    k = keys.astype(np.float64)
    return np.where(mask, 0.0, k), np.where(mask, k, 0.0)


def sketch(keys: np.ndarray, S: np.ndarray, m_o: int, n_out: int):
    """keys [G][T][d] (exact 16-bit values as float), S [m][d] (exact values).
    Returns dict: idx, signs_in (bool [G][T][m]), p_in, norms_in (fp16 bits),
    signs_out (bool [G][T][m_o]), p_out, norms_out (fp16 bits)."""
    G, T, d = keys.shape
    idx = outlier_indices(keys, n_out)
    k_in, k_out = split(keys, idx)
    p_in = k_in @ S.T
    p_out = k_out @ S[:m_o].T
    n_in = pairwise_norm_f32(k_in)
    # ||k_out||: fp32 squares of the outlier values in stored order
    k32 = keys.astype(np.float32).reshape(G, T // GROUP, GROUP, d)
    acc = np.zeros((G, T // GROUP, GROUP), np.float32)
    for r in range(n_out):
        v = np.take_along_axis(k32, idx[:, :, None, r:r + 1].astype(np.int64).repeat(GROUP, 2), axis=3)[..., 0]
        acc = (acc + (v * v).astype(np.float32)).astype(np.float32)
    n_out32 = np.sqrt(acc).astype(np.float32).reshape(G, T)
    return dict(idx=idx, p_in=p_in, signs_in=p_in >= 0, norms_in=f32_to_f16_bits(n_in), p_out=p_out,
                signs_out=p_out >= 0, norms_out=f32_to_f16_bits(n_out32))


def pack_signs(bits: np.ndarray) -> np.ndarray:
    """bool [..., m] -> uint8 [..., m/8], bit j of byte b = sign of coordinate 8b + j."""
    return np.packbits(bits.astype(np.uint8), axis=-1, bitorder="little")


def unpack_signs(packed: np.ndarray, m: int) -> np.ndarray:
    return np.unpackbits(np.asarray(packed, np.uint8), axis=-1, count=m, bitorder="little").astype(bool)


def score(q: np.ndarray, S: np.ndarray, m_o: int, idx, signs_in, norms_in, signs_out, norms_out):
    """q [G][nq][d] (exact values), signs as bool arrays, norms fp16 bits.
    Returns float64 scores [G][nq][T]."""
    G, nq, d = q.shape
    m = S.shape[0]
    T = signs_in.shape[1]
    c = math.sqrt(math.pi / 2.0)
    n_in = np.asarray(norms_in, np.uint16).view(np.float16).astype(np.float64)
    n_o = np.asarray(norms_out, np.uint16).view(np.float16).astype(np.float64)
    sq = q.astype(np.float64) @ S.T                           # [G][nq][m]
    s_in = 2.0 * signs_in.astype(np.float64) - 1.0            # [G][T][m]
    out = c / m * n_in[:, None, :] * np.einsum("gqm,gtm->gqt", sq, s_in)
    s_o = 2.0 * signs_out.astype(np.float64) - 1.0            # [G][T][m_o]
    for j in range(T // GROUP):
        O = idx[:, j, :].astype(np.int64)                     # [G][k]
        qo = np.zeros_like(q, dtype=np.float64)
        for g in range(G):
            qo[g][:, O[g]] = q[g][:, O[g]]
        u = qo @ S[:m_o].T                                    # [G][nq][m_o]
        sl = slice(j * GROUP, (j + 1) * GROUP)
        out[:, :, sl] += c / m_o * n_o[:, None, sl] * np.einsum("gqm,gtm->gqt", u, s_o[:, sl, :])
    return out
