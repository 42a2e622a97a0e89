"""Pins of the outlier-sketch oracle (QJL README "Algorithm in one paragraph";
qjl_apply.py key hook: per group of 32 tokens, the top-k coordinates by group
norm get their own sketch) against facts that do not come from the oracle:
the decomposition k = k_in + k_out, brute-force top-k, the reduction to the
plain QJL estimator of the C oracle, unbiasedness and the variance it saves."""
import math

import numpy as np
import pytest

import oracle as O
from oracle import outlier_sketch as X


def keys_with_outliers(G, T, d, seed, n_hot=6, mult=10.0):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((G, T, d))
    for g in range(G):
        hot = rng.choice(d, n_hot, replace=False)
        k[g][:, hot] *= mult
    return D16(k)


def D16(a):
    """Round to bf16 values (as float64)."""
    f = np.asarray(a, np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint32) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def test_split_is_a_partition_of_each_key():
    k = keys_with_outliers(2, 64, 32, 1)
    idx = X.outlier_indices(k, 5)
    assert idx.shape == (2, 2, 5)
    for g in range(2):
        for j in range(2):
            assert len(set(idx[g, j].tolist())) == 5
    k_in, k_out = X.split(k, idx)
    np.testing.assert_array_equal(k_in + k_out, k)
    assert not np.any((k_in != 0) & (k_out != 0))
    for g in range(2):
        for j in range(2):
            rows = slice(32 * j, 32 * j + 32)
            outside = np.setdiff1d(np.arange(32), idx[g, j])
            assert np.all(k_out[g, rows][:, outside] == 0)
            assert np.all(k_in[g, rows][:, idx[g, j]] == 0)


def test_top_k_is_the_largest_group_norms():
    # brute force: fp64 column norms over each group of 32 tokens; scales
    # spread so that no two columns come within rounding of each other
    rng = np.random.default_rng(2)
    G, T, d = 3, 96, 64
    scale = np.exp(rng.uniform(0, 3, (G, T // 32, d)))
    k = D16(rng.standard_normal((G, T, d)) * np.repeat(scale, 32, axis=1))
    idx = X.outlier_indices(k, 8)
    for g in range(G):
        for j in range(T // 32):
            nrm = np.sqrt(np.sum(k[g, 32 * j:32 * j + 32] ** 2, axis=0))
            want = np.argsort(-nrm, kind="stable")[:8]
            np.testing.assert_array_equal(idx[g, j], want)


def test_ties_go_to_the_lower_index():
    k = np.ones((1, 32, 16))
    np.testing.assert_array_equal(X.outlier_indices(k, 4)[0, 0], [0, 1, 2, 3])


def _plain_qjl_c_oracle(q, k, S, m):
    """The C oracle's pure-QJL score (sketch + norms from 16-bit keys)."""
    G, T, d = k.shape
    nq = q.shape[1]
    k16 = X_bits(k)
    S16 = X_bits(S)
    signs, _ = O.sketch(k16.reshape(-1), O.BF16, d, m, S16.reshape(m, d))
    norms = O.vec_norms(k16.reshape(-1), O.BF16, d)
    q16 = X_bits(q).reshape(-1)
    return O.score(q16, G, nq, d, m, S16.reshape(m, d), O.BF16, signs, norms, T).reshape(G, nq, T)


def X_bits(a):
    return (np.asarray(a, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_no_outliers_is_the_plain_qjl_estimator():
    G, T, d, m, nq = 2, 64, 64, 64, 3
    k = keys_with_outliers(G, T, d, 3)
    q = D16(np.random.default_rng(4).standard_normal((G, nq, d)))
    S = D16(np.random.default_rng(5).standard_normal((m, d)))
    r = X.sketch(k, S, 16, 0)
    got = X.score(q, S, 16, r["idx"], r["signs_in"], r["norms_in"], r["signs_out"], r["norms_out"])
    want = _plain_qjl_c_oracle(q, k, S, m)
    np.testing.assert_allclose(got, want, rtol=1e-9, atol=1e-9 * np.max(np.abs(want)))


def test_keys_inside_or_outside_the_outlier_set():
    G, T, d, m, nq, n_out = 1, 32, 32, 64, 2, 4
    rng = np.random.default_rng(6)
    q = D16(rng.standard_normal((G, nq, d)))
    S = D16(rng.standard_normal((m, d)))
    # every key zero off coordinates 0..3 (made the largest): no inlier part
    k = np.zeros((G, T, d))
    k[0, :, :4] = D16(rng.standard_normal((T, 4)) * 5)
    r = X.sketch(k, S, m, n_out)
    assert set(r["idx"][0, 0].tolist()) == {0, 1, 2, 3}
    assert np.all(r["norms_in"] == 0)
    got = X.score(q, S, m, r["idx"], r["signs_in"], r["norms_in"], r["signs_out"], r["norms_out"])
    c = math.sqrt(math.pi / 2) / m
    qo = np.zeros_like(q)
    qo[0][:, :4] = q[0][:, :4]
    n_o = r["norms_out"].view(np.float16).astype(np.float64)
    want = c * n_o[:, None, :] * np.einsum("gqm,gtm->gqt", qo @ S.T, 2.0 * r["signs_out"] - 1.0)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_unbiased_over_projections():
    # E over S of the estimator equals <q, k> (Monte Carlo, 4 sigma)
    d, m, m_o, n_out, trials = 32, 64, 64, 4, 3000
    rng = np.random.default_rng(7)
    k = keys_with_outliers(1, 32, d, 8, n_hot=3, mult=8.0)
    q = D16(rng.standard_normal((1, 1, d)))
    true = (q[0] @ k[0].T)[0]
    est = np.zeros((trials, 32))
    for i in range(trials):
        S = rng.standard_normal((m, d))
        r = X.sketch(k, S, m_o, n_out)
        n_in = X.pairwise_norm_f32(X.split(k, r["idx"])[0])
        est[i] = X.score(q, S, m_o, r["idx"], r["signs_in"], X.f32_to_f16_bits(n_in), r["signs_out"],
                         r["norms_out"])[0, 0]
    se = est.std(axis=0) / math.sqrt(trials)
    # fp16 norms bias each term by at most 2^-11 relative
    assert np.all(np.abs(est.mean(axis=0) - true) < 4 * se + 2e-3 * np.abs(true) + 1e-9)


def test_outlier_sketch_lowers_the_variance_on_outlier_channels():
    # keys with a few hot channels and a query with no weight on them: the
    # plain estimator's variance grows with ||q||^2 ||k||^2, the split one's
    # with ||q||^2 ||k_in||^2 (the outlier term sees q_O = 0 and vanishes)
    d, m, trials = 64, 64, 1500
    rng = np.random.default_rng(9)
    k = keys_with_outliers(1, 32, d, 10, n_hot=4, mult=12.0)
    hot = X.outlier_indices(k, 4)[0, 0]
    q = rng.standard_normal((1, 1, d))
    q[0, 0, hot] = 0.0
    q = D16(q)
    var = []
    for n_out in (0, 4):
        est = np.zeros((trials, 32))
        for i in range(trials):
            S = rng.standard_normal((m, d))
            r = X.sketch(k, S, m, n_out)
            est[i] = X.score(q, S, m, r["idx"], r["signs_in"], r["norms_in"], r["signs_out"], r["norms_out"])[0, 0]
        var.append(est.var(axis=0).mean())
    assert var[1] < 0.25 * var[0], var
