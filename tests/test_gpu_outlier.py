"""qjl_sketch_outlier / qjl_score_outlier on the GPU against the outlier-sketch
oracle (QJL README "Algorithm in one paragraph"; qjl_apply.py key hook).

Bars:
- outlier indices, ||k_in|| and ||k_out||: bit-exact (the same fp32 sums in
  the same order on both sides);
- sign bits of both sketches: equal except within the 1e-5 window of the
  existing key sketch (|P| / ||v|| <= 1e-5, reading of the tensor-core sums);
- scores: within 1e-3 * ||q|| * (||k_in|| + ||k_out||), the estimator's scale
  (the bar of the plain score, per term).
"""
import numpy as np
import pytest
import torch

from oracle import outlier_sketch as X
from kv_quantization_b200 import _lib as L
from kv_quantization_b200 import synth
from tests.gpu_checks import DEV, check_signs, report, u16

pytestmark = pytest.mark.gpu

d = 128


def bf16_values(t):
    return (u16(t).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def run(G, T, m, m_o, n_out, seed):
    k = synth.kv_with_channels(1, G, T, d, seed=seed, device=DEV).reshape(-1)
    S = torch.empty(m, d, dtype=torch.bfloat16, device=DEV)
    L.qjl_make_projection(seed + 1, m, d, S)
    nv = G * T
    signs = torch.empty(nv * m // 8, dtype=torch.uint8, device=DEV)
    norms = torch.empty(nv, dtype=torch.int16, device=DEV)
    oidx = torch.empty(nv // 32 * n_out + 16, dtype=torch.uint8, device=DEV)
    osg = torch.empty(nv * m_o // 8, dtype=torch.uint8, device=DEV)
    onr = torch.empty(nv, dtype=torch.int16, device=DEV)
    ws = torch.empty(L.qjl_sketch_outlier_workspace_bytes(nv, d), dtype=torch.uint8, device=DEV)
    L.qjl_sketch_outlier(k, d, m, S, m_o, n_out, signs, norms, oidx, osg, onr, ws)
    torch.cuda.synchronize()
    trace = L.rq_last_launch()
    assert "outlier_prep_kernel" in trace and "sketch" in trace, trace
    return dict(k=k, S=S, signs=signs, norms=norms, oidx=oidx, osg=osg, onr=onr, nv=nv)


@pytest.mark.parametrize("G,T,m,m_o,n_out", [(3, 96, 256, 256, 8), (2, 64, 256, 128, 8), (2, 160, 128, 64, 16),
                                             (1, 32, 64, 32, 1)])
def test_outlier_sketch_matches_oracle(G, T, m, m_o, n_out):
    r = run(G, T, m, m_o, n_out, seed=G * 7 + n_out)
    kv = bf16_values(r["k"]).reshape(G, T, d)
    Sv = bf16_values(r["S"]).reshape(m, d)
    o = X.sketch(kv, Sv, m_o, n_out)
    nv = r["nv"]
    np.testing.assert_array_equal(r["oidx"].cpu().numpy()[: nv // 32 * n_out].reshape(G, T // 32, n_out), o["idx"])
    np.testing.assert_array_equal(r["onr"].cpu().numpy().view(np.uint16), o["norms_out"].reshape(-1))
    np.testing.assert_array_equal(r["norms"].cpu().numpy().view(np.uint16), o["norms_in"].reshape(-1))
    k_in, k_out = X.split(kv, o["idx"])
    n_in = np.linalg.norm(k_in, axis=-1, keepdims=True)
    n_o = np.linalg.norm(k_out, axis=-1, keepdims=True)
    with np.errstate(invalid="ignore", divide="ignore"):
        p_in = np.where(n_in > 0, o["p_in"] / n_in, 0.0).reshape(-1)
        p_out = np.where(n_o > 0, o["p_out"] / n_o, 0.0).reshape(-1)
    check_signs(r["signs"].cpu().numpy(), X.pack_signs(o["signs_in"]).reshape(-1), p_in, nv, m)
    check_signs(r["osg"].cpu().numpy(), X.pack_signs(o["signs_out"]).reshape(-1), p_out, nv, m_o)
    report("outlier_sketch", G=G, T=T, m=m, m_o=m_o, n_out=n_out)


@pytest.mark.parametrize("G,T,m,m_o,n_out,nq", [(3, 96, 256, 256, 8, 32), (2, 160, 128, 64, 16, 5),
                                                (2, 64, 256, 128, 8, 40)])
def test_outlier_score_matches_oracle(G, T, m, m_o, n_out, nq):
    r = run(G, T, m, m_o, n_out, seed=G * 11 + nq)
    q = synth.normal((G, nq, d), seed=nq, device=DEV)
    scores = torch.empty(G, nq, T, dtype=torch.float32, device=DEV)
    ws = torch.empty(L.qjl_score_workspace_bytes(G, nq, d, m) // 4 + 4, dtype=torch.float32, device=DEV)
    L.qjl_score_outlier(q, G, nq, d, m, r["S"], r["signs"], r["norms"], T, m_o, n_out, r["oidx"], r["osg"], r["onr"],
                        scores, ws)
    torch.cuda.synchronize()
    assert "outlier_score_kernel" in L.rq_last_launch()
    # the oracle's score of the GPU's own sketch bits (the sketch is compared above)
    Sv = bf16_values(r["S"]).reshape(m, d)
    qv = bf16_values(q).reshape(G, nq, d)
    idx = r["oidx"].cpu().numpy()[: G * T // 32 * n_out].reshape(G, T // 32, n_out)
    s_in = X.unpack_signs(r["signs"].cpu().numpy().reshape(G, T, m // 8), m)
    s_out = X.unpack_signs(r["osg"].cpu().numpy().reshape(G, T, m_o // 8), m_o)
    n_in = r["norms"].cpu().numpy().view(np.uint16).reshape(G, T)
    n_out16 = r["onr"].cpu().numpy().view(np.uint16).reshape(G, T)
    want = X.score(qv, Sv, m_o, idx, s_in, n_in, s_out, n_out16)
    got = scores.cpu().numpy().astype(np.float64)
    qn = np.linalg.norm(qv, axis=-1)[:, :, None]
    kn = (n_in.view(np.float16).astype(np.float64) + n_out16.view(np.float16).astype(np.float64))[:, None, :]
    err = np.abs(got - want) / (qn * kn + 1e-30)
    assert np.all(err <= 1e-3), float(err.max())
    report("outlier_score", G=G, T=T, m=m, m_o=m_o, n_out=n_out, nq=nq, max_err=float(err.max()))


def test_outlier_score_full_kv_sampled():
    # the KV key workload (32 heads x 32768 tokens, m = 256, m_o = 256, 8
    # outliers per 32 tokens), end to end; 2 heads' scores against the oracle
    G, T, m, m_o, n_out, nq = 32, 32768, 256, 256, 8, 32
    r = run(G, T, m, m_o, n_out, seed=3)
    q = synth.normal((G, nq, d), seed=5, device=DEV)
    scores = torch.empty(G, nq, T, dtype=torch.float32, device=DEV)
    ws = torch.empty(L.qjl_score_workspace_bytes(G, nq, d, m) // 4 + 4, dtype=torch.float32, device=DEV)
    L.qjl_score_outlier(q, G, nq, d, m, r["S"], r["signs"], r["norms"], T, m_o, n_out, r["oidx"], r["osg"], r["onr"],
                        scores, ws)
    torch.cuda.synchronize()
    Sv = bf16_values(r["S"]).reshape(m, d)
    for g in (0, G - 1):
        kv = bf16_values(r["k"].reshape(G, T, d)[g:g + 1, :4096].contiguous()).reshape(1, 4096, d)
        o = X.sketch(kv, Sv, m_o, n_out)
        idx = r["oidx"].cpu().numpy()[: G * T // 32 * n_out].reshape(G, T // 32, n_out)[g:g + 1, :128]
        np.testing.assert_array_equal(idx, o["idx"])
        s_in = X.unpack_signs(r["signs"].cpu().numpy().reshape(G, T, m // 8)[g:g + 1, :4096], m)
        s_out = X.unpack_signs(r["osg"].cpu().numpy().reshape(G, T, m_o // 8)[g:g + 1, :4096], m_o)
        n_in = r["norms"].cpu().numpy().view(np.uint16).reshape(G, T)[g:g + 1, :4096]
        n_o = r["onr"].cpu().numpy().view(np.uint16).reshape(G, T)[g:g + 1, :4096]
        np.testing.assert_array_equal(n_o, o["norms_out"])
        qv = bf16_values(q[g:g + 1].contiguous()).reshape(1, nq, d)
        want = X.score(qv, Sv, m_o, idx, s_in, n_in, s_out, n_o)
        got = scores[g:g + 1, :, :4096].cpu().numpy().astype(np.float64)
        qn = np.linalg.norm(qv, axis=-1)[:, :, None]
        kn = (n_in.view(np.float16).astype(np.float64) + n_o.view(np.float16).astype(np.float64))[:, None, :]
        assert np.all(np.abs(got - want) <= 1e-3 * qn * kn)
    report("outlier_full_kv", G=G, T=T)
