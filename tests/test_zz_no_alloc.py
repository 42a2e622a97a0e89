"""qjl_score_noalloc: the score entry point for callers that cannot allocate
device memory (its scratch is a fixed array in the library's device image).

Collected last on purpose: if it fails, a run that stops at the first failure
has already run every other test.  It must pass both alone in a fresh process
and after the other tests (the array keeps whatever the previous call left)."""
import numpy as np
import pytest
import torch

from kv_quantization_b200 import _lib as L
from kv_quantization_b200 import synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _keys(G, T, d, m, bits):
    k = synth.normal((G, T, d), seed=31, device=DEV).reshape(-1)
    cent = L.rq_lloyd_max(bits)
    S = torch.empty(m, d, dtype=torch.bfloat16, device=DEV)
    L.qjl_make_projection(6, m, d, S)
    codes = torch.empty(L.rq_code_bytes(k.numel(), d, bits, L.RQ_CODES_PACKED), dtype=torch.uint8, device=DEV)
    norms = torch.empty(G * T, dtype=torch.int16, device=DEV)
    qs = torch.empty(G * T * m // 8, dtype=torch.uint8, device=DEV)
    qn = torch.empty(G * T, dtype=torch.int16, device=DEV)
    L.rq_quantize_qjl(k, d, bits, L.RQ_CODES_PACKED, 1, 12, cent, m, S, codes, norms, qs, qn)
    return cent, S, codes, norms, qs, qn


def test_noalloc_score_matches_workspace_score_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    G, T, d, m, bits, nq = 4, 300, 128, 128, 2, 32
    cent, S, codes, norms, qs, qn = _keys(G, T, d, m, bits)
    kw = dict(codes=codes, norms=norms, bits=bits, layout=L.RQ_CODES_PACKED, use_signs=1, sign_seed=12,
              centroids=cent)
    # two calls in a row with different queries: the second must not see the first's leftovers
    for seed in (40, 41):
        q = synth.normal((G, nq, d), seed=seed, device=DEV)
        ref = torch.empty(G, nq, T, dtype=torch.float32, device=DEV)
        ws = torch.empty(L.qjl_score_workspace_bytes(G, nq, d, m) // 4 + 1, dtype=torch.float32, device=DEV)
        L.qjl_score(q, G, nq, d, m, S, qs, qn, T, ref, ws, **kw)
        got = torch.full((G, nq, T), float("nan"), dtype=torch.float32, device=DEV)
        L.qjl_score_noalloc(q, G, nq, d, m, S, qs, qn, T, got, **kw)
        torch.cuda.synchronize()
        qf = q.float().cpu().numpy().astype(np.float64)
        nrm = np.array(norms.cpu().numpy().view(np.float16), np.float64).reshape(G, 1, T)
        rnm = np.array(qn.cpu().numpy().view(np.float16), np.float64).reshape(G, 1, T)
        tol = 1e-3 * np.linalg.norm(qf, axis=2)[:, :, None] * (nrm + rnm)
        err = np.abs(got.cpu().numpy().astype(np.float64) - ref.cpu().numpy().astype(np.float64))
        assert np.all(np.isfinite(got.cpu().numpy()))
        assert np.all(err <= tol)
    assert L.rq_device_error(True) == 0


def test_noalloc_rejects_oversized_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    G, nq, d, m = 4096, 128, 512, 512                 # needs far more than 8 MiB
    assert L.qjl_score_workspace_bytes(G, nq, d, m) > (8 << 20)
    t = torch.empty(16, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(L.RQError) as e:
        L.qjl_score_noalloc(t, G, nq, d, m, t, t, t, 1000, torch.empty(4, device=DEV))
    assert e.value.status == -3
