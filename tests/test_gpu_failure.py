"""The bounded-wait failure path, made to run on purpose without faulting or
hanging the GPU: rq_probe_bounded_wait enqueues one CTA that waits with a
short poll limit on an mbarrier nothing arrives on (no copy or MMA in flight),
records RQ_EDEVICE, frees its tensor memory and returns.  The test checks that
the call returns, that the error word reports the expiry and clears, and that
the device then still computes correct results."""
import numpy as np
import pytest
import torch

import oracle as O
from kv_quantization_b200 import _lib as L
from kv_quantization_b200 import synth
from tests.gpu_checks import DEV, check_scores, score_tol, u16

pytestmark = pytest.mark.gpu

RQ_EDEVICE = -6


def test_expired_wait_is_reported_and_device_stays_usable():
    torch.cuda.synchronize()
    assert L.rq_device_error(True) == 0
    for polls in (1, 1 << 12):
        L.rq_probe_bounded_wait(polls)
        assert L.rq_last_launch() == "bounded_wait_probe_kernel"
        torch.cuda.synchronize()                       # the probe returned instead of hanging
        assert L.rq_device_error(False) == RQ_EDEVICE  # reported ...
        assert L.rq_device_error(True) == RQ_EDEVICE   # ... until cleared
        assert L.rq_device_error(False) == 0
    # the context is intact: a quantize -> sketch -> score pass matches the oracle
    G, T, d, m, bits, nq = 2, 300, 128, 128, 3, 32
    k = synth.normal((G, T, d), seed=71, device=DEV).reshape(-1)
    q = synth.normal((G, nq, d), seed=72, device=DEV)
    cent = L.rq_lloyd_max(bits)
    S = torch.empty(m, d, dtype=torch.bfloat16, device=DEV)
    L.qjl_make_projection(73, m, d, S)
    codes = torch.empty(L.rq_code_bytes(k.numel(), d, bits, L.RQ_CODES_PACKED), dtype=torch.uint8, device=DEV)
    norms = torch.empty(G * T, dtype=torch.int16, device=DEV)
    qs = torch.empty(G * T * m // 8, dtype=torch.uint8, device=DEV)
    qn = torch.empty(G * T, dtype=torch.int16, device=DEV)
    L.rq_quantize_qjl(k, d, bits, L.RQ_CODES_PACKED, 1, 74, cent, m, S, codes, norms, qs, qn)
    scores = torch.empty(G, nq, T, dtype=torch.float32, device=DEV)
    ws = torch.empty(L.qjl_score_workspace_bytes(G, nq, d, m) // 4, dtype=torch.float32, device=DEV)
    L.qjl_score(q, G, nq, d, m, S, qs, qn, T, scores, ws, codes=codes, norms=norms, bits=bits,
                layout=L.RQ_CODES_PACKED, use_signs=1, sign_seed=74, centroids=cent)
    torch.cuda.synchronize()
    assert L.rq_device_error(True) == 0
    k16, q16 = u16(k), u16(q)
    sd = O.sign_diagonal(74, d)
    oc, on, _, _ = O.quantize(k16, O.BF16, d, bits, O.PACKED, sd, cent)
    assert np.array_equal(codes.cpu().numpy(), oc)
    assert np.array_equal(norms.cpu().numpy().view(np.uint16), on)
    want = O.score(q16, G, nq, d, m, u16(S), O.BF16, qs.cpu().numpy(), qn.cpu().numpy().view(np.uint16), T,
                   codes=oc, norms=on, bits=bits, layout=O.PACKED, signs_diag=sd, c32=cent)
    check_scores(scores.cpu().numpy(), want, score_tol(q16, G, nq, d, on.reshape(G, T)), "after expired wait")


def test_probe_rejects_out_of_range_limits():
    for polls in (0, (1 << 20) + 1):
        with pytest.raises(L.RQError) as e:
            L.rq_probe_bounded_wait(polls)
        assert e.value.status == -1
        assert L.rq_last_launch() == ""
