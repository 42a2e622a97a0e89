"""qjl_attention on the GPU against the oracle's attention (softmax of the
estimator scores applied to the fp64 value reconstructions).

Bars (from the arithmetic of the kernel; the oracle is fp64):
- every output coordinate within tol_q = (2 (e^(2 e_q) - 1) + 2^-9) V_q,
  V_q = max_t ||vh_t||_2 over the group's values, e_q = 1e-3 max_t |a_qt| the
  logit error the score's 1e-3 relative bar allows (a = scale * score): a
  relative weight error of at most e^(2 e_q) - 1 moves a convex combination by
  at most twice that times the spread of the values, and 2^-9 covers the two
  fp16 roundings of each product (the weight 2^14 p and the value
  c * (n / d), 2^-11 each) carried through the rotation;
- and, over all outputs of a case, ||got - want|| / ||want|| <= 2e-3 (the
  fp16 roundings, uncorrelated across tokens and coordinates).
Cases where the weights are exact (one key, equal keys, a hard maximum) use
2^-9 V_q alone.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from kv_quantization_b200 import _lib as L
from kv_quantization_b200 import synth
from tests.gpu_checks import DEV, num_sms, report, u16

pytestmark = pytest.mark.gpu

KERNELS = "score_v2_prologue,attention_kernel,attention_combine_kernel"


def compress(G, T, d, m, kbits, vbits, seed, two_stage, vlayout=L.RQ_CODES_PACKED, k=None, v=None):
    """Keys (pure QJL sketch, or two-stage codes + residual sketch) and values
    (rotated Lloyd-Max codes) of G groups, compressed by the library."""
    if k is None:
        k = synth.kv_with_channels(1, G, T, d, seed=seed, device=DEV).reshape(-1)
    if v is None:
        v = synth.kv_with_channels(1, G, T, d, seed=seed + 1, device=DEV).reshape(-1)
    S = torch.empty(m, d, dtype=torch.bfloat16, device=DEV)
    L.qjl_make_projection(seed + 2, m, d, S)
    n = G * T
    out = dict(k=k, v=v, S=S)
    if two_stage:
        kc = L.rq_lloyd_max(kbits)
        codes = torch.empty(L.rq_code_bytes(n * d, d, kbits, L.RQ_CODES_PACKED), dtype=torch.uint8, device=DEV)
        norms = torch.empty(n, dtype=torch.int16, device=DEV)
        qs = torch.empty(n * m // 8, dtype=torch.uint8, device=DEV)
        qn = torch.empty(n, dtype=torch.int16, device=DEV)
        L.rq_quantize_qjl(k, d, kbits, L.RQ_CODES_PACKED, 1, seed + 3, kc, m, S, codes, norms, qs, qn)
        out.update(signs=qs, sk=qn, codes=codes, norms=norms, kc=kc, kseed=seed + 3)
    else:
        qs = torch.empty(n * m // 8, dtype=torch.uint8, device=DEV)
        kn = torch.empty(n, dtype=torch.int16, device=DEV)
        L.qjl_sketch(k, d, m, S, qs, kn)
        out.update(signs=qs, sk=kn, codes=None, norms=None, kc=None, kseed=0)
    vc = L.rq_lloyd_max(vbits)
    vcodes = torch.empty(L.rq_code_bytes(n * d, d, vbits, vlayout), dtype=torch.uint8, device=DEV)
    vnorms = torch.empty(n, dtype=torch.int16, device=DEV)
    L.rq_quantize(v, d, vbits, vlayout, 1, seed + 4, vc, vcodes, vnorms)
    out.update(vcodes=vcodes, vnorms=vnorms, vc=vc, vseed=seed + 4, vlayout=vlayout)
    return out


def run_attention(c, q, G, nq, d, m, T, kbits, vbits, scale):
    out = torch.empty(G, nq, d, dtype=torch.float32, device=DEV)
    ws = torch.empty((L.qjl_attention_workspace_bytes(G, nq, d, m, T) + 3) // 4, dtype=torch.float32, device=DEV)
    kw = {}
    if c["codes"] is not None:
        kw = dict(codes=c["codes"], norms=c["norms"], bits=kbits, layout=L.RQ_CODES_PACKED, use_signs=1,
                  sign_seed=c["kseed"], centroids=c["kc"])
    L.qjl_attention(q, G, nq, d, m, c["S"], c["signs"], c["sk"], T, c["vcodes"], c["vnorms"], vbits, c["vc"], out, ws,
                    scale, v_layout=c["vlayout"], v_use_signs=1, v_sign_seed=c["vseed"], **kw)
    assert L.rq_last_launch() == KERNELS
    torch.cuda.synchronize()
    assert L.rq_device_error(True) == 0
    return out.cpu().numpy().astype(np.float64)


def oracle_attention(c, q, G, nq, d, m, T, kbits, vbits, scale, groups=None):
    """O.attention on the library's compressed keys and values (bit-exact with
    the oracle's own compression, which the other test files check), for all
    groups or the listed ones; returns (out, logits, value reconstructions)."""
    groups = list(range(G)) if groups is None else list(groups)
    mb = m // 8
    q16 = u16(q).reshape(G, nq, d)
    S16 = u16(c["S"])
    sg = c["signs"].cpu().numpy().reshape(G, T, mb)
    sk = c["sk"].cpu().numpy().view(np.uint16).reshape(G, T)
    vcb = L.rq_code_bytes(d, d, vbits, c["vlayout"])
    vcodes = c["vcodes"].cpu().numpy().reshape(G, T, vcb)
    vnorms = c["vnorms"].cpu().numpy().view(np.uint16).reshape(G, T)
    vs = O.sign_diagonal(c["vseed"], d)
    olay = O.INT8 if c["vlayout"] == L.RQ_CODES_INT8 else O.PACKED
    if c["codes"] is not None:
        cb = L.rq_code_bytes(d, d, kbits, L.RQ_CODES_PACKED)
        codes = c["codes"].cpu().numpy().reshape(G, T, cb)
        norms = c["norms"].cpu().numpy().view(np.uint16).reshape(G, T)
        ks = O.sign_diagonal(c["kseed"], d)
    outs, logits, vhs = [], [], []
    for g in groups:
        kw = {}
        if c["codes"] is not None:
            kw = dict(codes=codes[g].reshape(-1), norms=norms[g], bits=kbits, layout=O.PACKED, signs_diag=ks,
                      c32=c["kc"])
        o = O.attention(q16[g].reshape(-1), 1, nq, d, m, S16, O.BF16, sg[g].reshape(-1), sk[g], T,
                        vcodes[g].reshape(-1), vnorms[g], vbits, olay, vs, c["vc"], scale, **kw)
        sc = O.score(q16[g].reshape(-1), 1, nq, d, m, S16, O.BF16, sg[g].reshape(-1), sk[g], T, **kw)
        vh = O.dequantize_f64(vcodes[g].reshape(-1), vnorms[g], d, vbits, olay, vs, c["vc"]).reshape(T, d)
        outs.append(o[0])
        logits.append(scale * sc[0])
        vhs.append(vh)
    return np.stack(outs), np.stack(logits), np.stack(vhs)


def check_attention(got, want, logits, vh, label, exact_weights=False):
    """The per-query bound and the aggregate relative bar of the module docstring."""
    vmax = np.sqrt((vh ** 2).sum(-1)).max(-1)                            # [G]
    eq = 1e-3 * np.abs(logits).max(-1)                                   # [G, nq]
    wt = np.zeros_like(eq) if exact_weights else 2.0 * (np.exp(2.0 * eq) - 1.0)
    tol = (wt + 2.0 ** -9) * vmax[:, None]                                # [G, nq]
    err = np.abs(got - want)
    worst = float((err.max(-1) / tol).max())
    rel = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300))
    report("attention", label=label, n=int(err.size), worst_over_tol=worst, rel_l2=rel,
           max_abs=float(err.max()), out_rms=float(np.sqrt((want ** 2).mean())))
    assert worst <= 1.0, f"{label}: worst error {worst:.3f} of the bound"
    assert rel <= 2e-3, f"{label}: relative L2 error {rel:.2e}"


@pytest.mark.parametrize("two_stage,kbits,vbits,nq,T", [(False, 0, 4, 32, 1000), (True, 2, 4, 32, 777),
                                                        (True, 3, 3, 7, 513), (False, 0, 2, 19, 256),
                                                        (True, 4, 8, 32, 300)])
def test_attention_matches_oracle(two_stage, kbits, vbits, nq, T):
    G, d, m = 3, 128, 256 if not two_stage else 128
    c = compress(G, T, d, m, kbits, vbits, 80 + 7 * vbits + kbits, two_stage,
                 vlayout=L.RQ_CODES_INT8 if vbits == 8 else L.RQ_CODES_PACKED)
    q = synth.normal((G, nq, d), seed=81, device=DEV)
    scale = 1.0 / math.sqrt(d)
    got = run_attention(c, q, G, nq, d, m, T, kbits, vbits, scale)
    want, logits, vh = oracle_attention(c, q, G, nq, d, m, T, kbits, vbits, scale)
    check_attention(got, want, logits, vh, f"attention two={two_stage} kb={kbits} vb={vbits} nq={nq} T={T}")


def test_attention_single_key():
    G, T, nq, d, m = 2, 1, 5, 128, 128
    c = compress(G, T, d, m, 0, 4, 90, False)
    q = synth.normal((G, nq, d), seed=91, device=DEV)
    got = run_attention(c, q, G, nq, d, m, T, 0, 4, 0.1)
    want, logits, vh = oracle_attention(c, q, G, nq, d, m, T, 0, 4, 0.1)
    check_attention(got, want, logits, vh, "attention T=1", exact_weights=True)


def test_attention_equal_keys_average_values():
    """All keys of a group equal: uniform weights whatever the scores, so the
    output is the mean of the reconstructed values (tight bar)."""
    G, T, nq, d, m = 2, 700, 9, 128, 128
    k1 = synth.kv_with_channels(1, G, 1, d, seed=92, device=DEV)
    k = k1.expand(1, G, T, d).contiguous().reshape(-1)
    c = compress(G, T, d, m, 0, 4, 93, False, k=k)
    q = synth.normal((G, nq, d), seed=94, device=DEV)
    got = run_attention(c, q, G, nq, d, m, T, 0, 4, 0.2)
    want, logits, vh = oracle_attention(c, q, G, nq, d, m, T, 0, 4, 0.2)
    assert np.allclose(want, vh.mean(axis=1, keepdims=True), rtol=1e-12, atol=1e-12)
    check_attention(got, want, logits, vh, "attention equal keys", exact_weights=True)


def test_attention_hard_max_selects_one_value():
    """Each query equal to one of the keys and a scale so large that this key
    carries all the weight: the output is its reconstructed value (tight bar)."""
    G, T, nq, d, m = 1, 300, 4, 128, 256
    k = synth.normal((1, G, T, d), seed=95, device=DEV)
    picks = [3, 100, 257, 299]
    q = k[0, :, picks, :].contiguous().reshape(G, nq, d)
    c = compress(G, T, d, m, 0, 4, 95, False, k=k.reshape(-1))
    _, logits1, _ = oracle_attention(c, q, G, nq, d, m, T, 0, 4, 1.0)
    assert np.array_equal(np.argmax(logits1[0], axis=-1), picks)
    srt = np.sort(logits1[0], axis=-1)
    gap = float((srt[:, -1] - srt[:, -2]).min())
    assert gap > 0.05 * float(srt[:, -1].min())
    scale = 200.0 / gap
    got = run_attention(c, q, G, nq, d, m, T, 0, 4, scale)
    want, logits, vh = oracle_attention(c, q, G, nq, d, m, T, 0, 4, scale)
    assert np.allclose(want[0], vh[0][picks], rtol=0, atol=1e-9)
    check_attention(got, want, logits, vh, "attention hard max", exact_weights=True)


def test_attention_kv_cache_full_size_sampled_groups():
    """The KV-cache shape 4 x 8 heads x 32768 tokens x 128, pure QJL keys
    (m = 256) and 4-bit values, 32 queries per head: every group's key range
    spans several CTAs (partial slots and the combine); three groups are
    checked against the oracle over all 32768 keys."""
    B, H, T, d, m, nq = 4, 8, 32768, 128, 256, 32
    G = B * H
    k = synth.kv_with_channels(B, H, T, d, seed=3, device=DEV).reshape(-1)
    v = synth.kv_with_channels(B, H, T, d, seed=13, device=DEV).reshape(-1)
    c = compress(G, T, d, m, 0, 4, 97, False, k=k, v=v)
    q = synth.normal((G, nq, d), seed=5, device=DEV)
    scale = 1.0 / math.sqrt(d)
    got = run_attention(c, q, G, nq, d, m, T, 0, 4, scale)
    groups = [0, 13, G - 1]
    want, logits, vh = oracle_attention(c, q, G, nq, d, m, T, 0, 4, scale, groups=groups)
    check_attention(got[groups], want, logits, vh, "attention kv 4x8x32768 m=256 v4")


def test_attention_many_tiles_per_cta():
    """Short groups, so every CTA's range crosses several group boundaries
    (several partial slots per CTA) and runs several tiles."""
    G, T, nq, d, m = 3 * num_sms() // 2 + 5, 600, 16, 128, 128
    c = compress(G, T, d, m, 2, 3, 98, True)
    q = synth.normal((G, nq, d), seed=99, device=DEV)
    got = run_attention(c, q, G, nq, d, m, T, 2, 3, 0.09)
    groups = [0, 1, G // 2, G - 2, G - 1]
    want, logits, vh = oracle_attention(c, q, G, nq, d, m, T, 2, 3, 0.09, groups=groups)
    check_attention(got[groups], want, logits, vh, f"attention many tiles G={G}")
