"""Full-size and many-tile GPU parity: the persistent kernels in their steady
state (every CTA looping over several tiles: ring refills and wrap-around,
both TMEM accumulators, the deferred sign epilogue, the parity-1 barrier
waits), at the workload sizes the benchmark times.  The oracle cannot redo a
whole workload in seconds, so each test compares a sample of blocks, keys or
(group, query, token) scores chosen to cover every CTA's first, second, third
and last tiles under both tile splits the kernels use, plus random ones; at
many-tile mid sizes it covers every tile.  Scores are also checked end to end:
raw keys -> the oracle's own compressed keys -> the oracle's scores, against
raw keys -> the library's compressed keys -> the library's scores.
"""
import numpy as np
import pytest
import torch

import oracle as O
from kv_quantization_b200 import _lib as L
from kv_quantization_b200 import synth
from tests.gpu_checks import (DEV, check_codes, check_scores, check_signs, code_mismatch_blocks, num_sms,
                              report, sample_units, score_tol, take_rows, u16)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def no_device_timeouts():
    yield
    torch.cuda.synchronize()
    assert L.rq_device_error(True) == 0
    torch.cuda.empty_cache()


def fused(x, d, bits, layout, seed, cent, m, S):
    nb = x.numel() // d
    codes = torch.empty(L.rq_code_bytes(x.numel(), d, bits, layout), dtype=torch.uint8, device=DEV)
    norms = torch.empty(nb, dtype=torch.int16, device=DEV)
    qs = torch.empty(nb * m // 8, dtype=torch.uint8, device=DEV)
    qn = torch.empty(nb, dtype=torch.int16, device=DEV)
    L.rq_quantize_qjl(x, d, bits, layout, 1, seed, cent, m, S, codes, norms, qs, qn)
    return codes, norms, qs, qn


def check_fused_sample(x, d, bits, layout, seed, cent, m, S, codes, norms, qs, qn, blocks, label):
    """Sampled blocks of a fused quantize + residual sketch against the oracle.
    Returns the oracle's compressed keys for the sample and the per-block
    flags of windowed (allowed) code or sign mismatches."""
    nb_full = x.numel() // d
    cb = L.rq_code_bytes(d, d, bits, layout)
    x16 = take_rows(x, blocks, d).reshape(-1)
    s = O.sign_diagonal(seed, d)
    oc, on, _, _ = O.quantize(x16, O.BF16, d, bits, layout, s, cent)
    gc = take_rows(codes, blocks, cb).reshape(-1)
    nmis = check_codes(gc, oc, x16, O.BF16, d, bits, layout, s, cent)
    assert np.array_equal(take_rows(norms, blocks, 1).reshape(-1).view(np.uint16), on)
    r_bf, rn = O.residual(x16, O.BF16, oc, on, d, bits, layout, s, cent)
    assert np.array_equal(take_rows(qn, blocks, 1).reshape(-1).view(np.uint16), rn)
    osg, p = O.sketch(r_bf, O.BF16, d, m, u16(S), want_p=True)
    gs = take_rows(qs, blocks, m // 8).reshape(-1)
    bad = check_signs(gs, osg, p, len(blocks), m, full_bits=nb_full * m)
    if nmis:
        bad = bad | code_mismatch_blocks(gc, oc, len(blocks), d, bits, layout)
    report("fused", label=label, blocks=int(len(blocks)), of=int(nb_full), code_mismatch=int(nmis),
           sign_mismatch_vectors=int(bad.sum()))
    return oc, on, osg, rn, bad


@pytest.mark.parametrize("bits", [3, 4, 5])
def test_weight_4096sq_fused_qjl_full_size(bits):
    """4096 x 4096 bf16 Student-t weight with outliers, d = 128, signs seed 1,
    QJL m = 128 (S seed 2): 1024 tiles over the persistent CTAs, two sampled
    blocks in every tile."""
    d, m = 128, 128
    x = synth.student_t_outliers(4096, 4096, seed=1, device=DEV).reshape(-1)
    cent = L.rq_lloyd_max(bits)
    S = torch.empty(m, d, dtype=torch.bfloat16, device=DEV)
    L.qjl_make_projection(2, m, d, S)
    codes, norms, qs, qn = fused(x, d, bits, L.RQ_CODES_PACKED, 1, cent, m, S)
    assert L.rq_last_launch() == "qjl_v6_quant_kernel"
    torch.cuda.synchronize()
    rng = np.random.default_rng(bits)
    blocks = np.unique(np.concatenate([sample_units(x.numel() // d, 128, num_sms(), rng, per_tile=2)]))
    check_fused_sample(x, d, bits, L.RQ_CODES_PACKED, 1, cent, m, S, codes, norms, qs, qn, blocks,
                       f"weight4096sq b{bits}")


@pytest.mark.parametrize("bits", [3, 4, 5])
def test_weight_4096sq_every_block_fresh_buffers(bits):
    """Quantize then dequantize the 4096 x 4096 weight into freshly allocated,
    sentinel-filled buffers, twice, and compare every block with the oracle:
    a read of shared memory that ran ahead of the bulk copy filling it would
    show up here as stale data in the first pass after new codes."""
    d = 128
    x = synth.student_t_outliers(4096, 4096, seed=1, device=DEV).reshape(-1)
    n = x.numel()
    cent = L.rq_lloyd_max(bits)
    x16 = u16(x)
    s = O.sign_diagonal(1, d)
    oc, on, _, _ = O.quantize(x16, O.BF16, d, bits, O.PACKED, s, cent)
    for trial in range(2):
        codes = torch.full((L.rq_code_bytes(n, d, bits, L.RQ_CODES_PACKED),), 0x5A, dtype=torch.uint8, device=DEV)
        norms = torch.full((n // d,), 0x3C00, dtype=torch.int16, device=DEV)
        L.rq_quantize(x, d, bits, L.RQ_CODES_PACKED, 1, 1, cent, codes, norms)
        out = torch.full_like(x, float("nan"))
        L.rq_dequantize(codes, norms, n, d, bits, L.RQ_CODES_PACKED, 1, 1, cent, out)
        torch.cuda.synchronize()
        gc = codes.cpu().numpy()
        nmis = check_codes(gc, oc, x16, O.BF16, d, bits, O.PACKED, s, cent)
        assert np.array_equal(norms.cpu().numpy().view(np.uint16), on)
        oo, _ = O.dequantize(gc, on, d, bits, O.PACKED, s, cent, O.BF16)
        assert np.array_equal(u16(out), oo), f"trial {trial}: {int((u16(out) != oo).sum())} values differ"
        report("weight4096sq_full", bits=bits, trial=trial, code_mismatch=int(nmis))


def sampled_tokens(G, T, sms, rng):
    """(group, token) pairs: the sampled units of the flat [G*T] key array,
    regrouped as the same token set for every group (scores compare on a
    rectangular [G][Ts] sample)."""
    flat = sample_units(G * T, 128, sms, rng)
    toks = np.unique(flat % T)
    if toks.size > 96:
        toks = np.unique(np.concatenate([toks[:: max(1, toks.size // 96)], [0, T - 1]]))
    return toks


def test_kv_cache_key_sketch_and_score_full_size():
    """KV-cache keys 4 x 8 x 32768 x 128 (N(0,1), 4 channels per head x10):
    QJL m = 256 (S seed 3) over 8192 tiles, sampled keys against the oracle;
    then the pure-QJL score of 32 queries per (batch, head) over all keys,
    sampled tokens against the oracle -- from the library's signs, and end to
    end from the oracle's own sketch of the raw keys."""
    B, H, T, d, m, nq = 4, 8, 32768, 128, 256, 32
    G = B * H
    k = synth.kv_with_channels(B, H, T, d, seed=3, device=DEV).reshape(-1)
    S = torch.empty(m, d, dtype=torch.bfloat16, device=DEV)
    L.qjl_make_projection(3, m, d, S)
    signs = torch.empty(G * T * m // 8, dtype=torch.uint8, device=DEV)
    kn = torch.empty(G * T, dtype=torch.int16, device=DEV)
    L.qjl_sketch(k, d, m, S, signs, kn)
    assert L.rq_last_launch() == "sketch_v3_kernel"
    q = synth.normal((G, nq, d), seed=5, device=DEV)
    scores = torch.empty(G, nq, T, dtype=torch.float32, device=DEV)
    ws = torch.empty(L.qjl_score_workspace_bytes(G, nq, d, m) // 4, dtype=torch.float32, device=DEV)
    L.qjl_score(q, G, nq, d, m, S, signs, kn, T, scores, ws)
    assert L.rq_last_launch() == "score_v2_prologue,score_v5_kernel"
    torch.cuda.synchronize()
    rng = np.random.default_rng(7)
    sms = num_sms()
    # sketch: sampled keys of the flat [G*T] array
    keys = sample_units(G * T, 128, sms, rng)
    k16 = take_rows(k, keys, d).reshape(-1)
    os_, p = O.sketch(k16, O.BF16, d, m, u16(S), want_p=True)
    bad = check_signs(take_rows(signs, keys, m // 8).reshape(-1), os_, p, len(keys), m, full_bits=G * T * m)
    assert np.array_equal(take_rows(kn, keys, 1).reshape(-1).view(np.uint16), O.vec_norms(k16, O.BF16, d))
    report("sketch", label="kv 4x8x32768x128 m=256", keys=int(len(keys)), of=G * T,
           sign_mismatch_vectors=int(bad.sum()))
    # score on a [G][Ts] sample of tokens
    toks = sampled_tokens(G, T, sms, rng)
    Ts = toks.size
    rows = (np.arange(G)[:, None] * T + toks[None, :]).reshape(-1)
    g_sig = take_rows(signs, rows, m // 8).reshape(-1)
    g_kn = take_rows(kn, rows, 1).reshape(-1).view(np.uint16)
    q16 = u16(q)
    got = scores.cpu().numpy()[:, :, toks].astype(np.float64)
    want = O.score(q16, G, nq, d, m, u16(S), O.BF16, g_sig, g_kn, Ts)
    tol = score_tol(q16, G, nq, d, g_kn.reshape(G, Ts))
    check_scores(got, want, tol, "kv 4x8x32768 pure QJL m=256, library keys")
    # end to end: the oracle sketches the sampled raw keys itself
    kr16 = take_rows(k, rows, d).reshape(-1)
    o_sig, o_p = O.sketch(kr16, O.BF16, d, m, u16(S), want_p=True)
    o_kn = O.vec_norms(kr16, O.BF16, d)
    same = ~check_signs(g_sig, o_sig, o_p, G * Ts, m, full_bits=G * T * m)
    want_e2e = O.score(q16, G, nq, d, m, u16(S), O.BF16, o_sig, o_kn, Ts)
    mask = np.broadcast_to(same.reshape(G, 1, Ts), got.shape)
    check_scores(got, want_e2e, score_tol(q16, G, nq, d, o_kn.reshape(G, Ts)),
                 "kv 4x8x32768 pure QJL m=256, end to end", mask=mask)


@pytest.mark.parametrize("d", [256, 512])
def test_turboquant_keys_full_size(d):
    """131072 cached tokens x 8 KV heads at head dim d in bf16, N(0,1): 2-bit
    rotated Lloyd-Max (signs seed 4) + QJL m = d residual sketch (S seed 5)
    over 8192 tiles, sampled blocks against the oracle; then 32 queries per
    head scored against all keys, sampled tokens against the oracle (from the
    library's compressed keys, and end to end from the oracle's own)."""
    G, T, bits, nq = 8, 131072, 2, 32
    m = d
    k = synth.normal((G, T, d), seed=6 if d == 256 else 8, device=DEV).reshape(-1)
    cent = L.rq_lloyd_max(bits)
    S = torch.empty(m, d, dtype=torch.bfloat16, device=DEV)
    L.qjl_make_projection(5, m, d, S)
    codes, norms, qs, qn = fused(k, d, bits, L.RQ_CODES_PACKED, 4, cent, m, S)
    assert L.rq_last_launch() == ("qjl_v7_quant_kernel" if d == 256 else "qjl_v8_quant_kernel")
    q = synth.normal((G, nq, d), seed=7, device=DEV)
    scores = torch.empty(G, nq, T, dtype=torch.float32, device=DEV)
    ws = torch.empty(L.qjl_score_workspace_bytes(G, nq, d, m) // 4, dtype=torch.float32, device=DEV)
    L.qjl_score(q, G, nq, d, m, S, qs, qn, T, scores, ws, codes=codes, norms=norms, bits=bits,
                layout=L.RQ_CODES_PACKED, use_signs=1, sign_seed=4, centroids=cent)
    assert L.rq_last_launch() == "score_v2_prologue,score_v5_kernel"
    torch.cuda.synchronize()
    rng = np.random.default_rng(d)
    sms = num_sms()
    blocks = sample_units(G * T, 128, sms, rng)
    check_fused_sample(k, d, bits, L.RQ_CODES_PACKED, 4, cent, m, S, codes, norms, qs, qn, blocks,
                       f"keys 131072x8 d={d}")
    toks = sampled_tokens(G, T, sms, rng)
    Ts = toks.size
    rows = (np.arange(G)[:, None] * T + toks[None, :]).reshape(-1)
    cb = L.rq_code_bytes(d, d, bits, L.RQ_CODES_PACKED)
    g_codes = take_rows(codes, rows, cb).reshape(-1)
    g_n = take_rows(norms, rows, 1).reshape(-1).view(np.uint16)
    g_sig = take_rows(qs, rows, m // 8).reshape(-1)
    g_rn = take_rows(qn, rows, 1).reshape(-1).view(np.uint16)
    q16 = u16(q)
    sd = O.sign_diagonal(4, d)
    got = scores.cpu().numpy()[:, :, toks].astype(np.float64)
    want = O.score(q16, G, nq, d, m, u16(S), O.BF16, g_sig, g_rn, Ts, codes=g_codes, norms=g_n, bits=bits,
                   layout=O.PACKED, signs_diag=sd, c32=cent)
    check_scores(got, want, score_tol(q16, G, nq, d, g_n.reshape(G, Ts)), f"two-stage d={d}, library keys")
    # end to end from the oracle's own compression of the sampled raw keys
    oc, on, osg, orn, bad = check_fused_sample(k, d, bits, L.RQ_CODES_PACKED, 4, cent, m, S, codes, norms, qs, qn,
                                               rows, f"keys 131072x8 d={d} score sample")
    want_e2e = O.score(q16, G, nq, d, m, u16(S), O.BF16, osg, orn, Ts, codes=oc, norms=on, bits=bits,
                       layout=O.PACKED, signs_diag=sd, c32=cent)
    mask = np.broadcast_to((~bad).reshape(G, 1, Ts), got.shape)
    check_scores(got, want_e2e, score_tol(q16, G, nq, d, on.reshape(G, Ts)), f"two-stage d={d}, end to end",
                 mask=mask)


# Fallback kernels at many tiles per CTA (3 x SMs tiles + a ragged tail):
# every tile sampled.
MANY_TILE_FUSED = [
    # d, bits, m, layout, kernel
    (128, 7, 128, L.RQ_CODES_PACKED, "qjl_v3_quant_kernel"),
    (256, 8, 64, L.RQ_CODES_PACKED, "qjl_v3_quant_kernel"),
    (64, 3, 72, L.RQ_CODES_PACKED, "qjl_mma_kernel<fused>"),
    (128, 4, 264, L.RQ_CODES_INT8, "qjl_mma_kernel<fused>"),
    (512, 8, 16, L.RQ_CODES_PACKED, "qjl_mma_kernel<fused>"),
    (512, 4, 264, L.RQ_CODES_PACKED, "quantize_kernel"),
    (256, 3, 128, L.RQ_CODES_PACKED, "qjl_v7_quant_kernel"),
    (512, 2, 72, L.RQ_CODES_PACKED, "qjl_v8_quant_kernel"),
    (128, 2, 40, L.RQ_CODES_PACKED, "qjl_v6_quant_kernel"),
]


@pytest.mark.parametrize("d,bits,m,layout,kernel", MANY_TILE_FUSED)
def test_fused_many_tiles(d, bits, m, layout, kernel):
    nb = 3 * num_sms() * 128 + 11
    x = synth.student_t_outliers(1, nb * d, seed=40 + d + bits, device=DEV).reshape(-1)
    cent = L.rq_lloyd_max(bits)
    S = torch.empty(m, d, dtype=torch.bfloat16, device=DEV)
    L.qjl_make_projection(41, m, d, S)
    codes, norms, qs, qn = fused(x, d, bits, layout, 42, cent, m, S)
    assert L.rq_last_launch() == kernel
    torch.cuda.synchronize()
    blocks = sample_units(nb, 128, num_sms(), np.random.default_rng(d * bits + m))
    check_fused_sample(x, d, bits, layout, 42, cent, m, S, codes, norms, qs, qn, blocks,
                       f"{kernel} d={d} b={bits} m={m} x{nb}")


MANY_TILE_SKETCH = [
    (128, 128, "sketch_v3_kernel"),
    (128, 512, "qjl_mma_kernel<sketch>"),
    (256, 256, "qjl_mma_kernel<sketch>"),
    (512, 512, "sketch_kernel"),
]


@pytest.mark.parametrize("d,m,kernel", MANY_TILE_SKETCH)
def test_sketch_many_tiles(d, m, kernel):
    n = 3 * num_sms() * 128 + 37
    k = synth.kv_with_channels(1, 1, n, d, seed=50 + d, device=DEV).reshape(-1)
    S = torch.empty(m, d, dtype=torch.bfloat16, device=DEV)
    L.qjl_make_projection(51, m, d, S)
    signs = torch.empty(n * m // 8, dtype=torch.uint8, device=DEV)
    kn = torch.empty(n, dtype=torch.int16, device=DEV)
    L.qjl_sketch(k, d, m, S, signs, kn)
    assert L.rq_last_launch() == kernel
    torch.cuda.synchronize()
    keys = sample_units(n, 128, num_sms(), np.random.default_rng(d + m))
    k16 = take_rows(k, keys, d).reshape(-1)
    os_, p = O.sketch(k16, O.BF16, d, m, u16(S), want_p=True)
    check_signs(take_rows(signs, keys, m // 8).reshape(-1), os_, p, len(keys), m, full_bits=n * m)
    assert np.array_equal(take_rows(kn, keys, 1).reshape(-1).view(np.uint16), O.vec_norms(k16, O.BF16, d))


@pytest.mark.parametrize("d,bits,m,nq,kernel", [(128, 4, 128, 32, "score_v5_kernel"), (256, 2, 256, 20, "score_v5_kernel"),
                                                (128, 3, 64, 24, "score_v4_kernel"), (128, 3, 64, 144, "score_kernel")])
def test_score_many_tiles(d, bits, m, nq, kernel):
    """Scores over 3 x SMs token tiles per group set (the score's chunk ring
    wraps many times), every tile sampled."""
    G = 3
    T = num_sms() * (256 if kernel == "score_v5_kernel" else 128) + 77
    k = synth.normal((G, T, d), seed=60 + d, device=DEV).reshape(-1)
    cent = L.rq_lloyd_max(bits)
    S = torch.empty(m, d, dtype=torch.bfloat16, device=DEV)
    L.qjl_make_projection(61, m, d, S)
    codes, norms, qs, qn = fused(k, d, bits, L.RQ_CODES_PACKED, 62, cent, m, S)
    q = synth.normal((G, nq, d), seed=63, device=DEV)
    scores = torch.empty(G, nq, T, dtype=torch.float32, device=DEV)
    ws = torch.empty(L.qjl_score_workspace_bytes(G, nq, d, m) // 4, dtype=torch.float32, device=DEV)
    L.qjl_score(q, G, nq, d, m, S, qs, qn, T, scores, ws, codes=codes, norms=norms, bits=bits,
                layout=L.RQ_CODES_PACKED, use_signs=1, sign_seed=62, centroids=cent)
    assert L.rq_last_launch().split(",")[-1] == kernel
    torch.cuda.synchronize()
    rng = np.random.default_rng(d + nq)
    toks = np.unique(np.concatenate([[0, T - 1], [rng.integers(t, min(T, t + 128)) for t in range(0, T, 128)]]))
    Ts = toks.size
    rows = (np.arange(G)[:, None] * T + toks[None, :]).reshape(-1)
    cb = L.rq_code_bytes(d, d, bits, L.RQ_CODES_PACKED)
    g_n = take_rows(norms, rows, 1).reshape(-1).view(np.uint16)
    q16 = u16(q)
    want = O.score(q16, G, nq, d, m, u16(S), O.BF16, take_rows(qs, rows, m // 8).reshape(-1),
                   take_rows(qn, rows, 1).reshape(-1).view(np.uint16), Ts,
                   codes=take_rows(codes, rows, cb).reshape(-1), norms=g_n, bits=bits, layout=O.PACKED,
                   signs_diag=O.sign_diagonal(62, d), c32=cent)
    got = scores.cpu().numpy()[:, :, toks].astype(np.float64)
    check_scores(got, want, score_tol(q16, G, nq, d, g_n.reshape(G, Ts)), f"many tiles d={d} nq={nq}")
