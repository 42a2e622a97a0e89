"""Comparison helpers shared by the GPU parity tests (librq against the oracle).

Bars, from the arithmetic each side follows:
  * codes, norms, reconstructions, residual norms, the projection matrix:
    bit-exact (both sides compute in the same canonical fp32 order); any code
    mismatch must also sit within 1e-5 of a decision boundary and their count
    stay below 1e-6 of the elements;
  * sign bits: bit-exact except where |P_i| / ||v|| <= 1e-5 (the GPU
    accumulates in fp32, the oracle in fp64), count below 1e-6 of the bits;
  * scores: |gpu - oracle| <= 1e-3 * ||q|| * ||k|| -- the error scale of a dot
    product of that size, ||k|| the key's stored norm (the sketch norm for a
    pure QJL key, the first-stage block norm for a two-stage key).  The
    oracle is fp64 from the same 16-bit inputs.
"""
import json
import os

import numpy as np
import torch

import oracle as O
from kv_quantization_b200 import _lib as L
from kv_quantization_b200 import synth

DEV = "cuda:0"

_REPORT = []


def report(kind, **fields):
    """Record one parity measurement; written as JSON lines at session end to
    the path in RQ_PARITY_REPORT (if set)."""
    _REPORT.append(dict(kind=kind, **fields))


def write_report():
    path = os.environ.get("RQ_PARITY_REPORT")
    if path and _REPORT:
        with open(path, "w") as f:
            for r in _REPORT:
                f.write(json.dumps(r) + "\n")


def u16(t):
    return synth.as_u16(t).reshape(-1)


def dt_code(dtype):
    return O.BF16 if dtype == torch.bfloat16 else O.F16


def num_sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def f16_values(h):
    return np.asarray(h, np.uint16).view(np.float16).astype(np.float64)


def check_codes(g_codes, o_codes, x16, dtype, d, bits, layout, signs, cent):
    """Bit-exact codes, or mismatches confined to the 1e-5 boundary window.
    Returns the per-block mismatch flags' count."""
    if np.array_equal(g_codes, o_codes):
        return 0
    nb = x16.size // d
    gi = O.unpack_codes(g_codes, nb, d, bits, layout)
    oi = O.unpack_codes(o_codes, nb, d, bits, layout)
    bad = np.nonzero(gi != oi)[0]
    y64 = O.rotate_f64(x16, dtype, d, signs)
    t = O.boundaries(cent).astype(np.float64)
    near = np.min(np.abs(y64[bad][:, None] - t[None, :]), axis=1) <= 1e-5
    assert near.all(), f"{(~near).sum()} code mismatches outside the boundary window"
    assert bad.size < max(1.0, 1e-6 * x16.size), f"{bad.size} windowed mismatches"
    return bad.size


def code_mismatch_blocks(g_codes, o_codes, nb, d, bits, layout):
    gi = O.unpack_codes(g_codes, nb, d, bits, layout).reshape(nb, d)
    oi = O.unpack_codes(o_codes, nb, d, bits, layout).reshape(nb, d)
    return np.any(gi != oi, axis=1)


def check_signs(g, o, p_rel, n, m, full_bits=None):
    """Sign bits equal except within the 1e-5 window.  `full_bits` is the
    number of bits the sample stands for (the mismatch budget scales with
    it).  Returns the per-vector mismatch flags."""
    gb = np.unpackbits(g.reshape(n, m // 8), axis=1, bitorder="little")
    ob = np.unpackbits(o.reshape(n, m // 8), axis=1, bitorder="little")
    diff = gb != ob
    if not diff.any():
        return np.zeros(n, bool)
    bad = np.nonzero(diff.reshape(-1))[0]
    assert np.all(np.abs(p_rel[bad]) <= 1e-5), "sign mismatch outside the window"
    budget = max(1.0, 1e-6 * (full_bits if full_bits else n * m))
    assert bad.size < budget, f"{bad.size} windowed sign mismatches"
    return diff.any(axis=1)


def score_tol(q16, G, nq, d, key_norms16):
    """1e-3 * ||q|| * ||k|| for [G][nq][T] scores; key_norms16: fp16 patterns [G][T]."""
    qf = (np.asarray(q16, np.uint32) << 16).view(np.float32).astype(np.float64).reshape(G, nq, d)
    qn = np.linalg.norm(qf, axis=2)[:, :, None]
    kn = f16_values(key_norms16).reshape(G, 1, -1)
    return 1e-3 * qn * kn


def check_scores(got, want, tol, label, mask=None):
    """|got - want| <= tol elementwise (on `mask` when given); records the
    error against the tolerance scale and the raw relative error |d|/|s|."""
    got = np.asarray(got, np.float64)
    err = np.abs(got - want)
    if mask is not None:
        err, tol_m, want_m = err[mask], tol[mask], want[mask]
    else:
        tol_m, want_m = tol, want
    scale = tol_m / 1e-3
    rel = err / np.maximum(np.abs(want_m), 1e-300)
    report("score", label=label, n=int(err.size), max_err_over_qk=float((err / scale).max()),
           p50_rel=float(np.percentile(rel, 50)), p99_rel=float(np.percentile(rel, 99)),
           max_rel=float(rel.max()))
    assert np.all(err <= tol_m), f"{label}: worst error {float((err / scale).max()):.3e} of ||q|| ||k||"


def sample_tiles(ntiles, sms, rng, extra=512):
    """Tile indices covering every persistent CTA's first and last tiles under
    both tile splits the kernels use (contiguous ranges [t0, t1) per CTA, and
    strided t = cta + i * grid), their second and third tiles, plus random
    ones; every tile when there are few."""
    if ntiles <= 4096:
        return np.arange(ntiles)
    grid = min(ntiles, sms)
    s = set(range(min(ntiles, 3 * grid))) | set(range(max(0, ntiles - 2 * grid), ntiles))
    for b in range(grid):
        t0, t1 = ntiles * b // grid, ntiles * (b + 1) // grid
        s |= {t0, t0 + 1, t0 + 2, t1 - 3, t1 - 2, t1 - 1}
    s |= set(rng.choice(ntiles, min(extra, ntiles), replace=False).tolist())
    return np.array(sorted(t for t in s if 0 <= t < ntiles))


def sample_units(n, tile, sms, rng, per_tile=1):
    """Unit (block / vector) indices: `per_tile` random ones inside each
    sampled tile of `tile` units, plus the first and last unit."""
    ntiles = (n + tile - 1) // tile
    tiles = sample_tiles(ntiles, sms, rng)
    out = [0, n - 1]
    for t in tiles:
        lo, hi = t * tile, min(n, (t + 1) * tile)
        out.extend(rng.integers(lo, hi, size=per_tile).tolist())
    return np.unique(np.array(out, np.int64))


def take_rows(t, rows, width):
    """Rows `rows` of the [*, width] view of device tensor t, as a numpy array
    (16-bit tensors come back as uint16 bit patterns)."""
    if t.dtype in (torch.bfloat16, torch.float16, torch.int16):
        t = t.view(torch.int16)
    idx = torch.from_numpy(np.asarray(rows, np.int64)).to(t.device)
    a = t.reshape(-1, width)[idx].cpu().numpy()
    return a.view(np.uint16) if a.dtype == np.int16 else a
