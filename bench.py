"""Benchmark of the rotated-quantization + QJL hot path on B200.

One step = the whole path over one 4096 x 4096 bf16 weight (Student-t nu=4,
std 0.02, 0.1% outliers x20; d = 128; seeded signs): for bits 3, 4 and 5,
rq_quantize_qjl (norm, sign flip, Walsh-Hadamard, Lloyd-Max search, packed
codes, fused residual + 1-bit QJL sketch with m = 128) then rq_dequantize.
Metric: quantize+dequantize input GB/s = 3 x 33.55 MB / step time, with L2
flushed between steps (inputs fit in L2).  Secondary: QJL score tokens/s on
the KV-cache (4 x 8 x 32768 keys, head_dim 128, m = 256, 32 queries) and the
TurboQuant-style 3-bit keys (131072 x 8, head_dim 256, 2-bit + QJL m = d).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

N > 1 runs one replica per GPU (torchrun; nothing is exchanged but the
barrier and the max-over-ranks step time).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

D, M = 128, 128
BITS = (3, 4, 5)
ROWS = COLS = 4096
SIGN_SEED, PROJ_SEED = 1, 2
WORKLOAD = "weight 4096x4096 bf16 student-t(4) std 0.02 + 0.1% outliers x20; d=128; bits 3,4,5 packed; " \
           "seeded signs; fused QJL residual sketch m=128; quantize+dequantize"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="rq", choices=["rq", "reference"])
    p.add_argument("--no-secondary", action="store_true")
    p.add_argument("--no-cpu", action="store_true")
    p.add_argument("--kernels-once", action="store_true",
                   help="run each hot kernel once on inputs larger than L2 (profiling driver), print nothing else")
    return p.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


class Clocks:
    """nvidia-smi samples (every 20 ms) kept for the timed window only."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.5)        # let the sampler come up before the timed window
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def window(self, t0, t1):
        self.t0, self.t1 = t0, t1

    def stop(self):
        if self.proc:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for t, line in self.lines:
            if self.t0 is not None and not (self.t0 <= t <= self.t1 + 0.05):
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------- device arm

def make_inputs(dev):
    import torch
    from kv_quantization_b200 import synth
    return synth.student_t_outliers(ROWS, COLS, seed=1, device=dev).reshape(-1)


def reduce_max_ms(total_ms, world, device=None):
    """Max over ranks of the per-rank timed milliseconds (the job ends with its
    slowest replica); identity on one rank."""
    if world <= 1:
        return float(total_ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(total_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank_step, world, steps, max_ms):
    """Whole-job throughput: the units every replica processed / the max time."""
    return units_per_rank_step * world * steps / (max_ms * 1e-3)


# DRAM bytes (read + write) of one 4-bit launch of each headline kernel, measured with
# ncu (--set full) on the 8192 x 8192 weight; scaled to a workload by element count.
# Writes still dirty in L2 when a kernel ends are not in the DRAM count.
NCU_DRAM_BYTES_8192SQ = {"qjl_v6": 134.53e6 + 25.83e6, "dequantize_v5": 34.65e6 + 74.65e6}


def alg_bytes_quant(n, bits):
    return n * 2 + n * bits / 8 + 2 * n / D


def alg_bytes_quant_qjl(n, bits):
    return n * 2 + n * bits / 8 + 2 * n / D + n * M / (8 * D) + 2 * n / D


def alg_bytes_dequant(n, bits):
    return n * bits / 8 + 2 * n / D + n * 2


def run_device(args, rank, world):
    import torch
    import kv_quantization_b200 as rq
    from kv_quantization_b200 import synth

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    rq.lib()
    x = make_inputs(dev)
    n = x.numel()
    S = torch.empty(M, D, dtype=torch.bfloat16, device=dev)
    rq.qjl_make_projection(PROJ_SEED, M, D, S)
    tabs = {b: rq.rq_lloyd_max(b) for b in BITS}
    bufs = {}
    for b in BITS:
        bufs[b] = dict(
            codes=torch.empty(rq.rq_code_bytes(n, D, b, rq.RQ_CODES_PACKED), dtype=torch.uint8, device=dev),
            norms=torch.empty(n // D, dtype=torch.int16, device=dev),
            qs=torch.empty(n // D * M // 8, dtype=torch.uint8, device=dev),
            qn=torch.empty(n // D, dtype=torch.int16, device=dev),
            out=torch.empty_like(x))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    n_ev = 2 * len(BITS)

    def l2_flush():
        flush.view(torch.int32).sum()   # read 256 MB: evicts earlier data from the 126 MB L2

    def step(evs=None):
        # every kernel starts with a cold L2 (flush outside its event pair)
        k = 0
        for b in BITS:
            B = bufs[b]
            l2_flush()
            if evs: evs[k][0].record(stream)
            rq.rq_quantize_qjl(x, D, b, rq.RQ_CODES_PACKED, 1, SIGN_SEED, tabs[b], M, S, B["codes"], B["norms"],
                               B["qs"], B["qn"])
            if evs: evs[k][1].record(stream)
            k += 1
            l2_flush()
            if evs: evs[k][0].record(stream)
            rq.rq_dequantize(B["codes"], B["norms"], n, D, b, rq.RQ_CODES_PACKED, 1, SIGN_SEED, tabs[b], B["out"])
            if evs: evs[k][1].record(stream)
            k += 1

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    kern_ms = [[0.0] * n_ev for _ in range(args.steps)]
    step_ms = []
    clk = Clocks(dev.index)
    clk.start()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    evs_all = []
    for s in range(args.steps):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_ev)]
        step(evs)
        evs_all.append(evs)
    torch.cuda.synchronize()
    t1 = time.time()
    if world > 1:
        dist.barrier()
    clk.window(t0, t1)
    clk.stop()
    for s, evs in enumerate(evs_all):
        for k in range(n_ev):
            kern_ms[s][k] = evs[k][0].elapsed_time(evs[k][1])
        step_ms.append(sum(kern_ms[s]))
    total_ms = reduce_max_ms(sum(step_ms), world, dev)
    in_bytes = n * 2 * len(BITS)
    value = job_rate(in_bytes, world, args.steps, total_ms) / 1e9
    hbm, tf, src = peaks()
    # dominant kernel: the larger of quantize_qjl / dequantize by total time
    q_ms = [statistics.mean(kern_ms[s][2 * i] for s in range(args.steps)) for i in range(len(BITS))]
    dq_ms = [statistics.mean(kern_ms[s][2 * i + 1] for s in range(args.steps)) for i in range(len(BITS))]
    if sum(q_ms) >= sum(dq_ms):
        dom, alg, ms = "qjl_v6_quant_kernel<b,bf16,signs> (d=128)", sum(alg_bytes_quant_qjl(n, b) for b in BITS), sum(q_ms)
        traffic = NCU_DRAM_BYTES_8192SQ["qjl_v6"] * n / 8192 ** 2
    else:
        dom, alg, ms = "dequantize_v5_kernel<b,bf16,signs> (d=128)", sum(alg_bytes_dequant(n, b) for b in BITS), sum(dq_ms)
        traffic = NCU_DRAM_BYTES_8192SQ["dequantize_v5"] * n / 8192 ** 2
    achieved = alg / (ms * 1e-3) / 1e9
    per_kernel = {f"quantize_qjl_b{b}_ms": round(q, 4) for b, q in zip(BITS, q_ms)}
    per_kernel.update({f"dequantize_b{b}_ms": round(q, 4) for b, q in zip(BITS, dq_ms)})
    per_kernel.update({f"quantize_qjl_b{b}_gbs": round(alg_bytes_quant_qjl(n, b) / (q * 1e-3) / 1e9, 1)
                       for b, q in zip(BITS, q_ms)})
    per_kernel.update({f"dequantize_b{b}_gbs": round(alg_bytes_dequant(n, b) / (q * 1e-3) / 1e9, 1)
                       for b, q in zip(BITS, dq_ms)})

    # quantize + dequantize alone (no QJL stage), same workload and cold L2
    qd = {}
    for b in BITS:
        B = bufs[b]
        tq, tdq = [], []
        for _ in range(max(5, min(args.steps, 50))):
            l2_flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            rq.rq_quantize(x, D, b, rq.RQ_CODES_PACKED, 1, SIGN_SEED, tabs[b], B["codes"], B["norms"])
            e1.record(stream)
            l2_flush()
            e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e2.record(stream)
            rq.rq_dequantize(B["codes"], B["norms"], n, D, b, rq.RQ_CODES_PACKED, 1, SIGN_SEED, tabs[b], B["out"])
            e3.record(stream)
            torch.cuda.synchronize()
            tq.append(e0.elapsed_time(e1))
            tdq.append(e2.elapsed_time(e3))
        mq, mdq = statistics.mean(tq), statistics.mean(tdq)
        qd[f"b{b}"] = {"quantize_ms": round(mq, 4), "dequantize_ms": round(mdq, 4),
                       "quantize_gbs": round(alg_bytes_quant(n, b) / (mq * 1e-3) / 1e9, 1),
                       "dequantize_gbs": round(alg_bytes_dequant(n, b) / (mdq * 1e-3) / 1e9, 1),
                       "input_gbs": round(n * 2 / ((mq + mdq) * 1e-3) / 1e9, 1),
                       "pct_hbm": round(100 * (alg_bytes_quant(n, b) + alg_bytes_dequant(n, b)) /
                                        ((mq + mdq) * 1e-3) / 1e9 / peaks()[0], 1)}

    # end to end through the public API with host buffers
    e2e = e2e_measure(args, x, S, tabs, bufs, dev)
    secondary = [] if args.no_secondary else secondary_scores(dev)
    result = {
        "metric": "quantize+dequantize input GB/s", "value": round(value, 2), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 in, fp32 arithmetic", "data": "synthetic (seeded)",
        "config": {"workload": WORKLOAD, "elements": n, "d": D, "bits": list(BITS), "qjl_m": M,
                   "l2": "flushed (256 MB read) before every kernel; step time = sum of kernel times", "parallelism": f"replicas x{world}"},
        "pct_hbm_peak": round(100 * achieved / hbm, 1),
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                     "frac": round(achieved / hbm, 4), "peak_source": src, "traffic": round(traffic),
                     "traffic_note": "ncu dram read+write of the 4-bit launch on the 8192^2 weight, scaled by "
                                     "elements; per launch (achieved covers the 3-bit, 4-bit and 5-bit launches)",
                     "alg_bytes_per_launch_4bit": round(alg_bytes_quant_qjl(n, 4) if dom.startswith("qjl")
                                                        else alg_bytes_dequant(n, 4)),
                     "alg_bytes_per_step": alg},
        "kernels": per_kernel,
        "quantize_dequantize_only": qd,
        "e2e": e2e,
        "gpu_launches": n_ev * args.steps,
        "clocks": clk.summary(),
        "secondary": secondary,
    }
    return result


def e2e_measure(args, x, S, tabs, bufs, dev):
    import torch
    import kv_quantization_b200 as rq
    n = x.numel()
    hx = torch.empty(n, dtype=torch.bfloat16, pin_memory=True)
    hx.copy_(x.cpu())
    hout = {b: {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in bufs[b].items()} for b in BITS}
    dx = torch.empty_like(x)
    stream = torch.cuda.current_stream()
    bo = sum(v.numel() * v.element_size() for b in BITS for v in bufs[b].values())

    def one():
        dx.copy_(hx, non_blocking=True)
        for b in BITS:
            B = bufs[b]
            rq.rq_quantize_qjl(dx, D, b, rq.RQ_CODES_PACKED, 1, SIGN_SEED, tabs[b], M, S, B["codes"], B["norms"],
                               B["qs"], B["qn"])
            rq.rq_dequantize(B["codes"], B["norms"], n, D, b, rq.RQ_CODES_PACKED, 1, SIGN_SEED, tabs[b], B["out"])
            for k, v in B.items():
                hout[b][k].copy_(v, non_blocking=True)

    for _ in range(2):
        one()
    torch.cuda.synchronize()
    steps = max(3, min(args.steps, 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    return {"value": round(n * 2 * len(BITS) / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": n * 2, "d2h_bytes_per_step": bo, "ms_per_step": round(ms, 4)}


def secondary_scores(dev, reps=5):
    """QJL score tokens/s (key token-heads scored against all 32 queries per s)."""
    import torch
    import kv_quantization_b200 as rq
    from kv_quantization_b200 import synth
    out = []
    # KV cache 4 x 8 x 32768 x 128, K via QJL m = 256, pure QJL score
    G, T, d, m, nq = 32, 32768, 128, 256, 32
    k = synth.kv_with_channels(4, 8, T, d, seed=3, device=dev).reshape(-1)
    S = torch.empty(m, d, dtype=torch.bfloat16, device=dev)
    rq.qjl_make_projection(3, m, d, S)
    signs = torch.empty(G * T * m // 8, dtype=torch.uint8, device=dev)
    kn = torch.empty(G * T, dtype=torch.int16, device=dev)
    q = synth.normal((G, nq, d), seed=5, device=dev)
    scores = torch.empty(G, nq, T, dtype=torch.float32, device=dev)
    ws = torch.empty(rq.qjl_score_workspace_bytes(G, nq, d, m) // 4, dtype=torch.float32, device=dev)
    out.append(_time_pair("kv 4x8x32768x128 QJL m=256",
                          lambda: rq.qjl_sketch(k, d, m, S, signs, kn),
                          lambda: rq.qjl_score(q, G, nq, d, m, S, signs, kn, T, scores, ws), G * T,
                          2 * m * d * G * T, k.numel() * 2 + signs.numel() + kn.numel() * 2, reps,
                          score_bytes=signs.numel() + kn.numel() * 2 + 4 * G * nq * T))
    del k, signs, kn, scores, ws
    # TurboQuant-style 3-bit keys, head_dim 256: 2-bit + QJL m = d
    G, T, d, bits = 8, 131072, 256, 2
    m = d
    k = synth.normal((G, T, d), seed=6, device=dev).reshape(-1)
    cent = rq.rq_lloyd_max(bits)
    S = torch.empty(m, d, dtype=torch.bfloat16, device=dev)
    rq.qjl_make_projection(5, m, d, S)
    codes = torch.empty(rq.rq_code_bytes(k.numel(), d, bits, rq.RQ_CODES_PACKED), dtype=torch.uint8, device=dev)
    norms = torch.empty(G * T, dtype=torch.int16, device=dev)
    qs = torch.empty(G * T * m // 8, dtype=torch.uint8, device=dev)
    qn = torch.empty(G * T, dtype=torch.int16, device=dev)
    q = synth.normal((G, nq, d), seed=7, device=dev)
    scores = torch.empty(G, nq, T, dtype=torch.float32, device=dev)
    ws = torch.empty(rq.qjl_score_workspace_bytes(G, nq, d, m) // 4, dtype=torch.float32, device=dev)
    out.append(_time_pair("keys 131072x8 d=256 2-bit+QJL m=d",
                          lambda: rq.rq_quantize_qjl(k, d, bits, rq.RQ_CODES_PACKED, 1, 4, cent, m, S, codes, norms,
                                                     qs, qn),
                          lambda: rq.qjl_score(q, G, nq, d, m, S, qs, qn, T, scores, ws, codes=codes, norms=norms,
                                               bits=bits, layout=rq.RQ_CODES_PACKED, use_signs=1, sign_seed=4,
                                               centroids=cent),
                          G * T, 2 * m * d * G * T, k.numel() * 2 + codes.numel() + qs.numel() + 4 * G * T, reps,
                          score_bytes=codes.numel() + qs.numel() + 4 * G * T + 4 * G * nq * T))
    del k, codes, norms, qs, qn, scores, ws
    # the same at head_dim 512 (m = d = 512)
    G, T, d, bits = 8, 131072, 512, 2
    m = d
    k = synth.normal((G, T, d), seed=8, device=dev).reshape(-1)
    S = torch.empty(m, d, dtype=torch.bfloat16, device=dev)
    rq.qjl_make_projection(9, m, d, S)
    codes = torch.empty(rq.rq_code_bytes(k.numel(), d, bits, rq.RQ_CODES_PACKED), dtype=torch.uint8, device=dev)
    norms = torch.empty(G * T, dtype=torch.int16, device=dev)
    qs = torch.empty(G * T * m // 8, dtype=torch.uint8, device=dev)
    qn = torch.empty(G * T, dtype=torch.int16, device=dev)
    q = synth.normal((G, nq, d), seed=10, device=dev)
    scores = torch.empty(G, nq, T, dtype=torch.float32, device=dev)
    ws = torch.empty(rq.qjl_score_workspace_bytes(G, nq, d, m) // 4, dtype=torch.float32, device=dev)
    out.append(_time_pair("keys 131072x8 d=512 2-bit+QJL m=d",
                          lambda: rq.rq_quantize_qjl(k, d, bits, rq.RQ_CODES_PACKED, 1, 4, cent, m, S, codes, norms,
                                                     qs, qn),
                          lambda: rq.qjl_score(q, G, nq, d, m, S, qs, qn, T, scores, ws, codes=codes, norms=norms,
                                               bits=bits, layout=rq.RQ_CODES_PACKED, use_signs=1, sign_seed=4,
                                               centroids=cent),
                          G * T, 2 * m * d * G * T, k.numel() * 2 + codes.numel() + qs.numel() + 4 * G * T, reps,
                          score_bytes=codes.numel() + qs.numel() + 4 * G * T + 4 * G * nq * T))
    return out


def _time_pair(name, prep, score, tokens, prep_flops, prep_bytes, reps=5, score_bytes=None):
    import torch
    prep()
    score()
    torch.cuda.synchronize()
    res = {"workload": name}
    if reps <= 1:
        return res
    for label, fn in (("compress", prep), ("score", score)):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        res[f"{label}_ms"] = round(ms, 4)
    res["score_tokens_per_s"] = round(tokens / (res["score_ms"] * 1e-3), 1)
    res["compress_gbs"] = round(prep_bytes / (res["compress_ms"] * 1e-3) / 1e9, 1)
    res["compress_tflops"] = round(prep_flops / (res["compress_ms"] * 1e-3) / 1e12, 2)
    hbm, tf, src = peaks()
    # compress: HBM-bound below the ridge (2 m d flops against 2 d + m/8 + ... bytes per vector)
    ridge = tf * 1e12 / (hbm * 1e9)
    if prep_flops / prep_bytes < ridge:
        res["compress_roofline"] = {"bound": "hbm", "achieved": res["compress_gbs"], "peak": hbm, "unit": "GB/s",
                                    "frac": round(res["compress_gbs"] / hbm, 4)}
    else:
        res["compress_roofline"] = {"bound": "tensor", "achieved": res["compress_tflops"], "peak": tf,
                                    "unit": "TFLOP/s", "frac": round(res["compress_tflops"] / tf, 4)}
    if score_bytes:
        gbs = score_bytes / (res["score_ms"] * 1e-3) / 1e9
        res["score_roofline"] = {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                                 "frac": round(gbs / hbm, 4),
                                 "note": "packed keys + norms read, fp32 scores written; prologue included"}
    return res


# ---------------------------------------------------------------------------- oracle arm

def oracle_sample(n_blocks, seed=1):
    """A bounded sample of the same workload for the CPU oracle: the first
    n_blocks blocks of the seeded matrix (generated on the CPU)."""
    import torch
    from kv_quantization_b200 import synth
    x = synth.student_t_outliers(ROWS, COLS, seed=seed, device="cpu").reshape(-1)[: n_blocks * D]
    return synth.as_u16(x).reshape(-1)


def oracle_step(x16):
    import oracle as O
    s = O.sign_diagonal(SIGN_SEED, D)
    S = O.projection(PROJ_SEED, M, D, O.BF16)
    for b in BITS:
        c = O.f32_table(b)
        codes, norms, _, _ = O.quantize(x16, O.BF16, D, b, O.PACKED, s, c)
        r, rn = O.residual(x16, O.BF16, codes, norms, D, b, O.PACKED, s, c)
        O.sketch(r, O.BF16, D, M, S)
        O.dequantize(codes, norms, D, b, O.PACKED, s, c, O.BF16)


def cpu_baseline(target_s=12.0):
    import oracle as O
    O.lib()
    x16 = oracle_sample(64)
    t0 = time.perf_counter()
    oracle_step(x16)
    per_block = (time.perf_counter() - t0) / 64
    nb = int(max(64, min(ROWS * COLS // D, target_s / max(per_block, 1e-9))))
    x16 = oracle_sample(nb)
    t0 = time.perf_counter()
    oracle_step(x16)
    dt = time.perf_counter() - t0
    return {"value": round(nb * D * 2 * len(BITS) / dt / 1e9, 6), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"first {nb} of {ROWS * COLS // D} blocks of the same matrix, bits 3/4/5, "
                      f"quantize+residual+sketch+dequantize, {dt:.1f} s single-threaded C"}


def run_reference(args):
    """The oracle as the reference arm: each step a bounded sample of the workload."""
    import oracle as O
    O.lib()
    nb = 256
    x16 = oracle_sample(nb)
    for _ in range(args.warmup):
        oracle_step(x16)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(x16)
    dt = time.perf_counter() - t0
    v = nb * D * 2 * len(BITS) * args.steps / dt / 1e9
    return {"impl": "reference", "metric": "quantize+dequantize input GB/s", "value": round(v, 6), "unit": "GB/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16 in, fp32/fp64 arithmetic",
            "data": "synthetic (seeded)",
            "config": {"workload": WORKLOAD, "sample_blocks_per_step": nb},
            "cpu_baseline": {"value": round(v, 6), "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": f"{nb} blocks of the workload per step"},
            "e2e": {"value": round(v, 6), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def kernels_once():
    """Each hot kernel once, inputs larger than L2: 8192 x 8192 bf16 weight
    (quantize, quantize+QJL, dequantize at 4 bits), the 4 x 8 x 32768 x 128 KV
    cache (QJL sketch m=256 and its score), 131072 x 8 keys at head_dim 256
    (2-bit + QJL m=d and its score)."""
    import torch
    import kv_quantization_b200 as rq
    from kv_quantization_b200 import synth
    dev = torch.device("cuda:0")
    x = synth.student_t_outliers(8192, 8192, seed=1, device=dev).reshape(-1)
    n, b = x.numel(), 4
    cent = rq.rq_lloyd_max(b)
    S = torch.empty(M, D, dtype=torch.bfloat16, device=dev)
    rq.qjl_make_projection(PROJ_SEED, M, D, S)
    codes = torch.empty(rq.rq_code_bytes(n, D, b, rq.RQ_CODES_PACKED), dtype=torch.uint8, device=dev)
    norms = torch.empty(n // D, dtype=torch.int16, device=dev)
    qs = torch.empty(n // D * M // 8, dtype=torch.uint8, device=dev)
    qn = torch.empty(n // D, dtype=torch.int16, device=dev)
    out = torch.empty_like(x)
    rq.rq_quantize(x, D, b, rq.RQ_CODES_PACKED, 1, SIGN_SEED, cent, codes, norms)
    rq.rq_quantize_qjl(x, D, b, rq.RQ_CODES_PACKED, 1, SIGN_SEED, cent, M, S, codes, norms, qs, qn)
    rq.rq_dequantize(codes, norms, n, D, b, rq.RQ_CODES_PACKED, 1, SIGN_SEED, cent, out)
    del x, out
    secondary_scores(dev, reps=1)
    torch.cuda.synchronize()
    assert rq.rq_device_error(True) == 0


def main():
    args = parse()
    if args.kernels_once:
        kernels_once()
        return
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    res = run_device(args, rank, world)
    if rank == 0:
        if not args.no_cpu:
            res["cpu_baseline"] = cpu_baseline()
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
