"""Benchmark of the rotated-quantization + QJL hot path on B200.

Headline (one step = the whole path over one batch of input): all linears of
32 Llama-7B-shaped decoder layers in bf16 (per layer q/k/v/o 4096x4096,
gate/up 11008x4096, down 4096x11008; 6.48e9 values, 13 GB), entries
N(0, 0.02^2) times a per-output-row scale exp(U[ln 1/2, ln 2]); d = 128,
4-bit Lloyd-Max codes packed, sign diagonal seeded 1000 + layer.  Per layer one
rq_quantize call (the layer's seven matrices are contiguous) then one
rq_dequantize call.  Metric: quantize+dequantize input GB/s = 2 bytes x 6.48e9
/ step time.  The input is 100x the L2, so no flush is needed.

Secondary lines (each its own roofline): the 256x512 fp16 weight round trip
(latency), the 4096x4096 bf16 weight with outliers at 3/4/5 bits with the
fused QJL residual sketch (m = 128), the KV cache 4x8x32768x128 (V: 4-bit
round trip; K: QJL m = 256 sketch and the pure-QJL score of 32 queries per
head), and TurboQuant-style 3-bit keys (2-bit + QJL m = d) at head dim 256
and 512 for 131072 tokens x 8 heads, with their scores.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

--gpus N > 1 runs one independent replica per GPU (relaunching itself under
torch.distributed.run when started without it); nothing is exchanged but a
barrier and the max-over-ranks step time.
"""
from __future__ import annotations

import argparse
import json
import os
import socket
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

D, BITS = 128, 4
LAYERS = 32
LLAMA7B = ((4096, 4096),) * 4 + ((11008, 4096),) * 2 + ((4096, 11008),)   # q k v o gate up down
LAYER_N = sum(r * c for r, c in LLAMA7B)                                # 202,375,168
WORKLOAD = ("all linears of 32 Llama-7B-shaped decoder layers, bf16 (6,476,005,376 values; per layer q/k/v/o "
            "4096x4096, gate/up 11008x4096, down 4096x11008), N(0,0.02^2) x per-row exp(U[ln .5, ln 2]); "
            "d=128, 4-bit packed Lloyd-Max, signs seeded 1000+layer; per layer rq_quantize then rq_dequantize")


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="rq", choices=["rq", "reference"])
    p.add_argument("--no-secondary", action="store_true")
    p.add_argument("--no-cpu", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--profile", default=None,
                   help="run one case's kernels once (profiling driver): c3_layer, weight4096_fused, kv_sketch, "
                        "kv_score, kv_attention, kv_outlier, kv_v, kv_v96, kv_dense, tq256, tq512; print nothing else")
    p.add_argument("--rank-selftest", action="store_true", help=argparse.SUPPRESS)
    return p.parse_args(argv)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def roofline_hbm(alg_bytes, ms, traffic=None, **extra):
    hbm, _, src = peaks()
    gbs = alg_bytes / (ms * 1e-3) / 1e9
    r = {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s", "frac": round(gbs / hbm, 4),
         "peak_source": src, "traffic": traffic}
    r.update(extra)
    return r


def roofline_tensor(flops, ms, **extra):
    _, tf, src = peaks()
    t = flops / (ms * 1e-3) / 1e12
    r = {"bound": "tensor", "achieved": round(t, 2), "peak": tf, "unit": "TFLOP/s", "frac": round(t / tf, 4),
         "peak_source": src}
    r.update(extra)
    return r


class Clocks:
    """nvidia-smi samples (every 20 ms), kept for the timed window only."""

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


# ---------------------------------------------------------------------------- replicas

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


def free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def relaunch_under_torchrun(args, argv):
    """`--gpus N` started as a plain process: run N replicas, one per GPU, by
    re-executing this script under torch.distributed.run (rank 0 prints)."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr=127.0.0.1", f"--master-port={free_port()}", os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


# ---------------------------------------------------------------------------- workloads

def make_llama(dev):
    """The 32-layer input as one contiguous bf16 buffer (layer-major), matrix
    i of the 224 drawn with seed 1000 + i."""
    import torch
    from kv_quantization_b200 import synth
    x = torch.empty(LAYERS * LAYER_N, dtype=torch.bfloat16, device=dev)
    off = 0
    for i in range(LAYERS * len(LLAMA7B)):
        r, c = LLAMA7B[i % len(LLAMA7B)]
        x[off:off + r * c] = synth.llama_linear(r, c, seed=1000 + i, device=dev).reshape(-1)
        off += r * c
    return x


def alg_quant(n, d=D, bits=BITS, m=0):
    b = n * 2 + n * bits / 8 + 2 * n / d
    if m:
        b += n * m / (8 * d) + 2 * n / d
    return b


def alg_dequant(n, d=D, bits=BITS):
    return n * bits / 8 + 2 * n / d + n * 2


def ev():
    import torch
    return torch.cuda.Event(enable_timing=True)


def l2_flusher(dev):
    import torch
    buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    return lambda: buf.view(torch.int32).sum()   # a 256 MB read evicts earlier data from the 126 MB L2


# DRAM bytes (read + write) per launch from one-kernel ncu captures of the
# current kernels (profiles/quantize_dequantize_llama7b_layer.md): the
# quantize and dequantize of one Llama-7B-shaped layer (202,375,168 values).
# Set back to None whenever either kernel changes.
NCU_DRAM_LAYER = {"quantize": 405_248_512 + 81_866_240, "dequantize": 104_401_152 + 345_138_944}


def run_headline(args, dev, world, rank):
    import torch
    import kv_quantization_b200 as rq
    cent = rq.rq_lloyd_max(BITS)
    x = make_llama(dev)
    n = x.numel()
    cb = LAYER_N * BITS // 8
    codes = torch.empty(LAYERS * cb, dtype=torch.uint8, device=dev)
    norms = torch.empty(n // D, dtype=torch.int16, device=dev)
    out = torch.empty_like(x)
    nb = LAYER_N // D
    layer = [(x[l * LAYER_N:(l + 1) * LAYER_N], codes[l * cb:(l + 1) * cb], norms[l * nb:(l + 1) * nb],
              out[l * LAYER_N:(l + 1) * LAYER_N]) for l in range(LAYERS)]
    stream = torch.cuda.current_stream()

    def step(evs=None):
        for l, (xl, cl, nl, ol) in enumerate(layer):
            if evs: evs[2 * l][0].record(stream)
            rq.rq_quantize(xl, D, BITS, rq.RQ_CODES_PACKED, 1, 1000 + l, cent, cl, nl)
            if evs: evs[2 * l][1].record(stream)
            if evs: evs[2 * l + 1][0].record(stream)
            rq.rq_dequantize(cl, nl, LAYER_N, D, BITS, rq.RQ_CODES_PACKED, 1, 1000 + l, cent, ol)
            if evs: evs[2 * l + 1][1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    n_ev = 2 * LAYERS
    evs_all = [[(ev(), ev()) for _ in range(n_ev)] for _ in range(args.steps)]
    clk = Clocks(dev.index)
    clk.start()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = ev(), ev()
    t0 = time.time()
    e0.record(stream)
    for s in range(args.steps):
        step(evs_all[s])
    e1.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    if world > 1:
        dist.barrier()
    clk.window(t0, t1)
    clk.stop()
    total_ms = reduce_max_ms(e0.elapsed_time(e1), world, dev)
    q_ms = [evs_all[s][2 * l][0].elapsed_time(evs_all[s][2 * l][1]) for s in range(args.steps) for l in range(LAYERS)]
    dq_ms = [evs_all[s][2 * l + 1][0].elapsed_time(evs_all[s][2 * l + 1][1])
             for s in range(args.steps) for l in range(LAYERS)]
    torch.cuda.synchronize()
    assert rq.rq_device_error(True) == 0
    in_bytes = n * 2
    value = job_rate(in_bytes, world, args.steps, total_ms) / 1e9
    mq, mdq = statistics.mean(q_ms), statistics.mean(dq_ms)
    if sum(q_ms) >= sum(dq_ms):
        dom = roofline_hbm(alg_quant(LAYER_N), mq, NCU_DRAM_LAYER["quantize"],
                           kernel="quantize_v5_kernel<4,bf16,signs> (d=128)",
                           alg_bytes_per_launch=alg_quant(LAYER_N), launches_timed=len(q_ms))
    else:
        dom = roofline_hbm(alg_dequant(LAYER_N), mdq, NCU_DRAM_LAYER["dequantize"],
                           kernel="dequantize_v5p_kernel<4,bf16,signs> (d=128)",
                           alg_bytes_per_launch=alg_dequant(LAYER_N), launches_timed=len(dq_ms))
    dom["traffic_note"] = ("ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch on one layer "
                           "(profiles/); null when not captured for this build")
    pair = roofline_hbm(alg_quant(LAYER_N) + alg_dequant(LAYER_N), mq + mdq)
    res = {
        "metric": "quantize+dequantize input GB/s", "value": round(value, 2), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 in/out, fp32 arithmetic, 4-bit codes", "data": "synthetic (seeded)",
        "config": {"workload": WORKLOAD, "elements": n, "d": D, "bits": BITS, "layers": LAYERS,
                   "l2": "inputs (13 GB) far larger than L2; no flush needed",
                   "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"},
        "pct_hbm_peak": round(100 * pair["frac"], 1),
        "roofline": dom,
        "kernels": {"quantize_ms_per_layer": round(mq, 4), "dequantize_ms_per_layer": round(mdq, 4),
                    "quantize": roofline_hbm(alg_quant(LAYER_N), mq),
                    "dequantize": roofline_hbm(alg_dequant(LAYER_N), mdq),
                    "pair": pair},
        "gpu_launches": n_ev * args.steps,
        "clocks": clk.summary(),
    }
    bufs = dict(x=x, codes=codes, norms=norms, out=out, cent=cent)
    return res, bufs


def run_e2e(args, dev, bufs):
    """The headline through the public API from pinned host buffers: per layer
    the input goes host -> device, quantize + dequantize run, and the codes,
    norms and reconstruction come back device -> host, pipelined over three
    streams (copy in / compute / copy out) with two device buffers per role."""
    import torch
    import kv_quantization_b200 as rq
    x, cent = bufs["x"], bufs["cent"]
    cb, nb = LAYER_N * BITS // 8, LAYER_N // D
    try:
        hx = torch.empty(x.numel(), dtype=torch.bfloat16, pin_memory=True)
    except RuntimeError as e:
        return {"unavailable": f"pinned host input buffer: {e}"}
    hx.copy_(x)
    x = None
    bufs.clear()                      # the device copies of the headline are not needed any more
    torch.cuda.empty_cache()
    dxin = [torch.empty(LAYER_N, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    dcodes = [torch.empty(cb, dtype=torch.uint8, device=dev) for _ in range(2)]
    dnorms = [torch.empty(nb, dtype=torch.int16, device=dev) for _ in range(2)]
    dout = [torch.empty(LAYER_N, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    hout = [torch.empty(LAYER_N, dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    hcodes = [torch.empty(cb, dtype=torch.uint8, pin_memory=True) for _ in range(2)]
    hnorms = [torch.empty(nb, dtype=torch.int16, pin_memory=True) for _ in range(2)]
    s_in, s_c, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    main = torch.cuda.current_stream()
    in_done = [torch.cuda.Event() for _ in range(2)]
    c_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]

    def one_step():
        s_in.wait_stream(main)
        s_c.wait_stream(main)
        s_out.wait_stream(main)
        for l in range(LAYERS):
            b = l & 1
            with torch.cuda.stream(s_in):
                if l >= 2:
                    s_in.wait_event(c_done[b])               # compute of layer l-2 has read dxin[b]
                dxin[b].copy_(hx[l * LAYER_N:(l + 1) * LAYER_N], non_blocking=True)
                in_done[b].record(s_in)
            with torch.cuda.stream(s_c):
                s_c.wait_event(in_done[b])
                if l >= 2:
                    s_c.wait_event(out_done[b])              # layer l-2's results have left the device
                rq.rq_quantize(dxin[b], D, BITS, rq.RQ_CODES_PACKED, 1, 1000 + l, cent, dcodes[b], dnorms[b],
                               stream=s_c)
                rq.rq_dequantize(dcodes[b], dnorms[b], LAYER_N, D, BITS, rq.RQ_CODES_PACKED, 1, 1000 + l, cent,
                                 dout[b], stream=s_c)
                c_done[b].record(s_c)
            with torch.cuda.stream(s_out):
                s_out.wait_event(c_done[b])
                hout[b].copy_(dout[b], non_blocking=True)
                hcodes[b].copy_(dcodes[b], non_blocking=True)
                hnorms[b].copy_(dnorms[b], non_blocking=True)
                out_done[b].record(s_out)
        main.wait_stream(s_in)
        main.wait_stream(s_c)
        main.wait_stream(s_out)

    one_step()
    torch.cuda.synchronize()
    steps = max(2, min(args.steps, 3))
    e0, e1 = ev(), ev()
    e0.record(main)
    for _ in range(steps):
        one_step()
    e1.record(main)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    h2d = LAYERS * LAYER_N * 2
    d2h = LAYERS * (LAYER_N * 2 + cb + nb * 2)
    return {"value": round(LAYERS * LAYER_N * 2 / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 3),
            "path": "rq_quantize + rq_dequantize per layer, pinned host in/out, copies overlapped with compute"}


def median_ms(fn, reps, flush=None, batch=1):
    """Median device time of one fn() call.  With batch > 1 (inputs larger
    than L2, no flush) each rep times `batch` back-to-back calls, so the
    host's per-call launch work overlaps the previous call's kernels."""
    import torch
    ts = []
    for _ in range(reps):
        if flush:
            flush()
        a, b = ev(), ev()
        a.record()
        for _ in range(batch):
            fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b) / batch)
    return statistics.median(ts)


def secondary_lines(dev, reps=10, only=None):
    """Each secondary workload's kernels timed with CUDA events (median of
    reps; L2 flushed before each rep where the input would fit in L2)."""
    import torch
    import kv_quantization_b200 as rq
    from kv_quantization_b200 import synth
    flush = l2_flusher(dev)
    out = []
    # the attention line runs on the key line's sketch, so it comes with it
    want = (lambda k: True) if only is None else (lambda k: k == only or (only == "kv_k" and k in ("kv_attn",
                                                                                                   "kv_outlier"))
                                                  or (only == "kv_outlier" and k == "kv_k"))

    if want("c1"):
        # 256 x 512 fp16, d = 128, 4-bit int8 codes, no signs: L2-resident latency
        x = synth.gaussian_matrix(256, 512, 0.02, seed=0, dtype=torch.float16, device=dev).reshape(-1)
        cent = rq.rq_lloyd_max(4)
        codes = torch.empty(x.numel(), dtype=torch.uint8, device=dev)
        norms = torch.empty(x.numel() // 128, dtype=torch.int16, device=dev)
        o = torch.empty_like(x)
        q = lambda: rq.rq_quantize(x, 128, 4, rq.RQ_CODES_INT8, 0, 0, cent, codes, norms)
        dq = lambda: rq.rq_dequantize(codes, norms, x.numel(), 128, 4, rq.RQ_CODES_INT8, 0, 0, cent, o)
        q(); dq()
        tq, tdq = median_ms(q, reps * 5), median_ms(dq, reps * 5)
        out.append({"workload": "weight 256x512 fp16 N(0,0.02^2), d=128, 4-bit int8 codes, no signs",
                    "quantize_us": round(tq * 1e3, 2), "dequantize_us": round(tdq * 1e3, 2),
                    "round_trip_us": round((tq + tdq) * 1e3, 2), "note": "L2-resident; latency-bound (launch + one wave)"})

    if want("weight4096"):
        x = synth.student_t_outliers(4096, 4096, seed=1, device=dev).reshape(-1)
        n = x.numel()
        m = 128
        S = torch.empty(m, D, dtype=torch.bfloat16, device=dev)
        rq.qjl_make_projection(2, m, D, S)
        res = {"workload": "weight 4096x4096 bf16 student-t(4) std 0.02 + 0.1% outliers x20; d=128, signs seed 1; "
                           "fused QJL residual sketch m=128 (S seed 2); bits 3/4/5", "l2": "flushed before each kernel"}
        for b in (3, 4, 5):
            cent = rq.rq_lloyd_max(b)
            codes = torch.empty(rq.rq_code_bytes(n, D, b, rq.RQ_CODES_PACKED), dtype=torch.uint8, device=dev)
            norms = torch.empty(n // D, dtype=torch.int16, device=dev)
            qs = torch.empty(n // D * m // 8, dtype=torch.uint8, device=dev)
            qn = torch.empty(n // D, dtype=torch.int16, device=dev)
            o = torch.empty_like(x)
            fq = lambda: rq.rq_quantize_qjl(x, D, b, rq.RQ_CODES_PACKED, 1, 1, cent, m, S, codes, norms, qs, qn)
            pq = lambda: rq.rq_quantize(x, D, b, rq.RQ_CODES_PACKED, 1, 1, cent, codes, norms)
            dq = lambda: rq.rq_dequantize(codes, norms, n, D, b, rq.RQ_CODES_PACKED, 1, 1, cent, o)
            fq(); dq()
            tf_, tq, tdq = median_ms(fq, reps, flush), median_ms(pq, reps, flush), median_ms(dq, reps, flush)
            res[f"b{b}"] = {"quantize_qjl_ms": round(tf_, 4), "quantize_ms": round(tq, 4), "dequantize_ms": round(tdq, 4),
                            "input_gbs_fused_pair": round(n * 2 / ((tf_ + tdq) * 1e-3) / 1e9, 1),
                            "input_gbs_pair": round(n * 2 / ((tq + tdq) * 1e-3) / 1e9, 1),
                            "quantize_qjl_roofline": roofline_hbm(alg_quant(n, bits=b, m=m), tf_),
                            "pair_roofline": roofline_hbm(alg_quant(n, bits=b) + alg_dequant(n, bits=b), tq + tdq)}
        out.append(res)
        del x, S

    if want("kv_v"):
        # V of the KV cache: RHT + 4-bit Lloyd-Max round trip
        v = synth.kv_with_channels(4, 8, 32768, 128, seed=13, device=dev).reshape(-1)
        n = v.numel()
        cent = rq.rq_lloyd_max(4)
        codes = torch.empty(n // 2, dtype=torch.uint8, device=dev)
        norms = torch.empty(n // 128, dtype=torch.int16, device=dev)
        o = torch.empty_like(v)
        q = lambda: rq.rq_quantize(v, 128, 4, rq.RQ_CODES_PACKED, 1, 14, cent, codes, norms)
        dq = lambda: rq.rq_dequantize(codes, norms, n, 128, 4, rq.RQ_CODES_PACKED, 1, 14, cent, o)
        q(); dq()
        tq, tdq = median_ms(q, reps, batch=4), median_ms(dq, reps, batch=4)
        out.append({"workload": "KV cache V 4x8x32768x128 bf16 N(0,1) (4 channels/head x10): RHT (signs seed 14) "
                                "+ 4-bit Lloyd-Max quantize then dequantize",
                    "quantize_ms": round(tq, 4), "dequantize_ms": round(tdq, 4),
                    "input_gbs": round(n * 2 / ((tq + tdq) * 1e-3) / 1e9, 1),
                    "roofline": roofline_hbm(alg_quant(n) + alg_dequant(n), tq + tdq)})
        del v, codes, norms, o

    if want("kv_v96"):
        # the same V line at head dim 96: blocks of a non-power-of-two size (block-diagonal 64 + 32 transform)
        dv = 96
        v = synth.kv_with_channels(4, 8, 32768, dv, seed=13, device=dev).reshape(-1)
        n = v.numel()
        cent = rq.rq_lloyd_max(4)
        codes = torch.empty(n // 2, dtype=torch.uint8, device=dev)
        norms = torch.empty(n // dv, dtype=torch.int16, device=dev)
        o = torch.empty_like(v)
        q = lambda: rq.rq_quantize(v, dv, 4, rq.RQ_CODES_PACKED, 1, 14, cent, codes, norms)
        dq = lambda: rq.rq_dequantize(codes, norms, n, dv, 4, rq.RQ_CODES_PACKED, 1, 14, cent, o)
        q(); dq()
        tq, tdq = median_ms(q, reps, batch=4), median_ms(dq, reps, batch=4)
        out.append({"workload": "KV cache V 4x8x32768x96 bf16 N(0,1) (4 channels/head x10), head dim 96: block-diagonal "
                                "64 + 32 RHT (signs seed 14) + 4-bit Lloyd-Max quantize then dequantize",
                    "quantize_ms": round(tq, 4), "dequantize_ms": round(tdq, 4),
                    "input_gbs": round(n * 2 / ((tq + tdq) * 1e-3) / 1e9, 1),
                    "roofline": roofline_hbm(alg_quant(n, d=dv) + alg_dequant(n, d=dv), tq + tdq)})
        del v, codes, norms, o

    if want("kv_dense"):
        # the V line with a dense random orthogonal rotation (128 x 128 tensor-core GEMM per tile of
        # 128 blocks) and the 4-bit Lloyd-Max codebook of the coordinate law of a uniform unit vector
        v = synth.kv_with_channels(4, 8, 32768, D, seed=13, device=dev).reshape(-1)
        n = v.numel()
        cent = rq.rq_beta_lloyd_max(D, 4)
        pi = torch.from_numpy(rq.rq_make_rotation(D, 17)).to(dev).to(torch.bfloat16)
        codes = torch.empty(n // 2, dtype=torch.uint8, device=dev)
        norms = torch.empty(n // D, dtype=torch.int16, device=dev)
        o = torch.empty_like(v)
        q = lambda: rq.rq_quantize_dense(v, D, pi, 4, rq.RQ_CODES_PACKED, cent, codes, norms)
        dq = lambda: rq.rq_dequantize_dense(codes, norms, n, D, pi, 4, rq.RQ_CODES_PACKED, cent, o)
        q(); dq()
        tq, tdq = median_ms(q, reps, batch=4), median_ms(dq, reps, batch=4)
        flops = 2.0 * n * D                                  # one d x d rotation per block, each way
        _, bf16_peak, _ = peaks()
        out.append({"workload": "KV cache V 4x8x32768x128 bf16 N(0,1) (4 channels/head x10): dense random orthogonal "
                                "rotation (QR of a Gaussian, seed 17) + 4-bit Beta-law Lloyd-Max quantize then "
                                "dequantize",
                    "quantize_ms": round(tq, 4), "dequantize_ms": round(tdq, 4),
                    "input_gbs": round(n * 2 / ((tq + tdq) * 1e-3) / 1e9, 1),
                    "tensor_tflops": round(2 * flops / ((tq + tdq) * 1e-3) / 1e12, 1),
                    "tensor_frac": round(2 * flops / ((tq + tdq) * 1e-3) / 1e12 / bf16_peak, 4),
                    "roofline": roofline_hbm(alg_quant(n) + alg_dequant(n), tq + tdq)})
        del v, codes, norms, o

    if want("kv_k"):
        G, T, d, m, nq = 32, 32768, 128, 256, 32
        k = synth.kv_with_channels(4, 8, T, d, seed=3, device=dev).reshape(-1)
        S = torch.empty(m, d, dtype=torch.bfloat16, device=dev)
        rq.qjl_make_projection(3, m, d, S)
        signs = torch.empty(G * T * m // 8, dtype=torch.uint8, device=dev)
        kn = torch.empty(G * T, dtype=torch.int16, device=dev)
        q = synth.normal((G, nq, d), seed=5, device=dev)
        scores = torch.empty(G, nq, T, dtype=torch.float32, device=dev)
        ws = torch.empty(rq.qjl_score_workspace_bytes(G, nq, d, m) // 4, dtype=torch.float32, device=dev)
        sk = lambda: rq.qjl_sketch(k, d, m, S, signs, kn)
        sc = lambda: rq.qjl_score(q, G, nq, d, m, S, signs, kn, T, scores, ws)
        sk(); sc()
        tk, ts = median_ms(sk, reps, batch=4), median_ms(sc, reps, flush)
        kbytes = k.numel() * 2 + signs.numel() + kn.numel() * 2
        sbytes = signs.numel() + kn.numel() * 2 + 4 * G * nq * T
        out.append({"workload": "KV cache K 4x8x32768x128 bf16 (4 channels/head x10): QJL sketch m=256 (S seed 3); "
                                "pure-QJL score of 32 queries per (batch, head)",
                    "sketch_ms": round(tk, 4), "score_ms": round(ts, 4),
                    "score_tokens_per_s": round(G * T / (ts * 1e-3), 1),
                    "sketch_roofline": roofline_hbm(kbytes, tk, flops=2 * m * d * G * T),
                    "score_roofline": roofline_hbm(sbytes, ts, note="signs + norms read, fp32 scores written; "
                                                                    "query prologue included")})
        if want("kv_outlier"):
            # the same keys with the per-group outlier sketch: 8 outliers per 32 tokens, m_o = 256
            mo, nout = 256, 8
            oidx = torch.empty(G * T // 32 * nout, dtype=torch.uint8, device=dev)
            osg = torch.empty(G * T * mo // 8, dtype=torch.uint8, device=dev)
            onr = torch.empty(G * T, dtype=torch.int16, device=dev)
            kin = torch.empty(rq.qjl_sketch_outlier_workspace_bytes(G * T, d), dtype=torch.uint8, device=dev)
            osk = lambda: rq.qjl_sketch_outlier(k, d, m, S, mo, nout, signs, kn, oidx, osg, onr, kin)
            osc = lambda: rq.qjl_score_outlier(q, G, nq, d, m, S, signs, kn, T, mo, nout, oidx, osg, onr, scores, ws)
            osk(); osc()
            tok_, tos = median_ms(osk, reps, batch=4), median_ms(osc, reps, flush)
            okbytes = k.numel() * 2 + signs.numel() + osg.numel() + 4 * G * T + oidx.numel()
            osbytes = sbytes + osg.numel() + 2 * G * T + oidx.numel() + 4 * G * nq * T
            out.append({"workload": "KV cache K 4x8x32768x128 bf16 (4 channels/head x10): QJL sketch m=256 with the "
                                    "per-group outlier sketch (8 of 128 coordinates per 32 tokens, m_o=256); score of "
                                    "32 queries per (batch, head) with the outlier term",
                        "sketch_ms": round(tok_, 4), "score_ms": round(tos, 4),
                        "score_tokens_per_s": round(G * T / (tos * 1e-3), 1),
                        "sketch_roofline": roofline_hbm(okbytes, tok_, note="keys read once; the masked copy's "
                                                                             "write and re-read are not counted"),
                        "score_roofline": roofline_hbm(osbytes, tos, note="main and outlier records read, fp32 "
                                                                          "scores written and re-read")})
            del oidx, osg, onr, kin
            sk()                                             # the plain sketch again for the attention line
        del scores, ws
        if want("kv_attn"):
            # attention decode over the sketched keys and the 4-bit values of the V line's recipe
            v = synth.kv_with_channels(4, 8, T, d, seed=13, device=dev).reshape(-1)
            vc = rq.rq_lloyd_max(4)
            vcodes = torch.empty(G * T * d // 2, dtype=torch.uint8, device=dev)
            vnorms = torch.empty(G * T, dtype=torch.int16, device=dev)
            rq.rq_quantize(v, d, 4, rq.RQ_CODES_PACKED, 1, 14, vc, vcodes, vnorms)
            del v
            aout = torch.empty(G, nq, d, dtype=torch.float32, device=dev)
            aws = torch.empty((rq.qjl_attention_workspace_bytes(G, nq, d, m, T) + 3) // 4, dtype=torch.float32,
                              device=dev)
            at = lambda: rq.qjl_attention(q, G, nq, d, m, S, signs, kn, T, vcodes, vnorms, 4, vc, aout, aws,
                                          1.0 / d ** 0.5, v_use_signs=1, v_sign_seed=14)
            at()
            ta = median_ms(at, reps, flush)
            abytes = signs.numel() + kn.numel() * 2 + vcodes.numel() + vnorms.numel() * 2 + q.numel() * 2 + \
                aout.numel() * 4
            out.append({"workload": "KV cache 4x8x32768x128 attention decode: the pure-QJL keys above (m=256) and "
                                    "4-bit values (signs seed 14), 32 queries per (batch, head), softmax scale "
                                    "1/sqrt(128); prologue + fused score/softmax/PV kernel + combine",
                        "attention_ms": round(ta, 4), "token_heads_per_s": round(G * T / (ta * 1e-3), 1),
                        "unfused_score_ms_for_context": round(ts, 4),
                        "roofline": roofline_hbm(abytes, ta, note="key signs + norms, value codes + norms read once; "
                                                                  "queries and outputs")})
            del vcodes, vnorms, aout, aws
        del k, signs, kn

    for d, seed in ((256, 6), (512, 8)):
        if not want(f"tq{d}"):
            continue
        G, T, bits, nq = 8, 131072, 2, 32
        m = d
        k = synth.normal((G, T, d), seed=seed, device=dev).reshape(-1)
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
        cp = lambda: rq.rq_quantize_qjl(k, d, bits, rq.RQ_CODES_PACKED, 1, 4, cent, m, S, codes, norms, qs, qn)
        sc = lambda: rq.qjl_score(q, G, nq, d, m, S, qs, qn, T, scores, ws, codes=codes, norms=norms, bits=bits,
                                  layout=rq.RQ_CODES_PACKED, use_signs=1, sign_seed=4, centroids=cent)
        cp(); sc()
        tc, ts = median_ms(cp, reps, batch=4), median_ms(sc, reps, flush)
        n = k.numel()
        cbytes = alg_quant(n, d=d, bits=bits, m=m)
        flops = 2 * m * d * G * T
        _, tf, _ = peaks()
        hbm = peaks()[0]
        tensor_bound = flops / cbytes > tf * 1e12 / (hbm * 1e9)
        sbytes = codes.numel() + qs.numel() + 4 * G * T + 4 * G * nq * T
        out.append({"workload": f"TurboQuant-style keys 131072 x 8 heads, d={d}, bf16 N(0,1): 2-bit (signs seed 4) + "
                                f"QJL m={m} residual (S seed 5); score of 32 queries per head",
                    "compress_ms": round(tc, 4), "score_ms": round(ts, 4),
                    "score_tokens_per_s": round(G * T / (ts * 1e-3), 1),
                    "compress_roofline": (roofline_tensor(flops, tc) if tensor_bound else
                                          roofline_hbm(cbytes, tc, flops=flops)),
                    "score_roofline": roofline_hbm(sbytes, ts, note="codes + signs + norms read, fp32 scores "
                                                                    "written; query prologue included")})
        del k, codes, norms, qs, qn, scores, ws
    torch.cuda.synchronize()
    assert rq.rq_device_error(True) == 0
    return out


# ---------------------------------------------------------------------------- oracle arm

def cpu_info():
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return model, os.cpu_count()


def oracle_llama_sample(frac=1):
    """The first 1/frac of each of layer 0's seven matrices (the same seeded
    values the device arm quantizes), as bf16 bit patterns."""
    from kv_quantization_b200 import synth
    parts = []
    for i, (r, c) in enumerate(LLAMA7B):
        w = synth.llama_linear(r, c, seed=1000 + i, device="cpu").reshape(-1)
        parts.append(synth.as_u16(w[: (r * c // frac) // D * D]).reshape(-1))
    return np.concatenate(parts)


def oracle_pair(x16, seed=1000):
    import oracle as O
    s = O.sign_diagonal(seed, D)
    c = O.f32_table(BITS)
    codes, norms, _, _ = O.quantize(x16, O.BF16, D, BITS, O.PACKED, s, c)
    O.dequantize(codes, norms, D, BITS, O.PACKED, s, c, O.BF16)


def cpu_baseline():
    """The oracle (single-threaded C), as it stands, on bounded samples: the
    headline's metric on a sample of the headline workload, plus one timing
    per secondary workload."""
    import torch
    import oracle as O
    from kv_quantization_b200 import synth
    O.lib()
    model, ncpu = cpu_info()
    x16 = oracle_llama_sample()
    t0 = time.perf_counter()
    oracle_pair(x16)
    dt = time.perf_counter() - t0
    res = {"value": round(x16.size * 2 / dt / 1e9, 6), "unit": "GB/s", "cores": 1, "kind": "oracle",
           "sample": f"all of layer 0's seven matrices ({x16.size} values), 4-bit quantize + "
                     f"dequantize, {dt:.1f} s on one thread",
           "cpu_model": model, "nproc": ncpu, "per_workload": {}}
    pw = res["per_workload"]
    # weight 256x512 fp16 (whole)
    w = synth.gaussian_matrix(256, 512, 0.02, seed=0, dtype=torch.float16, device="cpu").reshape(-1)
    w16 = synth.as_u16(w).reshape(-1)
    c4 = O.f32_table(4)
    t0 = time.perf_counter()
    cds, nrm, _, _ = O.quantize(w16, O.F16, 128, 4, O.INT8, None, c4)
    O.dequantize(cds, nrm, 128, 4, O.INT8, None, c4, O.F16)
    pw["weight256x512_round_trip_us"] = round((time.perf_counter() - t0) * 1e6, 1)
    # weight 4096^2 fused 4-bit, first 4096 blocks
    x = synth.student_t_outliers(4096, 4096, seed=1, device="cpu").reshape(-1)[: 4096 * 128]
    x16 = synth.as_u16(x).reshape(-1)
    S = O.projection(2, 128, 128, O.BF16)
    s = O.sign_diagonal(1, 128)
    t0 = time.perf_counter()
    cds, nrm, _, _ = O.quantize(x16, O.BF16, 128, 4, O.PACKED, s, c4)
    r, rn = O.residual(x16, O.BF16, cds, nrm, 128, 4, O.PACKED, s, c4)
    O.sketch(r, O.BF16, 128, 128, S)
    dt = time.perf_counter() - t0
    pw["weight4096_fused_b4_gbs"] = round(x16.size * 2 / dt / 1e9, 6)
    # KV keys: sketch of 16384 keys, score of 32 queries over 4096 keys
    k = synth.kv_with_channels(1, 1, 16384, 128, seed=3, device="cpu").reshape(-1)
    k16 = synth.as_u16(k).reshape(-1)
    S = O.projection(3, 256, 128, O.BF16)
    t0 = time.perf_counter()
    sg, _ = O.sketch(k16, O.BF16, 128, 256, S)
    dt = time.perf_counter() - t0
    pw["kv_sketch_keys_per_s"] = round(16384 / dt, 1)
    kn = O.vec_norms(k16, O.BF16, 128)
    q16 = synth.as_u16(synth.normal((1, 32, 128), seed=5, device="cpu")).reshape(-1)
    t0 = time.perf_counter()
    O.score(q16, 1, 32, 128, 256, S, O.BF16, sg[: 4096 * 32], kn[:4096], 4096)
    pw["kv_score_token_heads_per_s"] = round(4096 / (time.perf_counter() - t0), 1)
    # attention decode: 32 queries over 2048 sketched keys and 4-bit values of one head
    v16 = synth.as_u16(synth.kv_with_channels(1, 1, 2048, 128, seed=13, device="cpu")).reshape(-1)
    vs = O.sign_diagonal(14, 128)
    vcd, vnr, _, _ = O.quantize(v16, O.BF16, 128, 4, O.PACKED, vs, c4)
    t0 = time.perf_counter()
    O.attention(q16, 1, 32, 128, 256, S, O.BF16, sg[: 2048 * 32], kn[:2048], 2048, vcd, vnr, 4, O.PACKED, vs, c4,
                1.0 / 128 ** 0.5)
    pw["kv_attention_token_heads_per_s"] = round(2048 / (time.perf_counter() - t0), 1)
    # V cache at head dim 96 (block-diagonal transform): 16384 blocks round trip
    v96 = synth.as_u16(synth.kv_with_channels(1, 1, 16384, 96, seed=13, device="cpu")).reshape(-1)
    s96 = O.sign_diagonal(14, 96)
    t0 = time.perf_counter()
    cds, nrm, _, _ = O.quantize(v96, O.BF16, 96, 4, O.PACKED, s96, c4)
    O.dequantize(cds, nrm, 96, 4, O.PACKED, s96, c4, O.BF16)
    pw["kv_v96_round_trip_gbs"] = round(v96.size * 2 / (time.perf_counter() - t0) / 1e9, 6)
    # V cache with the dense rotation and the Beta codebook: 16384 blocks round trip (numpy fp64)
    from oracle import dense_rotation as DR
    pi16 = DR.to16(DR.rotation(17, 128), O.BF16)
    cb = DR.beta_lloyd_max(128, 4).astype(np.float32)
    vd = synth.as_u16(synth.kv_with_channels(1, 1, 16384, 128, seed=13, device="cpu")).reshape(-1)
    t0 = time.perf_counter()
    cds, nrm, _, _ = DR.quantize(vd, O.BF16, 128, pi16, 4, O.PACKED, cb)
    DR.dequantize(cds, nrm, 16384, 128, pi16, 4, O.PACKED, DR.to16(cb, O.BF16), O.BF16, O.BF16)
    pw["kv_dense_round_trip_gbs"] = round(vd.size * 2 / (time.perf_counter() - t0) / 1e9, 6)
    # TurboQuant-style keys at d = 256 / 512: compress 2048 keys, score 32 queries over 2048 keys
    for d in (256, 512):
        kk = synth.normal((1, 2048, d), seed=6, device="cpu").reshape(-1)
        kk16 = synth.as_u16(kk).reshape(-1)
        c2 = O.f32_table(2)
        sd = O.sign_diagonal(4, d)
        S = O.projection(5, d, d, O.BF16)
        t0 = time.perf_counter()
        cds, nrm, _, _ = O.quantize(kk16, O.BF16, d, 2, O.PACKED, sd, c2)
        r, rn = O.residual(kk16, O.BF16, cds, nrm, d, 2, O.PACKED, sd, c2)
        sg, _ = O.sketch(r, O.BF16, d, d, S)
        pw[f"tq{d}_compress_keys_per_s"] = round(2048 / (time.perf_counter() - t0), 1)
        q16 = synth.as_u16(synth.normal((1, 32, d), seed=7, device="cpu")).reshape(-1)
        t0 = time.perf_counter()
        O.score(q16, 1, 32, d, d, S, O.BF16, sg, rn, 2048, codes=cds, norms=nrm, bits=2, layout=O.PACKED,
                signs_diag=sd, c32=c2)
        pw[f"tq{d}_score_token_heads_per_s"] = round(2048 / (time.perf_counter() - t0), 1)
    return res


def run_reference(args):
    """The oracle as the reference arm, on the headline's metric and workload:
    each step a bounded sample (the first 1/64 of each of layer 0's matrices)."""
    import oracle as O
    O.lib()
    x16 = oracle_llama_sample(frac=64)
    for _ in range(args.warmup):
        oracle_pair(x16)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_pair(x16)
    dt = time.perf_counter() - t0
    v = x16.size * 2 * args.steps / dt / 1e9
    model, ncpu = cpu_info()
    sample = f"first 1/64 of each of layer 0's seven matrices ({x16.size} values) per step"
    return {"impl": "reference", "metric": "quantize+dequantize input GB/s", "value": round(v, 6), "unit": "GB/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16 in/out, fp32 arithmetic (fp64 where the oracle fixes it), 4-bit codes",
            "data": "synthetic (seeded)", "config": {"workload": WORKLOAD, "sample": sample},
            "cpu_baseline": {"value": round(v, 6), "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample,
                             "cpu_model": model, "nproc": ncpu},
            "e2e": {"value": round(v, 6), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------------------- profiling driver

def profile_case(case):
    """Run one case's kernels once on inputs larger than L2 (for one-kernel ncu
    captures); prints nothing."""
    import torch
    import kv_quantization_b200 as rq
    from kv_quantization_b200 import synth
    dev = torch.device("cuda:0")
    if case == "c3_layer":
        x = torch.empty(LAYER_N, dtype=torch.bfloat16, device=dev)
        off = 0
        for i, (r, c) in enumerate(LLAMA7B):
            x[off:off + r * c] = synth.llama_linear(r, c, seed=1000 + i, device=dev).reshape(-1)
            off += r * c
        cent = rq.rq_lloyd_max(BITS)
        codes = torch.empty(LAYER_N * BITS // 8, dtype=torch.uint8, device=dev)
        norms = torch.empty(LAYER_N // D, dtype=torch.int16, device=dev)
        out = torch.empty_like(x)
        rq.rq_quantize(x, D, BITS, rq.RQ_CODES_PACKED, 1, 1000, cent, codes, norms)
        rq.rq_dequantize(codes, norms, LAYER_N, D, BITS, rq.RQ_CODES_PACKED, 1, 1000, cent, out)
    else:
        key = {"weight4096_fused": "weight4096", "kv_sketch": "kv_k", "kv_score": "kv_k", "kv_attention": "kv_k",
               "kv_v": "kv_v", "kv_v96": "kv_v96", "kv_dense": "kv_dense", "kv_outlier": "kv_outlier", "tq256": "tq256", "tq512": "tq512"}[case]
        secondary_lines(dev, reps=1, only=key)
    torch.cuda.synchronize()
    assert rq.rq_device_error(True) == 0


# ---------------------------------------------------------------------------- main

def rank_selftest(args, rank, world):
    """CPU stand-in for the device arm, used by the multi-rank tests: each
    rank 'times' a fixed amount of work so that the launcher, the barrier and
    the max-over-ranks aggregation can be checked without a GPU."""
    local_ms = 10.0 * (rank + 1)
    total_ms = reduce_max_ms(local_ms * args.steps, world)
    return {"metric": "rank selftest units/s", "value": job_rate(100.0, world, args.steps, total_ms),
            "unit": "units/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_ms / args.steps}


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    args = parse(argv)
    if args.profile:
        profile_case(args.profile)
        return 0
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return relaunch_under_torchrun(args, argv)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    if world != args.gpus:
        print(json.dumps({"error": f"WORLD_SIZE={world} but --gpus {args.gpus}"}), flush=True)
        return 2
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0
    if world > 1:
        import datetime
        import torch.distributed as dist
        if args.rank_selftest:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
        else:
            import torch
            torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if args.rank_selftest:
        res = rank_selftest(args, rank, world)
    else:
        import torch
        import kv_quantization_b200 as rq
        dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
        torch.cuda.set_device(dev)
        rq.lib()
        res, bufs = run_headline(args, dev, world, rank)
        # every rank takes the same remaining steps (no collectives in them)
        res["e2e"] = {"skipped": "--no-e2e"} if args.no_e2e else run_e2e(args, dev, bufs)
        del bufs
        torch.cuda.empty_cache()
        res["secondary"] = [] if args.no_secondary else secondary_lines(dev)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if rank == 0:
        if not args.no_cpu and not args.rank_selftest:
            res["cpu_baseline"] = cpu_baseline()
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
