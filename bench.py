#!/usr/bin/env python
"""Benchmark of the weight-only block-quantized lm_head matvec on B200.

Workload: the 248320 x 2048 lm_head at batch 1 (one decode token), one fused
dequant-matvec per weight format per step: fp4 (E2M1 + e8m0), int4 (symmetric,
MSE clip), int4km (per-row 16-entry palette), int8 (symmetric).  Weights are
seeded synthetic N(0, 0.02) with two outlier input columns x20, encoded on the
GPU by the library's own encoders (int4km: the 20-step per-row k-means
palette fit); activations N(0, 1) fp16.

Metric: effective weight GB/s = algorithmic bytes (codes + scales/palette +
x + y) / kernel time, and us per matvec.  Every input (~1.1 GB per step in
total) is larger than L2, so no flush is needed between steps.  The step is
captured once as a CUDA graph (four launches on one stream) and replayed per
step, as a decode loop runs; per-format times come from graphs of ten
back-to-back launches of one format, and the call-by-call step time is
reported beside them.  The weights are fixed, so launches may stream them
while the preceding launch drains (qmv_set_weight_prefetch; --no-prefetch
turns that off).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) each rank runs an independent replica on its own GPU
(the op has no cross-GPU exchange); `value` sums the ranks' bytes over the
slowest rank's time.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "effective weight GB/s (% of HBM peak) & us per 248320x2048 lm_head matvec"
N_HEAD, K_HEAD = 248320, 2048
FORMATS = ("fp4", "int4", "int4km", "int8")
FALLBACK_HBM_GBS = 6650.0


O8_COLS = 64  # outlier columns of the mixed int4km + int8 format in the extra measurement


def algorithmic_bytes(fmt: str, N: int, K: int, B: int) -> int:
    """Bytes a matvec must move: packed codes + block scales (or palette) +
    activations (fp16) + outputs (fp32)."""
    if fmt == "int4km_o8":  # main int4km columns + int8 outlier columns with scales, the column list
        C = O8_COLS
        return N * (K - C) // 2 + N * 16 * 2 + N * C + N * (C // 32) * 2 + C * 4 + B * K * 2 + B * N * 4
    codes = N * K if fmt in ("int8", "int8km") else N * K // 2
    aux = {"fp4": N * (K // 32), "int4": N * (K // 32) * 2, "int8": N * (K // 32) * 2, "int4km": N * 16 * 2,
           "int4aff": N * (2 * (K // 32) + (K // 32 + 1) // 2), "int8km": ((N + 31) // 32) * 256 * 2}[fmt]
    return codes + aux + B * K * 2 + B * N * 4


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# the sources mv_kernel (the step's kernel) is built from: its counters in
# profiles/ stay valid while these are unchanged
MV_KERNEL_SOURCES = ("weight_only_quantized_qmv_b200/csrc/qmv_matvec.cu",
                     "weight_only_quantized_qmv_b200/csrc/qmv_device.cuh",
                     "weight_only_quantized_qmv_b200/csrc/qmv_kernel_common.cuh",
                     "weight_only_quantized_qmv_b200/csrc/qmv_internal.h", "include/qmv.h")


def csrc_digest(sources=MV_KERNEL_SOURCES) -> str:
    d = hashlib.sha256()
    for rel in sources:
        with open(os.path.join(ROOT, rel), "rb") as f:
            d.update(os.path.basename(rel).encode() + f.read())
    return d.hexdigest()[:16]


def profiled_traffic(kernel_fmt: str):
    """DRAM bytes of one full-head launch from the committed ncu summary (the
    65536-row capture scaled by rows: the kernel streams each weight byte
    once), if it was taken on the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "qmv_matvec_formats_65536x2048_b1.md")
    if not os.path.exists(p):
        return None
    txt = open(p).read()
    m = re.search(r"csrc_sha256_16:\s*([0-9a-f]+)", txt)
    if not m or m.group(1) != csrc_digest():
        return None
    m = re.search(rf"dram_bytes_per_launch\[{kernel_fmt}\]:\s*([0-9]+)", txt)
    return int(m.group(1)) if m else None


# ----------------------------------------------------------------- ranks

def max_over_ranks(ms: float, device) -> float:
    """The slowest rank's time: every rank takes the job's pace from it
    (all-reduce MAX on the process group; gloo on CPU tensors, NCCL on GPU)."""
    import torch
    import torch.distributed as tdist
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(bytes_per_rank_step: int, world: int, ms_step: float) -> float:
    """Whole-job throughput: every replica moves bytes_per_rank_step per step,
    all of them at the slowest rank's step time."""
    return bytes_per_rank_step * world / (ms_step * 1e-3) / 1e9


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples (200 ms) of SM clock and throttle reasons while the
    timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="qmv_clocks_", suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.gpu_index)], stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[4], parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[4]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------- workload

def build_workload(device, formats=FORMATS):
    """The head's weights encoded by the library in each format.  Each
    encoder runs once on a small slice first (module load and first-launch
    costs), then its time on the full head is taken with CUDA events."""
    import torch
    import weight_only_quantized_qmv_b200 as q
    from weight_only_quantized_qmv_b200 import synth
    g = synth.generator(0, device)
    W, _ = synth.weights(N_HEAD, K_HEAD, g, n_outlier_cols=2)
    x = synth.activations(1, K_HEAD, g)
    enc_ms = {}
    ops = {}
    for fmt, fn in (("fp4", q.encode_fp4), ("int4", q.encode_int4), ("int8", q.encode_int8),
                    ("int4km", q.encode_int4km)):
        if fmt not in formats:
            continue
        fn(W[:256].contiguous())  # warm-up launch
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        codes, aux = fn(W)
        b.record()
        torch.cuda.synchronize()
        enc_ms[fmt] = round(a.elapsed_time(b), 3)
        ops[fmt] = (codes, aux)  # int4km: (indices, palette)
    del W
    torch.cuda.empty_cache()
    flags = q.status_fetch()
    if flags:
        raise RuntimeError(f"encoder status flags 0x{flags:x}")
    return x, ops, enc_ms


def capture(fn, stream, reps):
    """A CUDA graph of `reps` calls of fn on `stream` (fn's first calls, which
    set kernel attributes, run outside the capture)."""
    import torch
    with torch.cuda.stream(stream):
        fn()
        fn()
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(reps):
                fn()
    stream.synchronize()
    return g


def graph_us(g, stream, reps_per_graph, replays):
    """Mean device time per call of a captured graph (CUDA events on its stream)."""
    import torch
    with torch.cuda.stream(stream):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(replays):
            g.replay()
        e1.record(stream)
    stream.synchronize()
    return e0.elapsed_time(e1) * 1e3 / (replays * reps_per_graph)


def graph_us_samples(g, stream, reps_per_graph, replays):
    """Device time per call (us) of each of `replays` replays of a captured
    graph: every replay is bracketed by its own CUDA events on the graph's
    stream (one warm-up replay first)."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(replays)]
    with torch.cuda.stream(stream):
        g.replay()
        for a, b in evs:
            a.record(stream)
            g.replay()
            b.record(stream)
    stream.synchronize()
    return [a.elapsed_time(b) * 1e3 / reps_per_graph for a, b in evs]


def spread(samples):
    """median / p10 / p90 / mean of a list of per-call times (us)."""
    v = sorted(samples)
    n = len(v)

    def q(f):  # nearest-rank percentile
        return v[min(n - 1, max(0, int(round(f * (n - 1)))))]
    return {"median": round(statistics.median(v), 3), "p10": round(q(0.10), 3), "p90": round(q(0.90), 3),
            "mean": round(statistics.mean(v), 3), "reps": n}


STAT_REPLAYS = 25  # replays per figure: >= 20 samples for median / p10 / p90


def cpu_model() -> str:
    """The host CPU's model name (lscpu, else /proc/cpuinfo)."""
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for line in out.splitlines():
            if line.lower().startswith("model name"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    try:
        for line in open("/proc/cpuinfo"):
            if line.lower().startswith("model name"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def read_ceiling_gbs(dev, stream, gib=2):
    """A read-only streaming ceiling for this GPU: the best of a few full
    reductions (torch amax, int32) over a buffer of `gib` GiB, larger than L2;
    bytes read / device time.  A measurement aid, not part of the library."""
    import torch
    n = gib * (1 << 30) // 4
    buf = torch.ones(n, dtype=torch.int32, device=dev)
    best = 0.0
    with torch.cuda.stream(stream):
        torch.amax(buf)
        for _ in range(5):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            torch.amax(buf)
            b.record(stream)
            stream.synchronize()
            best = max(best, n * 4 / (a.elapsed_time(b) * 1e-3) / 1e9)
    del buf
    torch.cuda.empty_cache()
    return best


def run_ours(args, rank, world, local_rank):
    import torch
    import weight_only_quantized_qmv_b200 as q
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    q.lib()
    formats = tuple(args.formats)
    x, ops, enc_ms = build_workload(dev, formats)
    torch.cuda.synchronize()
    # the decode loop's weights are fixed: let each launch stream its weights
    # while its predecessor drains (no work in the timed region writes them)
    q.set_weight_prefetch(not args.no_prefetch)
    fmt_id = {"fp4": q.FMT_FP4, "int4": q.FMT_INT4, "int4km": q.FMT_INT4KM, "int8": q.FMT_INT8}
    outs = {f: torch.empty((1, N_HEAD), dtype=torch.float32, device=dev) for f in formats}
    stream = torch.cuda.Stream(device=dev)

    def launch(f):
        c, a = ops[f]
        q.matvec(fmt_id[f], c, a, x, out=outs[f], stream=stream)

    def step():
        for f in formats:
            launch(f)

    # A decode step runs as a CUDA graph (the deployment form): one replay =
    # one matvec per format, back to back on one stream.
    step_graph = capture(step, stream, 1)

    dist = world > 1
    if dist:
        import torch.distributed as tdist

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step_graph.replay()
    torch.cuda.synchronize()
    if dist:
        tdist.barrier()
    torch.cuda.synchronize()

    cvd = os.environ.get("CUDA_VISIBLE_DEVICES")
    gpu_index = cvd.split(",")[local_rank].strip() if cvd else str(local_rank)
    with ClockSampler(gpu_index) as clk:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            t_start.record(stream)
            for _ in range(args.steps):
                step_graph.replay()
            t_end.record(stream)
        torch.cuda.synchronize()
    if dist:
        tdist.barrier()
    torch.cuda.synchronize()
    clocks = clk.summary()
    total_ms = t_start.elapsed_time(t_end)
    flags = q.status_fetch(stream)
    if flags:
        raise RuntimeError(f"kernel status flags 0x{flags:x}")

    ms_step = total_ms / args.steps
    if dist:
        ms_step = max_over_ranks(ms_step, dev)
    bytes_step = sum(algorithmic_bytes(f, N_HEAD, K_HEAD, 1) for f in formats)
    value = whole_job_gbs(bytes_step, world, ms_step)

    # per-format kernel time: graphs of 10 back-to-back launches of one
    # format, each replay timed with its own events (median / p10 / p90)
    peak, peak_src = hbm_peak()
    read_ceiling = None if args.no_extras else read_ceiling_gbs(dev, stream)
    per_fmt = {}
    for f in formats:
        g = capture(lambda f=f: launch(f), stream, 10)
        st = spread(graph_us_samples(g, stream, 10, STAT_REPLAYS))
        del g
        us = st["median"]
        nb = algorithmic_bytes(f, N_HEAD, K_HEAD, 1)
        gbs = nb / (us * 1e-6) / 1e9
        per_fmt[f] = {"us": us, "us_p10": st["p10"], "us_p90": st["p90"], "reps": st["reps"], "gbs": round(gbs, 1),
                      "frac_of_measured_hbm": round(gbs / peak, 4), "frac_of_8tbs": round(gbs / 8000.0, 4),
                      "frac_of_read_ceiling": round(gbs / read_ceiling, 4) if read_ceiling else None,
                      "bytes": nb}
    dom = max(formats, key=lambda f: per_fmt[f]["us"])
    roof = {"bound": "hbm", "kernel": f"mv_kernel<{dom}> lm_head 248320x2048 B=1",
            "achieved": per_fmt[dom]["gbs"], "peak": peak, "unit": "GB/s",
            "frac": round(per_fmt[dom]["gbs"] / peak, 4), "peak_source": f"{peak_src} (hbm copy)",
            "traffic": profiled_traffic(dom), "algorithmic_bytes": per_fmt[dom]["bytes"],
            "timing": f"median of {STAT_REPLAYS} replays of a graph of 10 launches, CUDA events per replay"}

    # the same step launched call by call (no graph), for context
    with torch.cuda.stream(stream):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_plain = max(10, min(300, args.steps // 10))
        e0.record(stream)
        for _ in range(n_plain):
            step()
        e1.record(stream)
    torch.cuda.synchronize()
    plain_us = e0.elapsed_time(e1) * 1e3 / n_plain

    # extra measurements (outside the timed region): batch 4 / 16 verify, the int4km decode step
    extra = measure_batches(q, ops, dev, stream) if not args.no_extras and "fp4" in formats else None
    dstep = (measure_decode_step(q, ops["int4km"][0], ops["int4km"][1], dev, stream)
             if not args.no_extras and "int4km" in formats else None)
    amax = None if args.no_extras else measure_argmax(q, ops, fmt_id, x, dev, stream, formats)
    nxt = None if args.no_extras else measure_next_formats(q, x, dev, stream, peak)

    # the same-box fp16 lm_head matvec (the pages' per-op comparison) and the
    # int8 head at its own shape
    fp16 = None if args.no_extras else measure_fp16_head(dev, stream, per_fmt)
    c2 = None if args.no_extras else measure_int8_head_c2(q, dev, stream, peak)

    # end to end through the C ABI with host buffers: H2D x, the matvecs, D2H
    # y, all on the step's stream; the step's outputs are the check
    ref_outs = {}
    with torch.cuda.stream(stream):
        step_graph.replay()
    stream.synchronize()
    for f in formats:
        ref_outs[f] = outs[f].cpu()
    e2e = None if args.no_extras else measure_e2e(q, ops, fmt_id, x, dev, stream, formats, ref_outs,
                                                    steps=min(200, max(20, args.steps // 10)))

    return {
        "ms_per_step": ms_step, "value": value, "per_fmt": per_fmt, "roofline": roof, "clocks": clocks,
        "encode_ms": enc_ms, "batches": extra, "e2e": e2e, "bytes_step": bytes_step,
        "gpu_launches": len(formats) * args.steps, "step_us_without_graph": round(plain_us, 2),
        "decode_step_int4km": dstep, "argmax_b1": amax, "next_formats": nxt, "fp16_head": fp16,
        "int8_head_130560": c2, "read_ceiling_gbs": round(read_ceiling, 1) if read_ceiling else None,
    }


def measure_fp16_head(dev, stream, per_fmt):
    """The same head in fp16 on this GPU: torch (cuBLAS) y = x W^T with W
    float16 [248320, 2048] (seeded N(0, 0.02)), batch 1, graphs of 10 calls.
    Bytes: W + x + y (fp16), ~1018 MB.  The ratios are the B200 counterpart
    of the pages' per-op 'int4km vs fp16' figure."""
    import torch
    from weight_only_quantized_qmv_b200 import synth
    g = synth.generator(3, dev)
    W16 = synth.weights(N_HEAD, K_HEAD, g)[0].to(torch.float16)
    x16 = synth.activations(1, K_HEAD, g)
    y16 = torch.empty((1, N_HEAD), dtype=torch.float16, device=dev)
    gr = capture(lambda: torch.matmul(x16, W16.t(), out=y16), stream, 10)
    st = spread(graph_us_samples(gr, stream, 10, STAT_REPLAYS))
    del gr, W16
    torch.cuda.empty_cache()
    nb = N_HEAD * K_HEAD * 2 + K_HEAD * 2 + N_HEAD * 2
    return {"us": st["median"], "us_p10": st["p10"], "us_p90": st["p90"], "bytes": nb,
            "gbs": round(nb / (st["median"] * 1e-6) / 1e9, 1), "kernel": "torch.matmul (cuBLAS), fp16",
            "speedup_vs_fp16": {f: round(st["median"] / v["us"], 3) for f, v in per_fmt.items()}}


def measure_int8_head_c2(q, dev, stream, peak):
    """The int8 head at its own shape (130560 x 2048, N(0, 0.02), clip 1.0):
    encode (after a warm-up launch) and the batch-1 matvec, timed apart."""
    import torch
    from weight_only_quantized_qmv_b200 import synth
    N = 130560
    g = synth.generator(0, dev)
    W, _ = synth.weights(N, K_HEAD, g)
    x = synth.activations(1, K_HEAD, g)
    q.encode_int8(W[:256].contiguous())
    enc = []
    for _ in range(3):
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        codes, scales = q.encode_int8(W)
        b.record()
        torch.cuda.synchronize()
        enc.append(a.elapsed_time(b))
    del W
    torch.cuda.empty_cache()
    out = torch.empty((1, N), dtype=torch.float32, device=dev)
    gr = capture(lambda: q.matvec_int8(codes, scales, x, out=out, stream=stream), stream, 10)
    st = spread(graph_us_samples(gr, stream, 10, STAT_REPLAYS))
    del gr
    if q.status_fetch(stream):
        raise RuntimeError("int8 head status flags")
    nb = algorithmic_bytes("int8", N, K_HEAD, 1)
    gbs = nb / (st["median"] * 1e-6) / 1e9
    return {"shape": [N, K_HEAD], "encode_ms": round(statistics.median(enc), 3),
            "encode_read_gbs": round(N * K_HEAD * 4 / (statistics.median(enc) * 1e-3) / 1e9, 1),
            "matvec_us": st["median"], "matvec_us_p10": st["p10"], "matvec_us_p90": st["p90"],
            "bytes": nb, "gbs": round(gbs, 1), "frac_of_measured_hbm": round(gbs / peak, 4)}


def measure_next_formats(q, x, dev, stream, peak):
    """The formats beyond the step's four, on the same head at batch 1 (graphs
    of 10 launches): affine int4, the mixed int4km + int8 outlier columns
    (64) and int8km (256-entry palettes per 32 rows, 20 Lloyd steps), all
    encoded on the GPU from the same synthetic weights (each encoder warmed
    up on a 64-row slice first)."""
    import torch
    from weight_only_quantized_qmv_b200 import synth
    g = synth.generator(0, dev)
    W, _ = synth.weights(N_HEAD, K_HEAD, g, n_outlier_cols=2)
    res = {}
    calls = {}
    enc = {}

    def timed(fn):
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        r = fn()
        b.record()
        torch.cuda.synchronize()
        return r, a.elapsed_time(b)

    q.encode_int4aff(W[:64].contiguous())
    q.encode_int4km_o8(W[:64].contiguous(), O8_COLS)
    q.encode_int8km(W[:64].contiguous())
    (c4a, a4a), enc["int4aff"] = timed(lambda: q.encode_int4aff(W))
    o8, enc["int4km_o8"] = timed(lambda: q.encode_int4km_o8(W, O8_COLS))
    (idx8, lut8), enc["int8km"] = timed(lambda: q.encode_int8km(W))
    del W
    torch.cuda.empty_cache()
    if q.status_fetch():
        raise RuntimeError("encoder status flags")
    out = torch.empty((1, N_HEAD), dtype=torch.float32, device=dev)
    calls["int4aff"] = lambda: q.matvec_int4aff(c4a, a4a, x, out=out, stream=stream)
    calls["int8km"] = lambda: q.matvec_int8km(idx8, lut8, x, out=out, stream=stream)
    calls["int4km_o8"] = lambda: q.matvec_int4km_o8(*o8, x, out=out, stream=stream)
    for f, fn in calls.items():
        gr = capture(fn, stream, 10)
        st = spread(graph_us_samples(gr, stream, 10, STAT_REPLAYS))
        del gr
        us = st["median"]
        nb = algorithmic_bytes(f, N_HEAD, K_HEAD, 1)
        gbs = nb / (us * 1e-6) / 1e9
        res[f] = {"us": us, "us_p10": st["p10"], "us_p90": st["p90"], "gbs": round(gbs, 1),
                  "frac_of_measured_hbm": round(gbs / peak, 4),
                  "bytes": nb, "encode_ms": round(enc[f], 2) if f in enc else None}
    res["int4km_o8"]["launches_per_call"] = 2
    res["int8km"]["weights"] = "GPU k-means fit (qmv_encode_int8km, 20 Lloyd steps)"
    return res


def measure_batches(q, ops, dev, stream):
    import torch
    from weight_only_quantized_qmv_b200 import synth
    g0 = synth.generator(7, dev)
    res = {}
    for B in (4, 16):
        x = synth.activations(B, K_HEAD, g0)
        out = torch.empty((B, N_HEAD), dtype=torch.float32, device=dev)
        c, a = ops["fp4"]
        g = capture(lambda: q.matvec_fp4(c, a, x, out=out, stream=stream), stream, 10)
        st = spread(graph_us_samples(g, stream, 10, STAT_REPLAYS))
        del g
        us = st["median"]
        res[f"fp4_b{B}"] = {"us": us, "us_p10": st["p10"], "us_p90": st["p90"],
                            "gbs": round(algorithmic_bytes("fp4", N_HEAD, K_HEAD, B) / (us * 1e-6) / 1e9, 1)}
    return res


def measure_argmax(q, ops, fmt_id, x, dev, stream, formats):
    """Greedy next token from the head: the fused matvec + argmax against the
    matvec followed by torch.argmax, per format at batch 1 (graphs of 10)."""
    import torch
    ws = q.argmax_workspace(dev)
    res = {}
    for f in formats:
        c, a = ops[f]
        idx = torch.empty(1, dtype=torch.int32, device=dev)
        val = torch.empty(1, dtype=torch.float32, device=dev)
        y = torch.empty((1, N_HEAD), dtype=torch.float32, device=dev)
        g1 = capture(lambda: q.matvec_argmax(fmt_id[f], c, a, x, ws, idx=idx, val=val, stream=stream), stream, 10)
        fused = graph_us(g1, stream, 10, 5)
        del g1

        def unfused():
            q.matvec(fmt_id[f], c, a, x, out=y, stream=stream)
            torch.argmax(y, dim=1)

        g2 = capture(unfused, stream, 10)
        plain = graph_us(g2, stream, 10, 5)
        del g2
        with torch.cuda.stream(stream):
            ref = int(torch.argmax(q.matvec(fmt_id[f], c, a, x, stream=stream), dim=1).item())
        res[f] = {"fused_us": round(fused, 2), "matvec_then_argmax_us": round(plain, 2),
                  "same_index": int(idx.item()) == ref}
    return res


DECODE_E, DECODE_TOPK, DECODE_H, DECODE_I, DECODE_LAYERS = 256, 8, 2048, 512, 10


def decode_step_weights(dev):
    """Stand-in int4km weights of the decode step (fitted shapes, random
    palettes and indices): 10 layers of q (4096x2048) and o (2048x4096), one
    routed-expert layer: gate and up [256, 512, 2048] stored as one stack
    [256, 1024, 2048] (each expert's gate rows, then its up rows) so that one
    gather launch serves both, and down [256, 2048, 512]."""
    from weight_only_quantized_qmv_b200 import synth
    g = synth.generator(11, dev)
    E, H, I = DECODE_E, DECODE_H, DECODE_I
    layers = []
    for _ in range(DECODE_LAYERS):
        ql, qi = synth.palette_tables(4096, H, g)
        ol, oi = synth.palette_tables(H, 4096, g)
        layers.append((qi, ql, oi, ol))
    gl, gi = synth.palette_tables(E * 2 * I, H, g)
    dl, di = synth.palette_tables(E * H, I, g)
    experts = (gi.view(E, 2 * I, H // 2), gl.view(E, 2 * I, 16), di.view(E, H, I // 2), dl.view(E, H, 16))
    return layers, experts, g


def decode_step_fn(q, layers, experts, lm_idx, lm_lut, B, dev, stream, g):
    """The decode step's 23 launches for B tokens (lm_head, 10 x (q, o),
    gate+up, down), as a closure on `stream`, and the number of distinct
    experts its routing selects."""
    import torch
    from weight_only_quantized_qmv_b200 import synth
    E, topk, H, I = DECODE_E, DECODE_TOPK, DECODE_H, DECODE_I
    gui, gul, di, dl = experts
    x_h = synth.activations(B, H, g)
    x_o = synth.activations(B, 4096, g)
    x_d = synth.activations(B, I, g, extra_shape=(topk,))
    ids = synth.routing(B, topk, E, g).to(dev)
    y_lm = torch.empty((B, lm_idx.shape[0]), dtype=torch.float32, device=dev)
    y_q = torch.empty((B, 4096), dtype=torch.float32, device=dev)
    y_o = torch.empty((B, H), dtype=torch.float32, device=dev)
    y_gu = torch.empty((B, topk, 2 * I), dtype=torch.float32, device=dev)
    y_d = torch.empty((B, topk, H), dtype=torch.float32, device=dev)

    def step():
        for qi, ql, oi, ol in layers:
            q.matvec_int4km(qi, ql, x_h, out=y_q, stream=stream)
            q.matvec_int4km(oi, ol, x_o, out=y_o, stream=stream)
        q.gather_matvec(q.FMT_INT4KM, gui, gul, ids, x_h, out=y_gu, stream=stream)
        q.gather_matvec(q.FMT_INT4KM, di, dl, ids, x_d, x_per_slot=True, out=y_d, stream=stream)
        q.matvec_int4km(lm_idx, lm_lut, x_h, out=y_lm, stream=stream)

    return step, len(set(ids.flatten().tolist()))


def measure_decode_step(q, lm_idx, lm_lut, dev, stream, reps=STAT_REPLAYS):
    """The int4km decode step of the workload list, timed as one CUDA graph per
    batch size: the 248320x2048 lm_head, 10 layers of q (4096x2048) and o
    (2048x4096), and one routed-expert layer (256 experts; gate and up
    512x2048 in one launch, down 2048x512; top-8 uniform routing).  Random palettes and
    indices of the fitted shapes; each launch reads fixed synthetic
    activations (the step's data flow between layers is not modelled)."""
    layers, experts, g = decode_step_weights(dev)
    E, topk, H, I = DECODE_E, DECODE_TOPK, DECODE_H, DECODE_I
    res = {}
    for B in (1, 8):
        step, n_exp = decode_step_fn(q, layers, experts, lm_idx, lm_lut, B, dev, stream, g)
        gph = capture(step, stream, 1)
        st = spread(graph_us_samples(gph, stream, 1, reps))
        del gph
        us = st["median"]
        dense = (algorithmic_bytes("int4km", N_HEAD, H, B)
                 + 10 * (algorithmic_bytes("int4km", 4096, H, B) + algorithmic_bytes("int4km", H, 4096, B)))
        expert = n_exp * (2 * (I * H // 2 + I * 32) + (H * I // 2 + H * 32))
        res[f"b{B}"] = {"us": us, "us_p10": st["p10"], "us_p90": st["p90"], "launches": 23,
                        "distinct_experts": n_exp, "bytes": dense + expert,
                        "gbs": round((dense + expert) / (us * 1e-6) / 1e9, 1)}
    return res


def measure_e2e(q, ops, fmt_id, x, dev, stream, formats, ref_outs, steps):
    """The step end to end through the public API with host buffers: per step
    the activations are copied in from pinned host memory and the four
    matvecs run on the step's stream; each output is copied back to pinned
    host memory on a second stream as soon as its matvec has finished (an
    event), overlapping the next matvec, and the step's stream waits for the
    copies before the step ends (and before the next step rewrites the
    outputs).  CUDA events on the step's stream bracket copy-in .. the last
    copy-out, the wall clock runs until the stream has drained, and the host
    copies of the last step are compared bit for bit with the graph step's
    outputs."""
    import torch
    x_host = x.cpu().pin_memory()
    y_host = {f: torch.empty((1, N_HEAD), dtype=torch.float32).pin_memory() for f in formats}
    x_dev = torch.empty_like(x)
    outs = {f: torch.empty((1, N_HEAD), dtype=torch.float32, device=dev) for f in formats}
    copy_stream = torch.cuda.Stream(device=dev)
    done = {f: torch.cuda.Event() for f in formats}

    def one():
        with torch.cuda.stream(stream):
            stream.wait_stream(copy_stream)  # the previous step's outputs are on the host
            x_dev.copy_(x_host, non_blocking=True)
            for f in formats:
                c, a = ops[f]
                q.matvec(fmt_id[f], c, a, x_dev, out=outs[f], stream=stream)
                done[f].record(stream)
                copy_stream.wait_event(done[f])
                with torch.cuda.stream(copy_stream):
                    y_host[f].copy_(outs[f], non_blocking=True)
            stream.wait_stream(copy_stream)  # the step ends with its outputs on the host

    for _ in range(5):
        one()
        stream.synchronize()
    for f in formats:
        y_host[f].zero_()
    times = []
    for _ in range(steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0 = time.perf_counter()
        with torch.cuda.stream(stream):
            e0.record(stream)
        one()
        with torch.cuda.stream(stream):
            e1.record(stream)
        stream.synchronize()
        times.append((e0.elapsed_time(e1), (time.perf_counter() - t0) * 1e3))
    checked = all(torch.equal(y_host[f], ref_outs[f]) for f in formats)
    if not checked:
        raise RuntimeError("e2e outputs differ from the graph step's outputs")
    ms_dev = statistics.median(t[0] for t in times)
    ms_wall = statistics.median(t[1] for t in times)
    bytes_step = sum(algorithmic_bytes(f, N_HEAD, K_HEAD, 1) for f in formats)
    return {"value": round(bytes_step / (ms_wall * 1e-3) / 1e9, 1), "unit": "GB/s",
            "ms_per_step_wall": round(ms_wall, 4), "ms_per_step_device": round(ms_dev, 4),
            "h2d_bytes_per_step": int(x_host.numel() * 2), "d2h_bytes_per_step": int(len(formats) * N_HEAD * 4),
            "steps": steps, "checked": checked,
            "how": "median per step; H2D x and 4 matvecs on the step's stream, each D2H y on a second stream after "
                   "its matvec (overlapping the next); wall clock until both drain; outputs equal the graph step's "
                   "bit for bit"}


# ----------------------------------------------------------------- CPU oracle

def oracle_encodings(W_rows):
    """The oracle's encodings of a row sample for the four formats (int4km:
    stand-in tables of the fitted shapes; the CPU fit of 16 centres per row
    is not part of the per-token path), with the encode times (s)."""
    import numpy as np
    import oracle
    enc, secs = {}, {}
    for f, fn in (("fp4", oracle.encode_fp4), ("int4", oracle.encode_int4), ("int8", oracle.encode_int8)):
        t0 = time.perf_counter()
        c, s, _ = fn(W_rows)
        secs[f] = time.perf_counter() - t0
        enc[f] = ({"fp4": oracle.FMT_FP4, "int4": oracle.FMT_INT4, "int8": oracle.FMT_INT8}[f], c, s)
    lut = np.sort(np.random.default_rng(0).standard_normal((W_rows.shape[0], 16)) * 0.02, axis=1).astype(np.float16)
    idx = np.random.default_rng(1).integers(0, 256, (W_rows.shape[0], K_HEAD // 2), dtype=np.uint8)
    enc["int4km"] = (oracle.FMT_INT4KM, idx, lut)
    return enc, secs


def oracle_sample(W_rows, x_np, seconds_target, enc=None):
    """Time the oracle's fp64 matvec on a row sample of the head for each
    format; returns (GB/s on the algorithmic-bytes definition, rows, threads,
    seconds, passes)."""
    import oracle
    if enc is None:
        enc, _ = oracle_encodings(W_rows)
    R = W_rows.shape[0]
    t0 = time.perf_counter()
    done = 0
    nbytes = 0
    while True:
        for f in FORMATS:
            fid, c, a = enc[f]
            oracle.matvec(fid, c, a, x_np, R, K_HEAD)
            nbytes += algorithmic_bytes(f, R, K_HEAD, 1)
        done += 1
        if time.perf_counter() - t0 >= seconds_target:
            break
    dt = time.perf_counter() - t0
    return nbytes / dt / 1e9, R, oracle.num_threads(), dt, done


def cpu_baseline(W, x, seconds=12.0, rows=8192):
    """The oracle on the host cores: encode (fp4, int4 with 11 clips, int8) and
    the fp64 matvec of all four formats on a row sample, the matvec on all
    cores (the reported value) and on one thread."""
    import oracle
    Wn = W[:rows].cpu().numpy()
    xn = x.cpu().numpy()
    enc, enc_s = oracle_encodings(Wn)
    gbs, R, thr, dt, passes = oracle_sample(Wn, xn, seconds, enc)
    n0 = oracle.num_threads()
    oracle.set_num_threads(1)
    try:
        gbs1, _, _, dt1, passes1 = oracle_sample(Wn, xn, 3.0, enc)
    finally:
        oracle.set_num_threads(n0)
    return {"value": round(gbs, 3), "unit": "GB/s", "cores": thr, "kind": "oracle", "cpu_model": cpu_model(),
            "single_thread_gbs": round(gbs1, 4),
            "encode_ms": {f: round(1e3 * v, 1) for f, v in enc_s.items()},
            "encode_read_gbs": {f: round(4.0 * R * K_HEAD / v / 1e9, 3) for f, v in enc_s.items()},
            "sample": f"fp64 oracle matvec, {R} of 248320 rows x 2048, all four formats, {passes} passes in "
                      f"{dt:.1f} s on {thr} threads and {passes1} in {dt1:.1f} s on one (bytes scaled by the "
                      f"algorithmic-bytes definition); encoders timed once on the same rows ({thr} threads)"}


def run_reference(args):
    """The reference arm: the CPU oracle as it stands, on the host cores, each
    step one bounded row-sample of the same workload."""
    import numpy as np
    import oracle
    from weight_only_quantized_qmv_b200 import synth
    import torch
    g = synth.generator(0, "cpu")
    budget_s = 150.0
    per_step_s = budget_s / max(1, args.steps + args.warmup)
    rows = 4096
    W, _ = synth.weights(rows, K_HEAD, g, n_outlier_cols=2)
    x = synth.activations(1, K_HEAD, g).numpy()
    Wn = W.numpy()
    # size the per-step row sample to the time budget
    probe_gbs, _, thr, _, _ = oracle_sample(Wn[:256], x, 0.5)
    bytes_per_row = sum(algorithmic_bytes(f, 1, K_HEAD, 1) for f in FORMATS)
    R = int(max(16, min(rows, probe_gbs * 1e9 * per_step_s / bytes_per_row)))
    enc = {}
    c, s, _ = oracle.encode_fp4(Wn[:R])
    enc["fp4"] = (oracle.FMT_FP4, c, s)
    c, s, _ = oracle.encode_int4(Wn[:R])
    enc["int4"] = (oracle.FMT_INT4, c, s)
    enc["int4km"] = (oracle.FMT_INT4KM, np.random.default_rng(1).integers(0, 256, (R, K_HEAD // 2), dtype=np.uint8),
                     np.sort(np.random.default_rng(0).standard_normal((R, 16)) * 0.02, axis=1).astype(np.float16))
    c, s, _ = oracle.encode_int8(Wn[:R])
    enc["int8"] = (oracle.FMT_INT8, c, s)

    def step():
        for f in FORMATS:
            fid, cc, aa = enc[f]
            oracle.matvec(fid, cc, aa, x, R, K_HEAD)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    bytes_step = sum(algorithmic_bytes(f, R, K_HEAD, 1) for f in FORMATS)
    value = bytes_step * args.steps / dt / 1e9
    sample = f"fp64 CPU oracle, {R} of 248320 rows x 2048 per format per step"
    return {
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"lm_head 248320x2048 batch 1, fp4+int4+int4km+int8 (row sample {R})",
                   "l2": "n/a (host)"},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": thr, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


# ----------------------------------------------------------------- main

PROFILE_CASES = ("fp4", "int4", "int4km", "int8", "int4aff", "int8km", "int4km_o8", "fp4_b16", "fp4_b16_tc",
                 "decode_step_b1", "decode_step_b8")


def profile_case(name: str) -> int:
    """A small case for a profiler: one format's matvec on 65536 x 2048
    weights (larger than L2, a few hundred MB on the device), encoded by the
    library, three launches at batch 1 (fp4_b16:
    batch 16 on the mma.sync kernel; fp4_b16_tc: on the tcgen05 kernel).
    Prints one line and exits."""
    import torch
    import weight_only_quantized_qmv_b200 as q
    from weight_only_quantized_qmv_b200 import synth
    N, K = 65536, K_HEAD
    if name.startswith("decode_step"):
        # the full decode step (23 launches: lm_head, 10 x (q, o), gate+up,
        # down), captured as a graph and replayed three times
        B = int(name[-1])
        dev = torch.device("cuda", 0)
        stream = torch.cuda.Stream(device=dev)
        layers, experts, g = decode_step_weights(dev)
        lm_lut, lm_idx = synth.palette_tables(N_HEAD, K, g)
        step, n_exp = decode_step_fn(q, layers, experts, lm_idx, lm_lut, B, dev, stream, g)
        q.set_weight_prefetch(True)
        gph = capture(step, stream, 1)
        with torch.cuda.stream(stream):
            for _ in range(3):
                gph.replay()
        stream.synchronize()
        flags = q.status_fetch()
        print(json.dumps({"profile_case": name, "launches_per_step": 23, "steps": 5, "distinct_experts": n_exp,
                          "flags": flags}), flush=True)
        return 1 if flags else 0
    g = synth.generator(0, "cuda")
    B = 16 if name.startswith("fp4_b16") else 1
    q.set_fp4_tensor_cores(name == "fp4_b16_tc")
    x = synth.activations(B, K, g)
    W, _ = synth.weights(N, K, g, n_outlier_cols=2)
    if name == "int8km":
        idx, lut = q.encode_int8km(W)
        run = lambda: q.matvec_int8km(idx, lut, x)
    else:
        if name == "int4km_o8":
            enc = q.encode_int4km_o8(W, O8_COLS)
            run = lambda: q.matvec_int4km_o8(*enc, x)
        else:
            fmt = name.split("_")[0]
            fid = {"fp4": q.FMT_FP4, "int4": q.FMT_INT4, "int4km": q.FMT_INT4KM, "int8": q.FMT_INT8,
                   "int4aff": q.FMT_INT4AFF}[fmt]
            encf = {"fp4": q.encode_fp4, "int4": q.encode_int4, "int4km": q.encode_int4km, "int8": q.encode_int8,
                    "int4aff": q.encode_int4aff}[fmt]
            c, a = encf(W)
            run = lambda: q.matvec(fid, c, a, x)
    del W
    for _ in range(3):
        y = run()
    torch.cuda.synchronize()
    flags = q.status_fetch()
    print(json.dumps({"profile_case": name, "N": N, "K": K, "B": B, "launches": 3,
                      "y_abs_sum": float(y.abs().sum()), "flags": flags}), flush=True)
    return 1 if flags else 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the CPU-oracle leg")
    ap.add_argument("--formats", nargs="+", choices=FORMATS, default=list(FORMATS),
                    help="weight formats in the step (default: all four, the benchmark workload)")
    ap.add_argument("--no-extras", action="store_true", help="skip the e2e and batch-4/16 measurements")
    ap.add_argument("--no-prefetch", action="store_true",
                    help="keep weight reads behind the preceding launch (qmv_set_weight_prefetch(0))")
    ap.add_argument("--profile-case", choices=PROFILE_CASES,
                    help="run one small case for a profiler (65536 x 2048, three launches) and exit")
    args = ap.parse_args()
    if args.profile_case:
        return profile_case(args.profile_case)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0

    import torch
    if world > 1:
        import datetime
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local_rank))
    try:
        r = run_ours(args, rank, world, local_rank)
    finally:
        pass
    out = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            from weight_only_quantized_qmv_b200 import synth
            g = synth.generator(0, "cuda")
            W, _ = synth.weights(8192, K_HEAD, g, n_outlier_cols=2)
            x = synth.activations(1, K_HEAD, g)
            cpu = cpu_baseline(W, x)
        out = {
            "metric": METRIC, "value": round(r["value"], 1), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(r["ms_per_step"], 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f16 operands, f32 accumulate", "data": "synthetic",
            "config": {"workload": "lm_head 248320x2048 batch 1; one matvec per format per step "
                                   f"({', '.join(args.formats)})",
                       "l2": "inputs larger than L2 (~1.1 GB read per step), no flush",
                       "launch": "the step is a CUDA graph replayed once per step",
                       "weight_prefetch": not args.no_prefetch,
                       "parallelism": "replicas" if world > 1 else "single GPU"},
            "per_format": r["per_fmt"], "roofline": r["roofline"], "cpu_baseline": cpu, "e2e": r["e2e"],
            "step_us_without_graph": r["step_us_without_graph"], "decode_step_int4km": r["decode_step_int4km"],
            "argmax_b1": r["argmax_b1"],
            "gpu_launches": r["gpu_launches"] * world, "clocks": r["clocks"], "encode_ms": r["encode_ms"],
            "batch_verify": r["batches"], "next_formats": r["next_formats"], "fp16_head": r["fp16_head"],
            "int8_head_130560": r["int8_head_130560"], "read_ceiling_gbs": r["read_ceiling_gbs"],
            "host_cpu": {"model": cpu_model(), "cores": os.cpu_count()},
        }
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as tdist
        tdist.barrier()
        tdist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
