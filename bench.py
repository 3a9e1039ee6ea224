#!/usr/bin/env python3
"""Benchmark of the KroQuant online activation quantizer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one pass of the whole hot path over one batch of each DiT-shaped
workload: the KroQuant quantizer, the SmoothQuant quantizer and the plain
MXFP4 quantizer, each on every layer input of PixArt-Sigma (M = 8192 tokens x
d = 1152 and 4608), SANA (2048 x 2240 and 5600, one shared factor set) and
FLUX (4608 x 3072 and 12288), bf16, seeded synthetic activations: 18 launches.
The headline value is the KroQuant quantizer's algorithmic HBM throughput,
2.53125 bytes per element (2 B bf16 in, 0.5 B codes, 1/32 B scale) over the
summed duration of its six launches; the same for SmoothQuant and plain MXFP4,
per workload and per layer, is reported beside it.

Timing: inputs resident in HBM and rotated over per-layer input sets so that
a set is read again only after >= 3x the L2 of other input; per (quantizer,
layer) a CUDA graph of min(K, 200) back-to-back launches; a round replays the
18 graphs in step order; CUDA events on the launching stream sit between
graph replays.  The clocks are spun up by untimed rounds that end right
before the timed region (the nvidia-smi sampler is started before them), and
the bounded-wait counter of the library must read 0 after the timed region.
Barrier + synchronize on both sides; max over ranks.  Multi-GPU: every rank
quantizes its own batch (weak scaling, no collective on the data path).

`--impl reference` times the CPU oracle (oracle/, plain C) on the host cores on
a bounded sample of the same workload and prints the same JSON line.

Besides the step line, the JSON carries the roofline of the dominant launch
(the KroQuant quantizer on the largest layer, FLUX d = 12288, with the DRAM
traffic of an ncu capture, valid for the kernel source it was taken on), the
end-to-end figure through host buffers (H2D, quantize and D2H pipelined over
three streams), the CPU-oracle baseline, the SM clocks sampled during the
timed region and the number of kernel launches.

Other modes (one JSON line each):
    --mode kernel --kernel K --shape MxD     one quantizer or variant at one shape
    --mode sweep [--kernels ...]             every shape of the sweep workload
    --mode sqnr                              quantisation-error proxy (SQNR)
    --mode gemm --shape MxNxK [--kernels v]  the W4A4 product, its tile configurations,
                                             and the chains quantize -> product and
                                             norm + quantize -> product
    --mode compare --kernels a,b --shapes MxD,...  several quantizers interleaved in one
                                             process, --reps rounds (one line per timing)
"""
from __future__ import annotations

import argparse
import hashlib
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "KroQuant quantizer HBM GB/s (bf16→MXFP4+E8M0) and % of B200 peak vs SQ"
BYTES_PER_ELEM = 2.0 + 0.5 + 1.0 / 32.0
WORKLOADS = ("pixart", "sana", "flux")
WORKLOAD_NAMES = {"pixart": "PixArt-Sigma", "sana": "SANA", "flux": "FLUX"}
GRAPH_STEPS = 200          # launches per captured graph
E2E_CHUNKS = 4             # row chunks per layer in the end-to-end (host buffer) pipeline
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0
KERNEL_SOURCES = [os.path.join(ROOT, "w4a4_mxfp4_post_b200", "csrc", "kroquant.cu")]

# DRAM traffic per launch of the dominant kernel (KroQuant quantizer on the
# largest layer, FLUX 4608 x 12288), from one ncu capture, valid only for the kernel source it was taken
# on (sha256 prefix of kernel_source_text: the kernel, its helpers and its
# launch path).  Updated after each capture.
TRAFFIC = {"source_sha": "8cd74afaa15c5b7a", "bytes_per_launch": 127987968.0,
           "capture": "ncu --set full, kq_packed_kernel, 4608x12288, dram__bytes_read.sum + dram__bytes_write.sum"}


# The code that determines the dominant kernel (KroQuant variant 2): the
# library source up to the end of kq_packed_kernel (which holds every device
# helper it uses) and the host functions that size and launch it.
KERNEL_START = "kq_packed_kernel(const uint4 *__restrict__ act"
LAUNCH_FUNCS = ("int sm_count(", "Geometry pinned_geometry(", "int resident_threads(",
                "int launch_pinned(const char *fn, KernelId id", "void launch(void (*kernel)", "int kq_launch(")


def _function_text(src: str, head: str) -> str:
    """From the line that starts with `head` to the next closing brace in column 0."""
    i = src.index("\n" + head) + 1
    j = src.index("\n}\n", i)
    return src[i:j + 3]


def kernel_source_text(src: str) -> str:
    i = src.index("\n" + KERNEL_START)
    j = src.index("\n}\n", i)
    return src[:j + 3] + "".join(_function_text(src, f) for f in LAUNCH_FUNCS)


def source_sha() -> str:
    with open(KERNEL_SOURCES[0]) as fh:
        src = fh.read()
    return hashlib.sha256(kernel_source_text(src).encode()).hexdigest()[:16]


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            v = float(json.load(fh)["hbm_gbs"])
        return v, "measured (MEASURED_PEAKS.json hbm_gbs, copy bandwidth)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s, earlier pool measurement)"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu: str):
        self.gpu = gpu
        self.proc = None
        self.lines = []
        self._t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self._t = threading.Thread(target=self._read, daemon=True)
        self._t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self._t:
            self._t.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [t.strip() for t in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- distributed
def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus and world > 1:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    pg = None
    if world > 1:
        import datetime

        import torch

        torch.cuda.set_device(local)

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        pg = dist
    return rank, local, world, pg


def allreduce_max(pg, values, device):
    if pg is None:
        return values
    import torch

    t = torch.tensor(values, dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return t.tolist()


def allreduce_sum(pg, values, device):
    if pg is None:
        return values
    import torch

    t = torch.tensor(values, dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.SUM)
    return t.tolist()


def barrier(pg):
    if pg is not None:
        pg.barrier()


# ----------------------------------------------------------------------------- inputs
def workload_inputs(seed_offset: int = 0, world: int = 1, rank: int = 0):
    """Layer inputs of every benchmark workload: the whole batch (world == 1), or rank's rows of it."""
    from w4a4_mxfp4_post_b200 import shard, synth

    layers = []
    for wl in WORKLOADS:
        for (M, d, model, shared, seed) in synth.workload_layers(wl):
            rows = shard.row_range(M, world, rank) if world > 1 else None
            x = synth.activation(model, M, d, seed + seed_offset, rows=rows)
            M = x.shape[0]
            F = synth.factors(d // 32, seed + seed_offset, shared=shared)
            m = synth.sq_multipliers(x)
            layers.append({"workload": wl, "M": M, "d": d, "x": x, "F": F, "m": m, "shared": shared})
    return layers


def workload_text():
    from w4a4_mxfp4_post_b200 import synth

    parts = []
    for wl in WORKLOADS:
        w = synth.WORKLOADS[wl]
        parts.append(f"{WORKLOAD_NAMES[wl]} M={w['M']} x d in {{{', '.join(str(d) for d in w['ds'])}}}"
                     + (" (one shared factor set)" if w["factors"] == "shared" else ""))
    return "DiT layer inputs: " + "; ".join(parts) + "; bf16 -> MXFP4 (E2M1 codes + E8M0 scales)"


# ----------------------------------------------------------------------------- CPU oracle timing
def time_oracle(layers, seconds: float, rows_per_pass=None):
    """Run the oracle (KQ, SQ, MX on every layer) over row samples for ~`seconds`."""
    import oracle

    t_kq = 0.0
    t_all = 0.0
    kq_bytes = 0.0
    passes = 0
    start = time.perf_counter()
    while True:
        for L in layers:
            M = L["M"] if rows_per_pass is None else min(L["M"], rows_per_pass)
            x = L["x"][:M]
            t0 = time.perf_counter()
            oracle.kq_quantize(x, L["F"], shared=L["shared"])
            t1 = time.perf_counter()
            oracle.sq_quantize(x, L["m"])
            oracle.mx_quantize(x)
            t2 = time.perf_counter()
            t_kq += t1 - t0
            t_all += t2 - t0
            kq_bytes += BYTES_PER_ELEM * M * L["d"]
        passes += 1
        if time.perf_counter() - start >= seconds:
            break
    return {"kq_gbs": kq_bytes / t_kq / 1e9, "passes": passes, "t_kq": t_kq, "t_all": t_all,
            "threads": oracle.num_threads()}


# ----------------------------------------------------------------------------- GPU arm
def gpu_arm(args, rank, local, world, pg):
    import torch

    import w4a4_mxfp4_post_b200 as kq

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    # weak: every rank quantizes its own batch; strong: the ranks split one batch by rows
    if args.scaling == "weak":
        layers = workload_inputs(seed_offset=rank)
    else:
        layers = workload_inputs(world=world, rank=rank)
    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20))

    # device buffers: per layer, enough input sets that a set is reused only
    # after >= 3x the L2 of other input has streamed by (and at least 4)
    layer_sets = []
    for L in layers:
        M, d = L["M"], L["d"]
        set_bytes = M * d * 2
        nsets = max(4, math.ceil(3 * l2 / set_bytes) + 1)
        x0 = torch.from_numpy(L["x"].view(np.int16)).to(dev).view(torch.bfloat16)
        xs = torch.empty((nsets, M, d), dtype=torch.bfloat16, device=dev)
        xs[:] = x0
        layer_sets.append({
            "n": nsets, "x": xs,
            "codes": torch.empty((nsets, M, d // 2), dtype=torch.uint8, device=dev),
            "scales": torch.empty((nsets, M, d // 32), dtype=torch.uint8, device=dev),
            "F": torch.from_numpy(L["F"]).to(dev), "m": torch.from_numpy(L["m"]).to(dev),
            "shared": L["shared"],
        })
    resident = sum(ls["n"] * L["M"] * L["d"] * 2 for ls, L in zip(layer_sets, layers))

    def launch(q, li, i, stream):
        ls = layer_sets[li]
        k = i % ls["n"]
        x, c, sc = ls["x"][k], ls["codes"][k], ls["scales"][k]
        if q == "kq":
            (kq.kq_quantize_shared if ls["shared"] else kq.kq_quantize)(x, ls["F"], c, sc, stream=stream)
        elif q == "sq":
            kq.sq_quantize(x, ls["m"], c, sc, stream=stream)
        else:
            kq.mx_quantize(x, c, sc, stream=stream)

    quantizers = ("kq", "sq", "mx")
    n_layers = len(layers)
    pairs = [(q, li) for li in range(n_layers) for q in quantizers]
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize(dev)
    kq.kq_wait_timeouts(reset=True)
    # warm-up steps (eager)
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            for q, li in pairs:
                launch(q, li, i, stream)
    stream.synchronize()

    # One CUDA graph per (quantizer, layer) holding S back-to-back launches;
    # a round replays the 18 graphs in step order, so K steps = K/S rounds
    # (the last round shorter).  Events sit only between graph replays.
    K = args.steps
    S = min(GRAPH_STEPS, K)
    full, tail = divmod(K, S)

    def capture(q, li, n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                launch(q, li, i, stream)
        return g

    graphs = {pl: capture(*pl, S) for pl in pairs}
    tails = {pl: capture(*pl, tail) for pl in pairs} if tail else {}
    for g in list(graphs.values()) + list(tails.values()):
        g.replay()
    stream.synchronize()

    rounds = [graphs] * full + ([tails] if tail else [])
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(pairs) + 1)] for _ in rounds]
    uuid = getattr(props, "uuid", None)
    gpu_id = f"GPU-{uuid}" if uuid is not None else str(local)
    clocks = ClockSampler(gpu_id) if rank == 0 else None
    if clocks:
        clocks.start()
    barrier(pg)
    # untimed rounds until the SM and HBM clocks have left their idle states;
    # they run right up to the timed region, so no launch of it starts cold
    t_end = time.perf_counter() + SPINUP_S
    with torch.cuda.stream(stream):
        while time.perf_counter() < t_end:
            for pl in pairs:
                graphs[pl].replay()
            stream.synchronize()
    barrier(pg)
    with torch.cuda.stream(stream):
        for r, gs in enumerate(rounds):
            evs[r][0].record(stream)
            for k, pl in enumerate(pairs):
                gs[pl].replay()
                evs[r][k + 1].record(stream)
    torch.cuda.synchronize(dev)
    barrier(pg)
    clk = clocks.stop() if clocks else None
    timeouts = kq.kq_wait_timeouts(reset=True)
    if timeouts:
        raise SystemExit(f"{timeouts} bounded waits of the library gave up during the benchmark: "
                         "its launches did not finish their work, the timing is void")

    total_ms = evs[0][0].elapsed_time(evs[-1][-1])
    per = {q: [0.0] * n_layers for q in quantizers}
    for r in range(len(rounds)):
        for k, (q, li) in enumerate(pairs):
            per[q][li] += evs[r][k].elapsed_time(evs[r][k + 1])
    us_local = {q: [1e3 * v / K for v in per[q]] for q in per}   # mean us per launch, gaps in the graph included

    # max over ranks of every per-launch mean and of the step time
    flat = [total_ms] + [us_local[q][li] for q in quantizers for li in range(n_layers)]
    vals = allreduce_max(pg, flat, dev)
    total_ms_max = vals[0]
    us = {q: vals[1 + qi * n_layers: 1 + (qi + 1) * n_layers] for qi, q in enumerate(quantizers)}
    elems = [L["M"] * L["d"] for L in layers]
    qbytes = sum(BYTES_PER_ELEM * e for e in elems)
    all_bytes = allreduce_sum(pg, [qbytes], dev)[0]          # units all ranks processed per step
    qt = {q: sum(us[q]) for q in quantizers}
    gbs = {q: all_bytes / (qt[q] * 1e-6) / 1e9 for q in quantizers}
    peak, peak_src = measured_peak()

    def rate(nbytes, t_us):
        g = nbytes / (t_us * 1e-6) / 1e9
        return {"gbs": round(g, 1), "frac_of_peak": round(g / peak, 4)}

    per_workload = {}
    for wl in WORKLOADS:
        idx = [li for li, L in enumerate(layers) if L["workload"] == wl]
        wb = sum(BYTES_PER_ELEM * elems[li] for li in idx)
        entry = {"layers": {f"{layers[li]['M']}x{layers[li]['d']}": {
            q: {"us": round(us[q][li], 3), **rate(BYTES_PER_ELEM * elems[li], us[q][li])} for q in quantizers}
            for li in idx}}
        for q in quantizers:
            entry[q] = rate(wb, sum(us[q][li] for li in idx))
        entry["kq_time_vs_sq"] = round(sum(us["kq"][li] for li in idx) / sum(us["sq"][li] for li in idx), 4)
        per_workload[WORKLOAD_NAMES[wl]] = entry

    # dominant kernel: the KroQuant launch on the largest layer
    dom = int(np.argmax(elems))
    dom_bytes = BYTES_PER_ELEM * elems[dom]
    achieved = dom_bytes / (us["kq"][dom] * 1e-6) / 1e9
    sha = source_sha()
    traffic = TRAFFIC["bytes_per_launch"] if TRAFFIC["source_sha"] == sha else None

    # end-to-end: pinned host input -> device -> kq_quantize -> host codes + scales
    e2e = e2e_kq(args, layers, dev, stream, kq, pg, world)

    out = {
        "metric": METRIC,
        "value": round(gbs["kq"], 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms_max / K, 6),
        "higher_is_better": True,
        "scaling": args.scaling,
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded DiT-shaped activations with per-channel outliers; no trained weights)",
        "config": {
            "workload": workload_text(),
            "layers": [f"{L['M']}x{L['d']}" for L in layers],
            "quantizers_per_step": list(quantizers),
            "l2": f"inputs larger than L2: per layer {[ls['n'] for ls in layer_sets]} rotating input sets "
                  f"({resident / 2**20:.0f} MiB resident, L2 {l2 / 2**20:.0f} MiB); a set is reused only after "
                  ">= 3x L2 of other input",
            "timing": f"per (quantizer, layer) a CUDA graph of {S} back-to-back launches; a step's 18 graphs "
                      "replayed in order; CUDA events between replays on the launching stream; untimed "
                      f"spin-up rounds ({SPINUP_S} s) end right before the timed region",
            "parallelism": f"dp{world} ({'independent batches' if args.scaling == 'weak' else 'row shards of one batch'}"
                           ", no collective on the data path)",
        },
        "kernels": {
            q: {"gbs": round(gbs[q], 1), "frac_of_peak": round(gbs[q] / peak, 4),
                "frac_of_8tbs_spec": round(gbs[q] / SPEC_HBM_GBS, 4)}
            for q in quantizers
        },
        "workloads": per_workload,
        "kq_time_vs_sq": round(qt["kq"] / qt["sq"], 4),
        "roofline": {"bound": "hbm", "kernel": f"kq_quantize {layers[dom]['M']}x{layers[dom]['d']}",
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "algorithmic_bytes_per_launch": dom_bytes, "peak_source": peak_src},
        "e2e": e2e,
        "gpu_launches": K * len(pairs),
        "wait_timeouts": timeouts,
        "clocks": clk,
        "kernel_source_sha": sha,
    }
    return out


def e2e_kq(args, layers, dev, stream, kq, pg, world):
    """KroQuant through the public API with host buffers, per step: every layer's
    bf16 input goes host -> device, is quantized, and its codes and scales go
    device -> host.  The rows of a layer are pipelined in E2E_CHUNKS chunks over
    three streams (H2D, quantize, D2H), so a chunk's D2H overlaps the next
    chunk's H2D (PCIe is full duplex); events order every reuse of a device
    chunk across steps.  All copies are inside the timed region."""
    import torch

    host = []
    for L in layers:
        M, d = L["M"], L["d"]
        host.append({
            "x": torch.from_numpy(L["x"].view(np.int16)).view(torch.bfloat16).pin_memory(),
            "codes": torch.empty((M, d // 2), dtype=torch.uint8).pin_memory(),
            "scales": torch.empty((M, d // 32), dtype=torch.uint8).pin_memory(),
            "dx": torch.empty((M, d), dtype=torch.bfloat16, device=dev),
            "dc": torch.empty((M, d // 2), dtype=torch.uint8, device=dev),
            "ds": torch.empty((M, d // 32), dtype=torch.uint8, device=dev),
            "F": torch.from_numpy(L["F"]).to(dev), "shared": L["shared"],
            "chunks": [(M * c // E2E_CHUNKS, M * (c + 1) // E2E_CHUNKS) for c in range(E2E_CHUNKS)],
        })
    s_in = torch.cuda.Stream(device=dev)
    s_out = torch.cuda.Stream(device=dev)
    # per (layer, chunk): the quantize that last read dx, the D2H that last read dc/ds
    last_q = {}
    last_out = {}

    def one():
        for li, h in enumerate(host):
            fn = kq.kq_quantize_shared if h["shared"] else kq.kq_quantize
            for ci, (r0, r1) in enumerate(h["chunks"]):
                key = (li, ci)
                if key in last_q:
                    s_in.wait_event(last_q[key])
                with torch.cuda.stream(s_in):
                    h["dx"][r0:r1].copy_(h["x"][r0:r1], non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
                stream.wait_event(ev_in)
                if key in last_out:
                    stream.wait_event(last_out[key])
                fn(h["dx"][r0:r1], h["F"], h["dc"][r0:r1], h["ds"][r0:r1], stream=stream)
                ev_q = torch.cuda.Event()
                ev_q.record(stream)
                last_q[key] = ev_q
                s_out.wait_event(ev_q)
                with torch.cuda.stream(s_out):
                    h["codes"][r0:r1].copy_(h["dc"][r0:r1], non_blocking=True)
                    h["scales"][r0:r1].copy_(h["ds"][r0:r1], non_blocking=True)
                ev_o = torch.cuda.Event()
                ev_o.record(s_out)
                last_out[key] = ev_o

    n = max(3, min(args.e2e_steps, args.steps))
    for _ in range(3):
        one()
    torch.cuda.synchronize(dev)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    barrier(pg)
    a.record(s_in)
    for _ in range(n):
        one()
    # the end waits for all three streams
    s_in.wait_stream(stream)
    s_in.wait_stream(s_out)
    b.record(s_in)
    b.synchronize()
    ms = allreduce_max(pg, [a.elapsed_time(b)], dev)[0]
    elems = sum(L["M"] * L["d"] for L in layers)
    h2d = sum(L["M"] * L["d"] * 2 for L in layers)
    d2h = sum(L["M"] * (L["d"] // 2 + L["d"] // 32) for L in layers)
    return {"value": round(world * BYTES_PER_ELEM * elems * n / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n,
            "path": f"pinned host bf16 -> cudaMemcpyAsync -> kq_quantize -> cudaMemcpyAsync -> pinned host, "
                    f"{E2E_CHUNKS} row chunks per layer pipelined over H2D / quantize / D2H streams"}


def cpu_baseline_block(layers, seconds):
    r = time_oracle(layers, seconds)
    return {"value": round(r["kq_gbs"], 4), "unit": "GB/s", "cores": r["threads"], "kind": "oracle",
            "sample": f"{r['passes']} full passes of the workload (KQ, SQ, MX on all six layers), "
                      f"{r['t_all']:.1f} s of oracle time; value = KQ bytes / KQ time"}


# ----------------------------------------------------------------------------- reference arm
def reference_arm(args, rank, world):
    """The CPU oracle as the reference implementation, on the host cores."""
    import oracle

    if rank != 0:
        return None
    layers = workload_inputs()
    oracle.kq_quantize(layers[0]["x"][:8], layers[0]["F"])         # load / warm
    # rows per step so that (warmup + steps) steps take about `budget` seconds
    t0 = time.perf_counter()
    probe = time_oracle(layers, 0.0, rows_per_pass=64)
    per_row = (time.perf_counter() - t0) / 64
    budget = args.ref_seconds
    rows = int(max(1, min(max(L["M"] for L in layers), budget / max(1, args.steps + args.warmup) / per_row)))
    for _ in range(args.warmup):
        time_oracle(layers, 0.0, rows_per_pass=rows)
    t_kq = 0.0
    kq_bytes = 0.0
    t_all = 0.0
    for _ in range(args.steps):
        r = time_oracle(layers, 0.0, rows_per_pass=rows)
        t_kq += r["t_kq"]
        t_all += r["t_all"]
        kq_bytes += sum(BYTES_PER_ELEM * min(L["M"], rows) * L["d"] for L in layers)
    value = kq_bytes / t_kq / 1e9
    del probe
    return {
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * t_all / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": workload_text(), "sample_rows_per_layer_per_step": rows},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"{rows} rows of each layer per step (KQ, SQ, MX), {args.steps} steps"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


SPINUP_S = 0.5


def _replay_seconds(g, stream):
    import torch

    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        g.replay()
        b.record(stream)
    b.synchronize()
    return a.elapsed_time(b) * 1e-3


class RotatingInputs:
    """Device inputs of one [M, d] layer, split into sets that rotate past the L2.

    One allocation holds `nsets` disjoint input sets (and their outputs) whose
    total is >= 3x the L2, capped by `budget_bytes`; launch i reads set
    i mod nsets, so no launch finds its input in the L2 from an earlier one.
    """

    def __init__(self, M, d, dev, l2, budget_bytes=None):
        import torch

        from w4a4_mxfp4_post_b200 import synth

        self.M, self.d = M, d
        x = synth.activation("pixart", M, d, 4)
        F = synth.factors(d // 32, 4)
        m = synth.sq_multipliers(x)
        set_bytes = M * d * 2 + M * (d // 2) + M * (d // 32)
        budget = budget_bytes or max(3 * l2, 2 * set_bytes)
        self.nsets = max(2, min(1024, math.ceil(budget / set_bytes)))
        self.xs = torch.empty((self.nsets, M, d), dtype=torch.bfloat16, device=dev)
        self.xs[:] = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
        self.cs = torch.empty((self.nsets, M, d // 2), dtype=torch.uint8, device=dev)
        self.ss = torch.empty((self.nsets, M, d // 32), dtype=torch.uint8, device=dev)
        self.F = torch.from_numpy(F).to(dev)
        self.m = torch.from_numpy(m).to(dev)
        self.P = torch.from_numpy(synth.lu_params(d // 32, 4)).to(dev)
        g, b = synth.adaln(2 if M % 2 == 0 else 1, d, 4)
        self.gamma, self.beta = torch.from_numpy(g).to(dev), torch.from_numpy(b).to(dev)


def time_launches(kind, inp, launches, warmup, stream, graph=True):
    """Mean device time (us) per launch over `launches` back-to-back launches.

    With graph=True the launches are captured in one CUDA graph and its second
    replay is timed by two events around it (inter-launch gaps included).
    """
    import torch

    import w4a4_mxfp4_post_b200 as kq

    def launch(i):
        k = i % inp.nsets
        if kind == "kq":
            kq.kq_quantize(inp.xs[k], inp.F, inp.cs[k], inp.ss[k], stream=stream)
        elif kind == "sq":
            kq.sq_quantize(inp.xs[k], inp.m, inp.cs[k], inp.ss[k], stream=stream)
        elif kind == "mx":
            kq.mx_quantize(inp.xs[k], inp.cs[k], inp.ss[k], stream=stream)
        elif kind == "norm_kq":
            kq.norm_kq_quantize(inp.xs[k], inp.gamma, inp.beta, inp.F, 1e-6, False, inp.cs[k], inp.ss[k], stream=stream)
        elif kind.startswith("norm_kq_v"):
            kq.norm_kq_quantize_variant(int(kind[9:]), inp.xs[k], inp.gamma, inp.beta, inp.F, 1e-6, False, inp.cs[k],
                                        inp.ss[k], stream=stream)
        elif kind == "kq_lu":
            kq.kq_quantize_lu(inp.xs[k], inp.P, False, inp.cs[k], inp.ss[k], stream=stream)
        elif kind.startswith("fwht"):
            kq.fwht_quantize(inp.xs[k], int(kind[4:]), inp.cs[k], inp.ss[k], stream=stream)
        elif kind.startswith("kq_v"):
            kq.kq_quantize_variant(int(kind[4:]), inp.xs[k], inp.F, False, inp.cs[k], inp.ss[k], stream=stream)
        elif kind.startswith("sq_v"):
            kq.sq_quantize_variant(int(kind[4:]), inp.xs[k], inp.m, inp.cs[k], inp.ss[k], stream=stream)
        elif kind.startswith("mx_v"):
            kq.mx_quantize_variant(int(kind[4:]), inp.xs[k], inp.cs[k], inp.ss[k], stream=stream)
        else:
            raise ValueError(f"unknown kernel {kind!r}")

    with torch.cuda.stream(stream):
        for i in range(warmup):
            launch(i)
    stream.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    if graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(launches):
                launch(i)
        # spin the clocks up (SM and HBM leave their idle states only under
        # sustained load): replay for >= SPINUP_S before the timed replays
        t_end = time.perf_counter() + SPINUP_S
        while time.perf_counter() < t_end:
            g.replay()
            stream.synchronize()
        reps = max(1, int(0.2 / max(1e-6, _replay_seconds(g, stream))))
        with torch.cuda.stream(stream):
            t0.record(stream)
            for _ in range(reps):
                g.replay()
            t1.record(stream)
        launches *= reps
    else:
        with torch.cuda.stream(stream):
            t0.record(stream)
            for i in range(launches):
                launch(i)
            t1.record(stream)
    stream.synchronize()
    return {"mean_us": 1e3 * t0.elapsed_time(t1) / launches, "nsets": inp.nsets, "graph": graph}


def kernel_mode(args):
    """One quantizer at one shape (the small committed case for ncu captures)."""
    import torch

    from w4a4_mxfp4_post_b200 import build

    build.build()
    dev = torch.device("cuda:0")
    M, d = (int(t) for t in args.shape.lower().split("x"))
    l2 = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 * 2 ** 20))
    inp = RotatingInputs(M, d, dev, l2, budget_bytes=args.budget_mb * 2 ** 20 if args.budget_mb else None)
    r = time_launches(args.kernel, inp, args.launches, args.warmup, torch.cuda.Stream(device=dev),
                      graph=not args.no_graph)
    gbs = BYTES_PER_ELEM * M * d / (r["mean_us"] * 1e-6) / 1e9
    peak, src = measured_peak()
    print(json.dumps({"mode": "kernel", "kernel": args.kernel, "M": M, "d": d, **r, "gbs": round(gbs, 1),
                      "frac_of_peak": round(gbs / peak, 4), "peak": peak, "peak_source": src}), flush=True)


def gemm_mode(args):
    """The W4A4 linear layer on MXFP4 operands (tcgen05 block-scaled MMA) at
    M x N x K, alone, chained after the KroQuant quantizer that feeds it
    (chain_us), and after the quantizer fused with LayerNorm + AdaLN
    (norm_chain_us: residual stream in, layer output out).

    Operands rotate over enough sets that each launch reads A and writes D
    outside L2 (>= 3x L2 between reuses).  The roofline is the tensor pipe:
    2 M N K flops against the measured bf16 GEMM peak x 4, the nominal
    fp4 / bf16 dense ratio (9 / 2.25 PFLOP/s).
    """
    import torch

    import w4a4_mxfp4_post_b200 as kq
    from w4a4_mxfp4_post_b200 import build, synth

    build.build()
    dev = torch.device("cuda:0")
    M, N, K = (int(t) for t in args.shape.lower().split("x"))
    l2 = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 * 2 ** 20))
    x = synth.activation("pixart", M, K, 5)
    F = synth.factors(K // 32, 5)
    W = torch.from_numpy(synth.weights(N, K, 5)).to(dev)
    Wf = kq.kq_fold_weights(W, torch.from_numpy(F).to(dev))
    bc, bsf = kq.mx_quantize_f32(Wf, sf_layout=True)
    set_bytes = M * K * 2 + M * K // 2 + kq.kq_sf_bytes(M, K) + M * N * 2
    nsets = max(2, min(64, math.ceil(3 * l2 / set_bytes)))
    Fd = torch.from_numpy(F).to(dev)
    xs = [torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16).clone() for _ in range(nsets)]
    acs, asfs = zip(*[kq.kq_quantize_sf(xs[i], Fd) for i in range(nsets)])
    outs = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(nsets)]
    g_ad, b_ad = synth.adaln(2 if M % 2 == 0 else 1, K, 5)
    gd, bd = torch.from_numpy(g_ad).to(dev), torch.from_numpy(b_ad).to(dev)
    stream = torch.cuda.Stream(device=dev)

    variants = [int(v) for v in args.kernels.split(",")] if args.kernels[0].isdigit() else [0]

    def run(kind, n):
        for i in range(n):
            k = i % nsets
            if kind == "chain":
                kq.kq_quantize_sf(xs[k], Fd, out_codes=acs[k], out_sf=asfs[k], stream=stream)
                kq.mxf4_gemm(acs[k], asfs[k], bc, bsf, out=outs[k], stream=stream)
            elif kind == "norm_chain":
                kq.norm_kq_quantize_sf(xs[k], gd, bd, Fd, out_codes=acs[k], out_sf=asfs[k], stream=stream)
                kq.mxf4_gemm(acs[k], asfs[k], bc, bsf, out=outs[k], stream=stream)
            else:
                kq.mxf4_gemm_variant(int(kind[1:]), acs[k], asfs[k], bc, bsf, out=outs[k], stream=stream)

    res = {}
    for kind in [f"v{v}" for v in variants] + ["chain", "norm_chain"]:
        with torch.cuda.stream(stream):
            run(kind, max(3, args.warmup))
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            run(kind, args.launches)
        t_end = time.perf_counter() + SPINUP_S
        while time.perf_counter() < t_end:
            g.replay()
            stream.synchronize()
        reps = max(1, int(0.3 / max(1e-6, _replay_seconds(g, stream))))
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            t0.record(stream)
            for _ in range(reps):
                g.replay()
            t1.record(stream)
        stream.synchronize()
        res[kind] = 1e3 * t0.elapsed_time(t1) / (args.launches * reps)
    flops = 2.0 * M * N * K
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            bf16 = float(json.load(fh)["bf16_tflops"])
        src = "measured bf16 burst (MEASURED_PEAKS.json) x 4 (nominal fp4/bf16 dense ratio)"
    except Exception:
        bf16, src = 1590.0, "fallback bf16 1.59 PFLOP/s x 4 (nominal fp4/bf16 dense ratio)"
    peak = 4.0 * bf16
    first = f"v{variants[0]}"
    tflops = flops / (res[first] * 1e-6) / 1e12
    out_bytes = M * N * 2 + M * K // 2 + N * K // 2
    line = {"mode": "gemm", "M": M, "N": N, "K": K, "nsets": nsets,
            "gemm_us": {k: round(v, 3) for k, v in res.items() if k not in ("chain", "norm_chain")},
            "chain_us": round(res["chain"], 3), "norm_chain_us": round(res["norm_chain"], 3),
            "tflops": round(tflops, 1), "peak_tflops": peak,
            "frac_of_peak": round(tflops / peak, 4), "peak_source": src,
            "hbm_gbs_min_bytes": round(out_bytes / (res[first] * 1e-6) / 1e9, 1)}
    if args.cpu_seconds > 0:
        # the oracle's product (double, OpenMP over rows) on a row sample of the
        # same operands, quantized by the oracle
        import oracle

        wc, ws = oracle.mx_quantize_f32(Wf.cpu().numpy())
        xc, xs = oracle.kq_quantize(x[: min(M, 64)], F)
        t0 = time.perf_counter()
        n = 0
        while n < xc.shape[0] and time.perf_counter() - t0 < min(args.cpu_seconds, 10.0):
            step = min(8, xc.shape[0] - n)
            oracle.mxf4_gemm(xc[n:n + step], xs[n:n + step], wc, ws)
            n += step
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": round(2.0 * n * N * K / dt / 1e12, 6), "unit": "TFLOP/s",
                                "cores": oracle.num_threads(), "kind": "oracle",
                                "sample": f"{n} rows of A x all {N} rows of B, K = {K}, {dt:.1f} s"}
    print(json.dumps(line), flush=True)


def sweep_mode(args):
    """Bandwidth sweep: every quantizer at every (M, d) of the sweep workload."""
    import torch

    from w4a4_mxfp4_post_b200 import build, synth

    build.build()
    dev = torch.device("cuda:0")
    l2 = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 * 2 ** 20))
    peak, src = measured_peak()
    rows = []
    kinds = args.kernels.split(",")
    stream = torch.cuda.Stream(device=dev)
    for M in synth.WORKLOADS["sweep"]["Ms"]:
        for d in synth.WORKLOADS["sweep"]["ds"]:
            row = {"M": M, "d": d, "bytes": BYTES_PER_ELEM * M * d}
            inp = RotatingInputs(M, d, dev, l2)
            row["input_sets"] = inp.nsets
            for kind in kinds:
                try:
                    r = time_launches(kind, inp, args.launches, args.warmup, stream)
                except Exception as e:  # a variant that this build does not carry
                    row[kind] = {"error": str(e).splitlines()[0]}
                    continue
                gbs = BYTES_PER_ELEM * M * d / (r["mean_us"] * 1e-6) / 1e9
                row[kind] = {"us": round(r["mean_us"], 3), "gbs": round(gbs, 1), "frac": round(gbs / peak, 4)}
            # a launch under 10 MB or 2 us measures launch latency and ramp, not the stream
            row["launch_bound"] = bool(row["bytes"] < 10e6 or any(
                isinstance(v, dict) and v.get("us", 1e9) < 2.0 for v in row.values()))
            del inp
            torch.cuda.empty_cache()
            rows.append(row)
            print(json.dumps(row), flush=True)
    if args.json_out:
        with open(args.json_out, "w") as fh:
            json.dump({"peak": peak, "peak_source": src, "rows": rows}, fh, indent=1)


def compare_mode(args):
    """Several quantizers side by side at each shape of --shapes, in one process.

    The kernels are timed in turn, and the whole round is repeated --reps
    times, so clock and thermal drift fall on all of them alike.  Each
    measurement is time_launches over RotatingInputs, as in kernel mode.
    """
    import torch

    from w4a4_mxfp4_post_b200 import build

    build.build()
    dev = torch.device("cuda:0")
    l2 = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 * 2 ** 20))
    peak, src = measured_peak()
    stream = torch.cuda.Stream(device=dev)
    kinds = args.kernels.split(",")
    rows = []
    for shape in args.shapes.split(","):
        M, d = (int(t) for t in shape.lower().split("x"))
        inp = RotatingInputs(M, d, dev, l2)
        for rep in range(args.reps):
            for kind in kinds:
                r = time_launches(kind, inp, args.launches, args.warmup, stream)
                gbs = BYTES_PER_ELEM * M * d / (r["mean_us"] * 1e-6) / 1e9
                row = {"mode": "compare", "M": M, "d": d, "kernel": kind, "rep": rep, "us": round(r["mean_us"], 3),
                       "gbs": round(gbs, 1), "frac_of_peak": round(gbs / peak, 4)}
                rows.append(row)
                print(json.dumps(row), flush=True)
        del inp
        torch.cuda.empty_cache()
    if args.json_out:
        with open(args.json_out, "w") as fh:
            json.dump({"peak": peak, "peak_source": src, "rows": rows}, fh, indent=1)


def sqnr_mode(args):
    """Quantisation-error proxy: SQNR of the round trip x -> codes/scales -> x^ per method.

    A dataset-free stand-in for the pages' quality comparison (learned
    block transform vs per-channel scaling vs plain MXFP4 vs fixed Hadamard):
    seeded activations with per-channel outliers, the inverse of each method's
    transform applied after decoding.  SQNR = 10 log10(sum x^2 / sum (x - x^)^2).
    """
    import torch

    import w4a4_mxfp4_post_b200 as kq
    from w4a4_mxfp4_post_b200 import build, synth

    build.build()
    torch.backends.cuda.matmul.allow_tf32 = False
    dev = torch.device("cuda:0")
    rows = []

    def sqnr(x, xh):
        return float(10 * torch.log10((x.double() ** 2).sum() / ((x.double() - xh.double()) ** 2).sum()))

    def lu_to_factors(P):
        a, b, c = P[..., 0].astype(np.float64), P[..., 1].astype(np.float64), P[..., 2].astype(np.float64)
        F = np.stack([np.stack([a, b], -1), np.stack([c * a, c * b - 1 / a], -1)], -2)
        return F.astype(np.float32)

    for name in ("pixart", "sana", "flux"):
        for (M, d, model, shared, seed) in synth.workload_layers(name):
            xb = synth.activation(model, M, d, seed)
            x = torch.from_numpy(xb.view(np.int16)).to(dev).view(torch.bfloat16)
            xf = x.float()
            nb = d // 32
            row = {"workload": name, "M": M, "d": d}
            c, s = kq.mx_quantize(x)
            row["mx"] = sqnr(xf, kq.mx_dequantize(c, s))
            m = torch.from_numpy(synth.sq_multipliers(xb)).to(dev)
            c, s = kq.sq_quantize(x, m)
            row["sq"] = sqnr(xf, kq.mx_dequantize(c, s) / m)
            F = synth.factors(nb, seed)
            Fd = torch.from_numpy(F).to(dev)
            c, s = kq.kq_quantize(x, Fd)
            row["kq_random_factors"] = sqnr(xf, kq.kq_inverse_f32(kq.mx_dequantize(c, s), Fd))
            H2 = np.tile(np.array([[1, 1], [1, -1]], np.float32) / np.float32(np.sqrt(2.0)), (nb, 5, 1, 1))
            Hd = torch.from_numpy(H2).to(dev)
            c, s = kq.kq_quantize(x, Hd)
            row["kq_hadamard_init"] = sqnr(xf, kq.kq_inverse_f32(kq.mx_dequantize(c, s), Hd))
            P = synth.lu_params(nb, seed)
            c, s = kq.kq_quantize_lu(x, torch.from_numpy(P).to(dev))
            Fl = torch.from_numpy(lu_to_factors(P)).to(dev)
            row["kq_lu_near_hadamard"] = sqnr(xf, kq.kq_inverse_f32(kq.mx_dequantize(c, s), Fl))
            for H in (128, 1024):
                if d % H:
                    continue
                c, s = kq.fwht_quantize(x, H)
                Hm = torch.from_numpy(scipy_hadamard(H) / np.sqrt(H)).to(dev).float()
                yh = kq.mx_dequantize(c, s).view(M, d // H, H)
                row[f"fwht_{H}"] = sqnr(xf, (yh @ Hm).view(M, d))   # H_H is symmetric and orthonormal
            rows.append(row)
            print(json.dumps(row), flush=True)
    if args.json_out:
        with open(args.json_out, "w") as fh:
            json.dump(rows, fh, indent=1)


def scipy_hadamard(n):
    import scipy.linalg

    return scipy.linalg.hadamard(n).astype(np.float64)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--scaling", choices=["weak", "strong"], default="weak",
                    help="weak: a batch per rank; strong: the ranks split one batch by rows")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="oracle time for the cpu_baseline block")
    ap.add_argument("--ref-seconds", type=float, default=60.0, help="budget of the reference arm")
    ap.add_argument("--json-out", default="")
    ap.add_argument("--mode", choices=["step", "kernel", "sweep", "sqnr", "gemm", "compare"], default="step",
                    help="step: the benchmark line; kernel: one quantizer at --shape; sweep: all shapes; "
                         "sqnr: quantisation-error proxy per method; gemm: the W4A4 product; "
                         "compare: several quantizers interleaved at --shapes")
    ap.add_argument("--kernel", default="kq",
                    help="kernel mode: kq, sq, mx, kq_v<variant>, sq_v<n>, mx_v<n>, kq_lu, fwht<H>, norm_kq or "
                         "norm_kq_v<n>")
    ap.add_argument("--kernels", default="kq,sq,mx",
                    help="sweep / compare mode: comma-separated kernels; gemm mode: comma-separated tile "
                         "configurations")
    ap.add_argument("--shape", default="8192x12288", help="kernel mode: MxD; gemm mode: MxNxK")
    ap.add_argument("--budget-mb", type=int, default=0, help="kernel mode: total input rotation bytes")
    ap.add_argument("--no-graph", action="store_true", help="kernel mode: eager launches")
    ap.add_argument("--launches", type=int, default=100, help="kernel / sweep / compare mode: timed launches")
    ap.add_argument("--shapes", default="8192x4608,8192x1152", help="compare mode: comma-separated MxD")
    ap.add_argument("--reps", type=int, default=3, help="compare mode: rounds over the kernels")
    args = ap.parse_args()
    if args.mode == "kernel":
        return kernel_mode(args)
    if args.mode == "sweep":
        return sweep_mode(args)
    if args.mode == "sqnr":
        return sqnr_mode(args)
    if args.mode == "gemm":
        return gemm_mode(args)
    if args.mode == "compare":
        return compare_mode(args)
    if args.steps < 1 or args.warmup < 3:
        raise SystemExit("need --steps >= 1 and --warmup >= 3")

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        out = reference_arm(args, rank, world)
        if out is not None:
            line = json.dumps(out)
            print(line, flush=True)
            if args.json_out:
                with open(args.json_out, "w") as fh:
                    fh.write(line + "\n")
        return

    from w4a4_mxfp4_post_b200 import build

    build.build()
    rank, local, world, pg = dist_setup(args.gpus)
    try:
        out = gpu_arm(args, rank, local, world, pg)
        if rank == 0:
            if world == 1:
                out["cpu_baseline"] = cpu_baseline_block(workload_inputs(), args.cpu_seconds)
            line = json.dumps(out)
            print(line, flush=True)
            if args.json_out:
                with open(args.json_out, "w") as fh:
                    fh.write(line + "\n")
    finally:
        if pg is not None:
            pg.destroy_process_group()


if __name__ == "__main__":
    main()
