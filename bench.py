#!/usr/bin/env python
"""Benchmark of the compressed-KV hot path on B200.

One step = the whole path for one decode token of every sequence of the 32K GQA
workload (batch 8, 32 query heads over 8 KV heads, d=128, context 32768, bf16,
16-token ring, 3-bit keys b1=2 + m=128, 2-bit values g=32):
    tq_decode_step = tq_append (1 new token per sequence: the oldest ring
               token is quantised into the packed cache, the new one enters the
               ring) + tq_decode_attention (query preparation, split-K partial
               whose last split per (batch, KV head) merges the splits), in two
               launches.
Inputs are resident in HBM before timing; L2 is flushed between steps, outside
the timed events: a 256 MB write, then a 256 MB read of a second buffer, so that
no dirty line of the flush is written back inside the timed region.  `value`
is algorithmic bytes (packed cache + ring + append traffic) per second.  Also
reported: the dominant kernel's roofline, end-to-end (host buffers, copies
inside the timed region), the key quantise throughput of the 131072-token x
8-head append workload, the CPU oracle baseline, clocks, and the number of
library kernel launches.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "compressed decode-attn HBM GB/s (% of 8 TB/s) and tokens/s; key-quantize Mkeys/s"
NOMINAL_HBM = 8000.0      # GB/s, the metric's reference figure
FALLBACK_HBM = 6650.0     # GB/s, used only when MEASURED_PEAKS.json is absent


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--splits", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-quantize", action="store_true")
    ap.add_argument("--no-other-decodes", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-sensitivity", action="store_true")
    ap.add_argument("--workload", default="gqa32k")
    ap.add_argument("--case", choices=sorted(CASES), default=None,
                    help="run one small per-kernel workload (for a profiler capture) instead "
                         "of the bench")
    return ap.parse_args()


def measured_bf16_tflops():
    """Dense bf16 tensor peak (burst) in TFLOP/s: measured, else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM, "fallback"


def source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "compressed_attention_turboquantprod_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_file: str, src_hash: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary,
    or None when the kernel source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", kernel_file)
    try:
        with open(p) as f:
            d = json.load(f)
        if d.get("source_hash") == src_hash:
            return d.get("dram_bytes_per_launch")
    except Exception:
        pass
    return None


class ClockSampler:
    """SM clocks and clock-event reasons sampled every 50 ms during the timed region,
    through NVML (read-only queries), else through one nvidia-smi query per sample."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40}

    def __init__(self, device_index: int, uuid: str | None = None, period_s: float = 0.05):
        self.index, self.uuid, self.period = device_index, uuid, period_s
        self.samples, self.reasons, self.smax = [], set(), None
        self._stop = None
        self._thread = None
        self.source = None

    def _nvml_reader(self):
        import pynvml
        pynvml.nvmlInit()
        h = None
        if self.uuid:
            try:
                h = pynvml.nvmlDeviceGetHandleByUUID(self.uuid)
            except Exception:
                h = None
        if h is None:
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
        self.smax = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
        get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            pynvml.nvmlDeviceGetCurrentClocksThrottleReasons

        def read():
            return (float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)), int(get_reasons(h)))
        self.source = "nvml"
        return read

    def _smi_reader(self):
        def read():
            r = subprocess.run(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                "-i", str(self.index)], capture_output=True, text=True, timeout=5)
            parts = [p.strip() for p in r.stdout.strip().split(",")]
            self.smax = float(parts[2])
            bits = 0
            for nm, val in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                                "sw_power_cap"), parts[5:9]):
                if val.lower() == "active":
                    bits |= self.REASONS[nm]
            return float(parts[1]), bits
        self.source = "nvidia-smi"
        return read

    def start(self):
        import threading
        try:
            read = self._nvml_reader()
            read()
        except Exception:
            try:
                read = self._smi_reader()
                read()
            except Exception:
                return
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    mhz, bits = read()
                    self.samples.append(mhz)
                    for nm, bit in self.REASONS.items():
                        if bits & bit:
                            self.reasons.add(nm)
                except Exception:
                    pass
                self._stop.wait(self.period)
        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()

    def stop(self):
        if self._thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        self._stop.set()
        self._thread.join(timeout=10)
        sm = self.samples
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.smax,
                "reasons": sorted(self.reasons), "samples": len(sm), "source": self.source}


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _reduce(x: float, world: int, op: str) -> float:
    """All-reduce of one float over the ranks (NCCL on GPUs, gloo on CPU)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = (torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl"
           else torch.device("cpu"))
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def reduce_max(x: float, world: int) -> float:
    return _reduce(x, world, "max")


def reduce_sum(x: float, world: int) -> float:
    return _reduce(x, world, "sum")


def aggregate(local_bytes: float, local_ms: float, world: int):
    """Whole-job throughput: every rank's bytes over the slowest rank's device time.
    Returns (GB/s, max ms)."""
    ms = reduce_max(local_ms, world)
    total = reduce_sum(local_bytes, world)
    return total / (ms * 1e-3) / 1e9, ms


# --------------------------------------------------------------------------- CPU oracle
def oracle_decode_sample(w, K1, V1, Q_steps, Kn, Vn, budget_s=12.0, min_reps=2, max_reps=None):
    """Time the oracle on one (batch, KV head) unit at full context: untimed prefill
    quantisation, then timed steps of append-one-token + decode of its G query heads.
    Returns (seconds per step, algorithmic bytes per step, reps, threads)."""
    import numpy as np
    from oracle import cache as ocache
    from oracle import codebook as ocb
    from oracle import projections as oproj
    po = oproj.make_projections(w.d, w.m, 0, with_rotation=w.b1 > 0)
    cb = ocb.build(w.d, w.b1) if w.b1 else None
    cap = w.T + 4096
    oc = ocache.OracleCache(1, 1, w.d, w.b1, w.m, w.vbits, w.group, w.W, cap, w.dtype, po, cb)
    oc.append(K1[None, None], V1[None, None])
    G = w.Hq // w.Hkv
    times, nbytes = [], []
    i = 0
    t_start = time.perf_counter()
    while True:
        t0 = time.perf_counter()
        oc.append(Kn[i % Kn.shape[0]][None, None, None], Vn[i % Vn.shape[0]][None, None, None])
        oc.decode(Q_steps[i % Q_steps.shape[0]][None, :G])
        times.append(time.perf_counter() - t0)
        nbytes.append(oc.n_comp * oc.lay.token_bytes + 2 * oc.n_ring * w.d * (4 if w.dtype == "f32" else 2))
        i += 1
        el = time.perf_counter() - t_start
        if (i >= min_reps and el >= budget_s) or (max_reps and i >= max_reps):
            break
    try:
        from threadpoolctl import threadpool_info
        threads = max([p.get("num_threads", 1) for p in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    return statistics.mean(times), statistics.mean(nbytes), i, threads


def oracle_prefill_sample(w, n=16, context=4096, reps=2):
    """Time the oracle's multi-token attention on one (batch, KV head) unit of workload
    w: a cache of `context` tokens (quantised untimed), then `reps` timed calls that
    score a chunk of n tokens.  Inputs are drawn on the host.  Returns (seconds per
    call, compressed tokens of the sample, threads)."""
    import numpy as np
    import synth
    from oracle import cache as ocache
    from oracle import codebook as ocb
    from oracle import projections as oproj
    G = w.Hq // w.Hkv
    w1 = w.scaled(B=1, Hkv=1, Hq=G, T=context)
    K, V = synth.keys_values(w1, device="cpu")
    Q, Kc, Vc = synth.prefill_chunk(w1, n, device="cpu")
    po = oproj.make_projections(w.d, w.m, 0, with_rotation=w.b1 > 0)
    cb = ocb.build(w.d, w.b1) if w.b1 else None
    oc = ocache.OracleCache(1, 1, w.d, w.b1, w.m, w.vbits, w.group, w.W, context + 64, w.dtype, po, cb)
    f = lambda t: t.double().numpy()
    oc.append(f(K), f(V))
    times = []
    for _ in range(reps):
        t0 = time.perf_counter()
        oc.prefill(f(Q), f(Kc), f(Vc))
        times.append(time.perf_counter() - t0)
    return statistics.mean(times), oc.n_comp, _oracle_threads()


def oracle_moments_sample(w, tokens=8192, reps=2):
    """Time the oracle's key variance on one batch row of a calibration layer shaped
    like workload w (all KV heads, `tokens` tokens), drawn on the host.  Returns
    (seconds per pass, bytes of the sample in the workload dtype, threads)."""
    import synth
    from oracle import sensitivity as osens
    K, _ = synth.keys_values(w.scaled(B=1, T=tokens), layer=5, device="cpu")
    x = K.double().numpy()
    times = []
    for _ in range(reps):
        t0 = time.perf_counter()
        osens.key_variance(x)
        times.append(time.perf_counter() - t0)
    return statistics.mean(times), K.numel() * K.element_size(), _oracle_threads()


def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([p.get("num_threads", 1) for p in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count()


def _host_unit(w, device):
    """K, V of unit (b=0, h=0) at full context and per-step inputs, as float64 numpy."""
    import numpy as np
    import synth
    import torch
    K, V = synth.keys_values(w.scaled(B=1, Hkv=1), device=device)
    Q, Kn, Vn = synth.decode_stream(w.scaled(B=1, Hkv=1, Hq=w.Hq // w.Hkv), 8, device=device)
    f = lambda t: t.to("cpu", torch.float32).numpy().astype(np.float64)
    return f(K[0, 0]), f(V[0, 0]), f(Q[:, 0]), f(Kn[:, 0, 0, 0]), f(Vn[:, 0, 0, 0])


# --------------------------------------------------------------------------- reference arm
def run_reference(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import synth
    w = synth.WORKLOADS[args.workload]
    dev = "cpu"
    units = w.B * w.Hkv
    # Size the per-step sample so that the whole run stays within ~150 s: one
    # (batch, KV head) unit, at full context when that fits, else at a shorter one.
    K1, V1, Qs, Kn, Vn = _host_unit(w, dev)
    t_full, _, _, _ = oracle_decode_sample(w, K1, V1, Qs, Kn, Vn, budget_s=0.0, min_reps=1, max_reps=1)
    n_total = max(1, args.warmup + args.steps)
    ctx = w.T
    if n_total * t_full > 150.0:
        ctx = max(1024, int(w.T * 150.0 / (n_total * t_full)) // 64 * 64)
    ws = w.scaled(T=ctx)
    K1, V1 = K1[:ctx], V1[:ctx]
    if args.warmup:
        oracle_decode_sample(ws, K1, V1, Qs, Kn, Vn, budget_s=0.0, min_reps=args.warmup,
                             max_reps=args.warmup)
    sec, nbytes, reps, threads = oracle_decode_sample(ws, K1, V1, Qs, Kn, Vn, budget_s=0.0,
                                                      min_reps=max(1, args.steps),
                                                      max_reps=max(1, args.steps))
    gbs = nbytes / sec / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": _config(w, args),
        "cpu_baseline": {"kind": "oracle", "value": gbs, "unit": "GB/s", "cores": threads,
                         "sample": f"1 of {units} (batch, KV-head) units per step at context {ctx} "
                                   f"(of {w.T}): append one token + decode its query heads, NumPy float64"},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "tokens_per_s": 1.0 / sec / units,
    }
    print(json.dumps(line), flush=True)
    return 0


def _config(w, args):
    return {"workload": f"{w.name}: batch {w.B}, {w.Hq} query heads over {w.Hkv} KV heads, d={w.d}, "
                        f"context {w.T} ({w.W}-token {w.dtype} ring), keys b1={w.b1} + QJL m={w.m}, "
                        f"values {w.vbits}-bit group {w.group}",
            "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "context": w.T, "ring": w.W,
            "b1": w.b1, "m": w.m, "vbits": w.vbits, "group": w.group, "input_dtype": w.dtype,
            "l2": "flushed between timed steps (256 MB write + 256 MB read of another buffer, "
                  "outside the events)",
            "parallelism": f"independent replicas per GPU (weak scaling)" if args.gpus > 1 else "1 GPU"}


# --------------------------------------------------------------------------- our arm
def run_ours(args):
    import numpy as np
    import torch
    world, rank, local = dist_setup(args)
    import synth
    from compressed_attention_turboquantprod_b200 import (Codebook, CompressedKVCache, Projections,
                                                           native)
    dev = torch.device("cuda", local)
    w = synth.WORKLOADS[args.workload].scaled(seed=rank)
    G = w.Hq // w.Hkv
    n_steps = args.warmup + args.steps
    pj, cb = Projections(w.d, w.m, 0, rotation=w.b1 > 0, device=dev), (
        Codebook(w.d, w.b1, device=dev) if w.b1 else None)
    cap = w.T - w.W + 2 * n_steps + 128
    cache = CompressedKVCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, w.W, cap,
                              dtype=w.torch_dtype, device=dev)
    K, V = synth.keys_values(w, device=dev)
    cache.append(K, V, pj, cb)
    del K, V
    torch.cuda.empty_cache()
    Qs, Kn, Vn = synth.decode_stream(w, n_steps, device=dev)
    ws = cache.workspace(w.Hq, args.splits)
    out = torch.empty(w.B, w.Hq, w.d, dtype=w.torch_dtype, device=dev)
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def flush_l2():
        flush_w.zero_()
        return flush_r.sum()
    stream = torch.cuda.current_stream(dev)
    scale = 1.0 / math.sqrt(w.d)
    cent = cb.centroids if cb else None
    bnd = cb.boundaries if cb else None
    es = 4 if w.dtype == "f32" else 2
    tb = cache.state.token_bytes

    def step_bytes():
        n_comp, n_ring = cache.n_comp, cache.n_ring
        dec = w.B * w.Hkv * (n_comp * tb + 2 * n_ring * w.d * es)
        app = w.B * w.Hkv * (2 * w.d * es + tb + 2 * w.d * es)   # read ring token + new token, write record + ring
        return dec, dec + app

    def step(i, evs=None, around_partial=False):
        """One step.  Timed steps use tq_decode_step (append + decode in one call,
        two launches), with evs = (start, end) at the step's boundaries.  With
        around_partial the same work runs as tq_append + tq_decode_prep +
        tq_decode_partial and evs bracket the partial kernel alone (an event
        between two kernels also ends the programmatic overlap of their launches)."""
        if not around_partial:
            if evs:
                evs[0].record(stream)
            native.tq_decode_step(cache.state, Kn[i], Vn[i], Qs[i], scale, pj.Pi, pj.S, pj.T, cent,
                                  bnd, out, None, args.splits, ws)
            if evs:
                evs[1].record(stream)
            return
        native.tq_append(cache.state, Kn[i], Vn[i], pj.Pi, pj.T, cent, bnd)
        native.tq_decode_prep(cache.state, Qs[i], scale, pj.Pi, pj.S, cent, args.splits, ws)
        if evs:
            evs[0].record(stream)
        native.tq_decode_partial(cache.state, w.Hq, scale, cent, None, args.splits, ws, out=out)
        if evs:
            evs[1].record(stream)

    props = torch.cuda.get_device_properties(dev)
    uuid = getattr(props, "uuid", None)
    try:
        nvml_index = int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local])
    except (KeyError, ValueError, IndexError):
        nvml_index = local
    clocks = ClockSampler(nvml_index, uuid=f"GPU-{uuid}" if uuid is not None else None,
                          period_s=0.01)
    clocks.start()
    for i in range(args.warmup):
        flush_l2()
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    dec_bytes, all_bytes = [], []
    for k in range(args.steps):
        flush_l2()
        step(args.warmup + k, events[k])
        db, ab = step_bytes()          # host state: the context the decode just read
        dec_bytes.append(db)
        all_bytes.append(ab)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    # the same steps again, timing the partial kernel alone (roofline)
    pevents = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    part_bytes_list = []
    for k in range(args.steps):
        flush_l2()
        step(args.warmup + k, pevents[k], around_partial=True)
        part_bytes_list.append(step_bytes()[0])
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    clk = clocks.stop()
    t_step = [e[0].elapsed_time(e[1]) for e in events]             # ms
    t_part = [e[0].elapsed_time(e[1]) for e in pevents]
    tot_ms = sum(t_step)
    value, tot_ms_max = aggregate(float(sum(all_bytes)), tot_ms, world)
    tokens_s = reduce_sum(float(w.B * args.steps), world) / (tot_ms_max * 1e-3)
    part_avg_ms = sum(t_part) / len(t_part)
    part_bytes = sum(part_bytes_list) / len(part_bytes_list)
    peak, peak_kind = measured_peak()
    src_hash = source_hash("decode_mma.cu", "mma_common.cuh")
    traffic = profiled_traffic("decode_partial_gqa32k.json", src_hash)
    achieved = part_bytes / (part_avg_ms * 1e-3) / 1e9

    # end to end: per step, H2D of the step's Q / new K / new V from pinned host
    # buffers and D2H of the output inside the timed region
    e2e = None
    if args.steps > 0:
        n_e2e = min(args.steps, 100)
        # one pinned host record per step holding that step's Q, new K and new V,
        # and a pinned output per step: tq_decode_step is called with these host
        # buffers themselves (pinned memory is mapped into the device address
        # space), so its kernels read the step's inputs and write its output
        # across the host link inside the timed region, with no staging copy
        parts = [Qs[0], Kn[0], Vn[0]]
        sizes = [t.numel() * t.element_size() for t in parts]
        rec = sum(sizes)
        host = torch.empty(n_e2e, rec, dtype=torch.uint8).pin_memory()
        for k in range(n_e2e):
            o = 0
            for t, nbytes in zip((Qs[k], Kn[k], Vn[k]), sizes):
                host[k, o:o + nbytes].copy_(t.contiguous().view(torch.uint8).reshape(-1).cpu())
                o += nbytes
        hviews = []
        for k in range(n_e2e):
            views, o = [], 0
            for t, nbytes in zip(parts, sizes):
                views.append(host[k, o:o + nbytes].view(t.dtype).view(t.shape))
                o += nbytes
            hviews.append(views)
        outh = torch.empty(n_e2e, *out.shape, dtype=out.dtype).pin_memory()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n_e2e)]
        e2e_bytes = 0
        n0 = cache.state.n_total
        snap = cache.buffer.clone()              # to replay step 0 on the device path below
        torch.cuda.synchronize()
        for k in range(n_e2e):
            flush_l2()
            qh, kh, vh = hviews[k]
            ev[k][0].record(stream)
            native.tq_decode_step(cache.state, kh, vh, qh, scale, pj.Pi, pj.S, pj.T, cent, bnd, outh[k],
                                  None, args.splits, ws)
            ev[k][1].record(stream)
            e2e_bytes += step_bytes()[1]
        torch.cuda.synchronize()
        e2e_ms_steps = [e[0].elapsed_time(e[1]) for e in ev]
        # step 0 replayed from the same cache state with device buffers: the same output
        cache.buffer.copy_(snap)
        del snap
        cache.state.n_total = n0
        native.tq_decode_step(cache.state, Kn[0], Vn[0], Qs[0], scale, pj.Pi, pj.S, pj.T, cent, bnd, out,
                              None, args.splits, ws)
        torch.cuda.synchronize()
        if not torch.equal(out.cpu().view(torch.uint8), outh[0].view(torch.uint8)):
            raise RuntimeError("end-to-end output from host buffers differs from the device path")
        e2e_ms = reduce_max(sum(e2e_ms_steps), world)
        e2e_val = reduce_sum(float(e2e_bytes), world) / (e2e_ms * 1e-3) / 1e9
        e2e = {"value": e2e_val, "unit": "GB/s", "h2d_bytes_per_step": int(rec),
               "d2h_bytes_per_step": int(out.numel() * out.element_size()),
               "ms_per_step": e2e_ms / n_e2e, "steps": n_e2e,
               "transfer": "tq_decode_step called on pinned host buffers: its kernels read Q, K, V "
                           "and write the output over the host link (mapped pinned memory)"}

    # multi-token (chunked prefill) attention on the same cache: chunks of n tokens
    prefill = None
    if not args.no_prefill:
        prefill = bench_prefill(w, cache, pj, cb, flush_l2, stream, step_bytes()[0], world)

    # key/value quantise throughput: 131072 tokens x 8 KV heads in chunks of 4096
    quant = qsample = None
    if not args.no_quantize:
        quant, qsample = bench_quantize(
            dev, world, keep_sample=rank == 0 and world == 1 and not args.no_cpu_baseline)
    structured = None
    if not args.no_quantize:
        structured = bench_structured_rotation(dev, world)
    sensitivity = None
    if not args.no_sensitivity:
        sensitivity = bench_sensitivity(dev, world, peak, flush_l2)
    others = None
    if not args.no_other_decodes:
        del cache, Qs, Kn, Vn
        torch.cuda.empty_cache()
        others = bench_other_decodes(dev, world, peak)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        K1, V1, Q1, Kn1, Vn1 = _host_unit(w, dev)
        sec, nb, reps, threads = oracle_decode_sample(w, K1, V1, Q1, Kn1, Vn1)
        cpu = {"kind": "oracle", "value": nb / sec / 1e9, "unit": "GB/s", "cores": threads,
               "sample": f"1 of {w.B * w.Hkv} (batch, KV-head) units at full context, {reps} steps "
                         "(append one token + decode its query heads), NumPy float64; GB/s of "
                         "that unit's packed bytes"}
        if prefill is not None:
            n0 = prefill["chunks"][0]["n"]
            sec_p, comp_s, thr = oracle_prefill_sample(w, n=n0)
            # the oracle's time is linear in the history and in the units: scaled to the
            # bench's history length and its B * Hkv units
            hist = prefill["history_tokens"]
            t_full = sec_p * (hist / comp_s) * (w.B * w.Hkv)
            prefill["cpu_baseline"] = {
                "kind": "oracle", "value": w.B * n0 / t_full, "unit": "query tokens/s",
                "cores": thr,
                "sample": f"one (batch, KV-head) unit, {comp_s}-token history, a {n0}-token chunk, "
                          f"NumPy float64, scaled by {hist}/{comp_s} history and "
                          f"{w.B * w.Hkv} units"}
        if qsample is not None:
            quant["parity_vs_oracle"] = oracle_quantize_counts(qsample)
        if sensitivity is not None:
            sec_m, nb_m, thr = oracle_moments_sample(synth.WORKLOADS["aqjl"])
            sensitivity["cpu_baseline"] = {
                "kind": "oracle", "value": nb_m / sec_m / 1e9, "unit": "GB/s", "cores": thr,
                "sample": "key variance of one batch row (8 KV heads x 8192 tokens x 128, fp16 "
                          "bytes) of the calibration layer, NumPy float64"}

    # per timed step (tq_decode_step): one grid for the quantise of the token leaving
    # the ring + ring write + query preparation, one partial kernel
    launches = 2 * args.steps
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": tot_ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": _config(w, args),
        "pct_of_8TBps": 100.0 * value / NOMINAL_HBM,
        "tokens_per_s": tokens_s,
        "roofline": {"bound": "hbm", "kernel": "k_decode_partial_mma", "achieved": achieved,
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "algorithmic_bytes_per_launch": part_bytes,
                     "avg_launch_ms": part_avg_ms, "source_hash": src_hash},
        "e2e": e2e,
        "quantize": quant,
        "structured_rotation": structured,
        "prefill": prefill,
        "sensitivity": sensitivity,
        "other_decodes": others,
        "cpu_baseline": cpu,
        "clocks": clk,
        "gpu_launches": launches,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    barrier(world)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def bench_prefill(w, cache, pj, cb, flush_l2, stream, hist_bytes, world, chunks=(16, 64), reps=20,
                  warm=3):
    """tq_prefill_attention on the decode bench's cache (the chunk is scored, not
    appended), L2 flushed before each call, CUDA events around the call (its four
    launches).  A plain decode (tq_decode_attention) of the same cache is timed the
    same way, so that n decodes can be compared with one chunk of n tokens."""
    import torch
    import synth
    from compressed_attention_turboquantprod_b200 import native
    dev = cache.buffer.device
    scale = 1.0 / math.sqrt(w.d)
    cent = cb.centroids if cb else None

    def timed(fn):
        for _ in range(warm):
            flush_l2()
            fn()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
        for k in range(reps):
            flush_l2()
            ev[k][0].record(stream)
            fn()
            ev[k][1].record(stream)
        torch.cuda.synchronize()
        return reduce_max(sum(e[0].elapsed_time(e[1]) for e in ev) / reps, world)

    Qd = synth.queries(w, device=dev)
    outd = torch.empty_like(Qd)
    wsd = cache.workspace(w.Hq, 0)
    t_dec = timed(lambda: native.tq_decode_attention(cache.state, Qd, scale, pj.Pi, pj.S, cent,
                                                     outd, None, 0, wsd))
    # executed tensor work of the history partial per (history token, query token, KV
    # head): int8 score MMAs (KS k-steps of 32 features x 4 heads x 4 slices; tcgen05
    # for chunks of 8 or more tokens) and f16 P V MMAs (128 channels x 4 heads x
    # hi/lo); int8 taken at twice the bf16 peak
    F = (1 << (w.b1 - 1)) if w.b1 > 0 else 0
    KS = F * w.d // 32 + w.m // 32
    G = w.Hq // w.Hkv
    bf16, bf16_kind = measured_bf16_tflops()
    units = w.B * w.Hkv
    res = []
    for n in chunks:
        Q, Kc, Vc = synth.prefill_chunk(w, n, device=dev)
        out = torch.empty_like(Q)
        ws = torch.empty(native.tq_prefill_workspace_bytes(cache.state, w.Hq, n, 0),
                         dtype=torch.uint8, device=dev)
        t = timed(lambda: native.tq_prefill_attention(cache.state, Q, Kc, Vc, scale, pj.Pi, pj.S,
                                                      cent, out, 0, ws))
        native.tq_prefill_check(cache.state, w.Hq, n, 0, ws)
        toks = reduce_sum(float(w.B * n), world)
        work = float(cache.n_comp) * units * n
        # the method's own work per (history token, query token, KV head): for each of
        # the G query heads the MSE dot (d), the QJL dot (m) and the P V row (d)
        algo_flops = work * 2 * G * ((w.d if w.b1 > 0 else 0) + w.m + w.d)
        algo_tflops = algo_flops / (t * 1e-3) / 1e12
        i8_ops, f16_ops = work * 16 * 32 * KS * 2, work * 128 * 8 * 2
        ideal_ms = (i8_ops / (2 * bf16 * 1e12) + f16_ops / (bf16 * 1e12)) * 1e3
        res.append({"n": n, "ms": t, "query_tokens_per_s": toks / (t * 1e-3),
                    "history_GB_per_s": reduce_sum(float(hist_bytes), world) / (t * 1e-3) / 1e9,
                    "vs_n_decodes": n * t_dec / t,
                    "tensor": {"bound": "tensor", "achieved": algo_tflops, "peak": bf16,
                               "unit": "TFLOP/s", "frac": algo_tflops / bf16,
                               "flops": "algorithmic: 2 G (d + m + d) per (history token, query "
                                        "token, KV head)",
                               "peak_kind": bf16_kind,
                               "executed": {"int8_tops": i8_ops / (t * 1e-3) / 1e12,
                                            "f16_tflops": f16_ops / (t * 1e-3) / 1e12,
                                            "ideal_ms_at_peak": ideal_ms,
                                            "frac_of_executed_ideal": ideal_ms / t}}})
    return {"chunks": res, "decode_ms": t_dec, "history_bytes": hist_bytes,
            "history_tokens": int(cache.n_comp),
            "timing": "CUDA events around the whole call (prep, history partials, exact segment, "
                      "merge), L2 flushed before each call, 20 calls after 3 warm-up calls"}


def bench_sensitivity(dev, world, peak, flush_l2, reps=10, warm=3):
    """Key moments (tq_key_moments) of one layer of calibration keys shaped like the
    A-QJL workload (batch 16, 8 KV heads, 8192 tokens, d=128, fp16: 268 MB, above
    L2), L2 flushed before each pass; then the host profile of 32 layers."""
    import time
    import torch
    import synth
    from compressed_attention_turboquantprod_b200 import LayerGroups, native
    w = synth.WORKLOADS["aqjl"].scaled(T=8192)
    K, V = synth.keys_values(w, layer=5, device=dev)
    del V
    out = torch.empty(2, dtype=torch.float64, device=dev)
    ws = torch.empty(native.tq_key_moments_workspace_bytes(), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(warm):
        flush_l2()
        native.tq_key_moments(K, out, ws)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
    for k in range(reps):
        flush_l2()
        ev[k][0].record(stream)
        native.tq_key_moments(K, out, ws)
        ev[k][1].record(stream)
    torch.cuda.synchronize()
    t = reduce_max(sum(e[0].elapsed_time(e[1]) for e in ev) / reps, world)
    nbytes = K.numel() * K.element_size()
    gbs = nbytes / (t * 1e-3) / 1e9
    var = [1.0 + 2.0 * l / 31 for l in range(32)]
    h0 = time.perf_counter()
    lg = LayerGroups.from_variances(var, 4, 336)
    host_ms = (time.perf_counter() - h0) * 1e3
    del K
    torch.cuda.empty_cache()
    return {"keys_bytes": nbytes, "moments_ms": t, "GB_per_s": reduce_sum(gbs, world),
            "roofline": {"bound": "hbm", "kernel": "k_key_moments", "achieved": gbs, "peak": peak,
                         "unit": "GB/s", "frac": gbs / peak},
            "host_profile_ms_32_layers": host_ms,
            "profile_of_variance_ramp": {"boundaries": lg.boundaries, "sketch_dims": lg.sketch_dims}}


def _time_decode(w, layer, dev, reps=10, warm=3):
    """Full-size cache of workload w (layer `layer`), then prep + partial (merged
    output) with L2 flushed before each decode; CUDA events around the partial.
    Returns (mean partial ms, mean prep+partial ms, algorithmic bytes per decode)."""
    import torch
    import synth
    from compressed_attention_turboquantprod_b200 import (Codebook, CompressedKVCache, Projections,
                                                           native)
    m = w.m_for_layer(layer)
    wl = w.scaled(m=m)
    pj = Projections(wl.d, m, layer, rotation=wl.b1 > 0, device=dev)
    cb = Codebook(wl.d, wl.b1, device=dev) if wl.b1 else None
    cache = CompressedKVCache(wl.B, wl.Hkv, wl.d, wl.b1, m, wl.vbits, wl.group, wl.W, wl.T,
                              dtype=wl.torch_dtype, device=dev)
    K, V = synth.keys_values(wl, layer=layer, device=dev)
    # the cache fill is a one-shot quantise-and-append of every token: timed on its
    # second run (the first one grows the stream-ordered pool of the operand image)
    stream = torch.cuda.current_stream(dev)
    fill_ms = 0.0
    for rep in range(2):
        cache.state.n_total = 0
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        cache.append(K, V, pj, cb)
        e1.record(stream)
        torch.cuda.synchronize()
        fill_ms = e0.elapsed_time(e1)
    del K, V
    torch.cuda.empty_cache()
    Q = synth.queries(wl, layer=layer, device=dev)
    ws = cache.workspace(wl.Hq, 0)
    out = torch.empty(wl.B, wl.Hq, wl.d, dtype=wl.torch_dtype, device=dev)
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    scale = 1.0 / math.sqrt(wl.d)
    cent = cb.centroids if cb else None
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps)]
    for i in range(warm + reps):
        flush_w.zero_()
        flush_r.sum()
        e = ev[i - warm] if i >= warm else None
        if e:
            e[0].record(stream)
        native.tq_decode_prep(cache.state, Q, scale, pj.Pi, pj.S, cent, 0, ws)
        if e:
            e[1].record(stream)
        native.tq_decode_partial(cache.state, wl.Hq, scale, cent, None, 0, ws, out=out)
        if e:
            e[2].record(stream)
    torch.cuda.synchronize()
    part = sum(a[1].elapsed_time(a[2]) for a in ev) / reps
    whole = sum(a[0].elapsed_time(a[2]) for a in ev) / reps
    es = 4 if wl.dtype == "f32" else 2
    nbytes = wl.B * wl.Hkv * (cache.n_comp * cache.state.token_bytes + 2 * cache.n_ring * wl.d * es)
    keys = wl.B * wl.Hkv * wl.T
    fill = {"ms": fill_ms, "keys": keys, "Mkeys_per_s": keys / (fill_ms * 1e-3) / 1e6,
            # reads of K and V, writes of the packed records (and the ring)
            "bytes": keys * 2 * wl.d * es + wl.B * wl.Hkv * (cache.n_comp * cache.state.token_bytes
                                                             + 2 * cache.n_ring * wl.d * es)}
    del cache, ws, out, flush_w, flush_r
    torch.cuda.empty_cache()
    return part, whole, nbytes, fill


def _aqjl_32_layer_step(w, dev, reps=5, warm=2):
    """Every layer of the A-QJL workload cached at full context (all 32 caches
    resident, about 30 GB), then one decode step over the 32 layers in order (each
    layer: query preparation and partial with the merged output), L2 flushed
    before each step, CUDA events around the step."""
    import torch
    import synth
    from compressed_attention_turboquantprod_b200 import CompressedKVCache, Projections, native
    layers = []
    nbytes = 0
    for layer in range(32):
        m = w.m_for_layer(layer)
        wl = w.scaled(m=m)
        pj = Projections(wl.d, m, layer, rotation=False, device=dev)
        cache = CompressedKVCache(wl.B, wl.Hkv, wl.d, 0, m, wl.vbits, wl.group, wl.W, wl.T,
                                  dtype=wl.torch_dtype, device=dev)
        K, V = synth.keys_values(wl, layer=layer, device=dev)
        cache.append(K, V, pj, None)
        del K, V
        Q = synth.queries(wl, layer=layer, device=dev)
        layers.append((cache, pj, Q, torch.empty_like(Q), cache.workspace(wl.Hq, 0)))
        nbytes += wl.B * wl.Hkv * (cache.n_comp * cache.state.token_bytes + 2 * cache.n_ring * wl.d * 2)
    torch.cuda.empty_cache()
    scale = 1.0 / math.sqrt(w.d)
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        for cache, pj, Q, out, ws in layers:
            native.tq_decode_attention(cache.state, Q, scale, None, pj.S, None, out, None, 0, ws)
    times = []
    for r in range(warm + reps):
        flush_w.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step()
        e1.record(stream)
        torch.cuda.synchronize()
        if r >= warm:
            times.append(e0.elapsed_time(e1))
    ms = sum(times) / len(times)
    del layers, flush_w
    torch.cuda.empty_cache()
    return ms, nbytes


def bench_other_decodes(dev, world, peak):
    """The A-QJL decodes (one layer of each sketch-size group timed alone, then a
    whole 32-layer token step over all resident layer caches) and the wide-head
    262K decode, at full size."""
    import synth
    res = {}
    w = synth.WORKLOADS["aqjl"]
    groups, tot_ms, tot_bytes = [], 0.0, 0.0
    for layer in (0, 8, 16, 24):
        part, whole, nb, fill = _time_decode(w, layer, dev)
        part, whole = reduce_max(part, world), reduce_max(whole, world)
        nb_all = reduce_sum(float(nb), world)
        groups.append({"layers": f"{layer}-{layer + 7}", "m": w.m_for_layer(layer),
                       "partial_ms": part, "decode_ms": whole, "GB_per_s": nb_all / (part * 1e-3) / 1e9,
                       "frac_of_peak": nb / (part * 1e-3) / 1e9 / peak,
                       "cache_fill": _fill_entry(fill, world, peak)})
        tot_ms += 8 * whole
        tot_bytes += 8 * nb_all
    step_ms, step_bytes = _aqjl_32_layer_step(w, dev)
    step_ms = reduce_max(step_ms, world)
    step_all = reduce_sum(float(step_bytes), world)
    res["aqjl"] = {"workload": "A-QJL: 32 layers, batch 16, 32 query heads over 8 KV heads, d=128, "
                               "context 65536, pure QJL fp16 keys, m 512/384/256/192 by layer group, "
                               "2-bit values g=32",
                   "step_32_layers": {"ms": step_ms, "GB_per_s": step_all / (step_ms * 1e-3) / 1e9,
                                      "frac_of_peak": step_bytes / (step_ms * 1e-3) / 1e9 / peak,
                                      "tokens_per_s": reduce_sum(16.0, world) / (step_ms * 1e-3),
                                      "cache_bytes": step_all,
                                      "timing": "all 32 layer caches resident; one decode per layer "
                                                "in order, events around the 32 decodes, L2 flushed "
                                                "before each step"},
                   "groups": groups,
                   "estimate_from_groups": {"GB_per_s": tot_bytes / (tot_ms * 1e-3) / 1e9,
                                            "tokens_per_s": reduce_sum(16.0, world) / (tot_ms * 1e-3),
                                            "ms_per_token_step": tot_ms,
                                            "how": "one layer per group timed, times 8"}}
    w = synth.WORKLOADS["wide"]
    part, whole, nb, fill = _time_decode(w, 0, dev)
    part, whole = reduce_max(part, world), reduce_max(whole, world)
    nb_all = reduce_sum(float(nb), world)
    res["wide"] = {"workload": "wide: batch 4, 16 query heads over 4 KV heads, d=256, context 262144, "
                               "keys b1=3 + m=256, 4-bit values g=64",
                   "partial_ms": part, "decode_ms": whole, "GB_per_s": nb_all / (part * 1e-3) / 1e9,
                   "frac_of_peak": nb / (part * 1e-3) / 1e9 / peak,
                   "tokens_per_s": reduce_sum(4.0, world) / (whole * 1e-3),
                   "cache_fill": _fill_entry(fill, world, peak)}
    return res


def _fill_entry(fill, world, peak):
    """The one-shot cache fill (every token quantised and appended in one call, on
    the tensor cores at these shapes) as Mkeys/s and HBM fraction of its bytes."""
    ms = reduce_max(fill["ms"], world)
    return {"ms": ms, "Mkeys_per_s": reduce_sum(float(fill["keys"]), world) / (ms * 1e-3) / 1e6,
            "GB_per_s": reduce_sum(float(fill["bytes"]), world) / (ms * 1e-3) / 1e9,
            "frac_of_peak": fill["bytes"] / (ms * 1e-3) / 1e9 / peak}


def bench_quantize(dev, world, reps=3, keep_sample=False):
    """Chunked append of the quantise workload; with keep_sample, the inputs and
    the packed region of (batch 0, KV head 0) on the host (for the oracle check
    of the CPU-baseline leg)."""
    import torch
    import synth
    from compressed_attention_turboquantprod_b200 import Codebook, CompressedKVCache, Projections
    w = synth.WORKLOADS["quant"]
    pj, cb = Projections(w.d, w.m, 0, device=dev), Codebook(w.d, w.b1, device=dev)
    K, V = synth.keys_values(w, device=dev)
    chunks = [(K[:, :, t:t + w.chunk].contiguous(), V[:, :, t:t + w.chunk].contiguous())
              for t in range(0, w.T, w.chunk)]
    sample = None
    if keep_sample:
        sample = {"K": K[0, 0].double().cpu().numpy(), "V": V[0, 0].double().cpu().numpy()}
    del K, V
    cache = CompressedKVCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, w.W, w.T,
                              dtype=w.torch_dtype, device=dev)
    stream = torch.cuda.current_stream(dev)

    def timed(proj):
        times = []
        for r in range(reps + 1):
            cache.state.n_total = 0
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for k, v in chunks:
                cache.append(k, v, proj, cb)
            e1.record(stream)
            torch.cuda.synchronize()
            if r > 0:
                times.append(e0.elapsed_time(e1))
        return reduce_max(min(times), world)
    ms = timed(pj)
    region = cache.buffer[:cache.state.region_bytes]
    ref_sum = int(region.view(torch.int32).sum().item())
    # the same 32 appends captured once as a CUDA graph and replayed: the device
    # time without the host's per-call launch work (same kernels, same bytes)
    graph = {}
    try:
        g = torch.cuda.CUDAGraph()
        cache.state.n_total = 0
        torch.cuda.synchronize()
        with torch.cuda.graph(g):
            for k, v in chunks:
                cache.append(k, v, pj, cb)
        times = []
        for r in range(reps + 1):
            region.zero_()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            if r > 0:
                times.append(e0.elapsed_time(e1))
        gms = reduce_max(min(times), world)
        graph = {"Mkeys_per_s": reduce_sum(float(w.T * w.Hkv * w.B), world) / (gms * 1e-3) / 1e6,
                 "ms": gms, "same_bytes_as_the_calls": int(region.view(torch.int32).sum().item()) == ref_sum}
        del g
    except Exception as ex:          # a capture the runtime refuses: report, do not fail
        graph = {"unavailable": str(ex)[:200]}
    torch.cuda.synchronize()
    # the same append with the structured (Hadamard) rotation
    ms_h = timed(Projections(w.d, w.m, 0, device=dev, structured=True))
    keys = reduce_sum(float(w.T * w.Hkv * w.B), world)
    tb = cache.state.token_bytes
    if sample is not None:
        # the Hadamard pass ran last: append once more with the QR projections
        cache.state.n_total = 0
        for k, v in chunks:
            cache.append(k, v, pj, cb)
        torch.cuda.synchronize()
        sample["region"] = cache.buffer[:cache.state.region_bytes].cpu().numpy()
    nbytes = w.T * w.Hkv * w.B * (2 * w.d * 2 + tb)
    res = {"Mkeys_per_s": keys / (ms * 1e-3) / 1e6, "ms": ms, "keys": int(keys),
            "graph": graph,
            "Mkeys_per_s_hadamard_rotation": keys / (ms_h * 1e-3) / 1e6,
            "GB_per_s": reduce_sum(float(nbytes), world) / (ms * 1e-3) / 1e9,
            "workload": "quant: 131072 tokens x 8 KV heads, d=128, bf16, appended in chunks of 4096; "
                        "keys b1=2 + m=128, values 2-bit g=32 (key + value per key)"}
    return res, sample


def bench_structured_rotation(dev, world, reps=5):
    """What the fast Walsh-Hadamard transform buys where the rotation runs on CUDA
    cores: the SGEMM tile quantiser (d = 64, the head dim without a tensor-core
    path; 8 KV heads x 16384 tokens per append) and the single-token append of a
    decode step on the 32K GQA shape, each with the dense QR rotation and with the
    structured one (same data)."""
    import torch
    import synth
    from compressed_attention_turboquantprod_b200 import Codebook, CompressedKVCache, Projections
    stream = torch.cuda.current_stream(dev)

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return reduce_max(e0.elapsed_time(e1) / reps, world)

    res = {}
    w = _sgemm_workload()
    K, V = synth.keys_values(w, device=dev)
    cb = Codebook(w.d, w.b1, device=dev)
    keys = w.B * w.Hkv * w.T
    for structured in (False, True):
        pj = Projections(w.d, w.m, 0, device=dev, structured=structured)
        cache = CompressedKVCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, 0, w.T,
                                  dtype=w.torch_dtype, device=dev, structured=structured)

        def call():
            cache.state.n_total = 0
            cache.append(K, V, pj, cb)
        ms = timed(call)
        res["tile_quantise_d64_Mkeys_per_s_" + ("hadamard" if structured else "dense")] = \
            reduce_sum(keys / (ms * 1e-3) / 1e6, world)
        del cache
    del K, V
    w = synth.WORKLOADS["gqa32k"].scaled(T=4096)
    K, V = synth.keys_values(w, device=dev)
    cb = Codebook(w.d, w.b1, device=dev)
    n_calls = reps + 1
    _, Kn, Vn = synth.decode_stream(w, n_calls, device=dev)
    for structured in (False, True):
        pj = Projections(w.d, w.m, 0, device=dev, structured=structured)
        cache = CompressedKVCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, w.W,
                                  w.T + n_calls + 64, dtype=w.torch_dtype, device=dev,
                                  structured=structured)
        cache.append(K, V, pj, cb)
        state = {"i": 0}

        def step():
            i = state["i"]
            state["i"] = i + 1
            cache.append(Kn[i], Vn[i], pj, cb)
        ms = timed(step)
        res["single_token_append_us_" + ("hadamard" if structured else "dense")] = ms * 1e3
        del cache
    res["workloads"] = ("tile quantiser: d=64, b1=2, m=64, 2-bit values g=32, 8 KV heads x 16384 "
                        "bf16 tokens per append; single-token append: batch 8, 8 KV heads, d=128, "
                        "b1=2, m=128, 16-token ring (the token leaving the ring is quantised)")
    return res


def _sgemm_workload():
    """A shape the tile quantiser keeps on the CUDA-core SGEMM (d = 64)."""
    import synth
    return synth.Workload("quantize_sgemm", B=1, Hq=16, Hkv=8, d=64, T=16384, W=0, b1=2, m=64,
                          vbits=2, group=32, dtype="bf16", k_outlier_frac=0.02,
                          v_outlier_frac=0.02, outlier_scale=8.0)


def oracle_quantize_counts(sample):
    """The oracle's one-shot quantisation of the sampled unit's 131072 tokens
    against the library's chunked append of them: near-boundary exemption counts
    of the key codes and sign bits, and value fields (must be bit-exact)."""
    import numpy as np
    import synth
    from oracle import cache as ocache, codebook as ocb, layout as olayout
    from oracle import projections as oproj, quantize as oq
    w = synth.WORKLOADS["quant"]
    po, cb = oproj.make_projections(w.d, w.m, 0), ocb.build(w.d, w.b1)
    oc = ocache.OracleCache(1, 1, w.d, w.b1, w.m, w.vbits, w.group, w.W, w.T, w.dtype, po, cb)
    oc.append(sample["K"][None, None], sample["V"][None, None])
    r = oc.rec[0][0]
    n = r["rho"].shape[0]
    buf = np.zeros(oc.lay.total_bytes, np.uint8)
    buf[:oc.lay.region_bytes] = sample["region"][:oc.lay.region_bytes]
    fg = olayout.decode_fields(olayout.read_region(buf, oc.lay, 0, 0, n), oc.lay)
    counts = oq.band_agreement(fg["idx"], fg["bits"], r, cb[1])
    counts["value_field_mismatches"] = int(
        np.sum(fg["codes"] != r["codes"]) + np.sum(fg["scale"] != r["scale"].astype(np.float32))
        + np.sum(fg["vmin"] != r["vmin"].astype(np.float32)))
    counts["sample"] = "batch 0, KV head 0: all 131072 tokens of the chunked append"
    return counts


# --------------------------------------------------------------------------- per-kernel cases
# Small workloads (inputs above L2 where the kernel streams, a few GB at most), one
# call repeated, each reaching one or two kernels that the main bench does not
# time on its own; `bench.py --case NAME` prints one JSON line with the mean call
# time (CUDA events, L2 flushed before each call).
CASES = {
    "decode_cuda_core": "CUDA-core decode (k_decode_prep, k_decode_partial, k_decode_combine): "
                        "batch 8, 16 query heads over 8 KV heads (G = 2: no tensor-core path), "
                        "d = 64, context 32768, keys b1 = 2 + QJL m = 64, 2-bit values g = 32, bf16",
    "quantize_sgemm": "64-token SGEMM tile quantise (k_quantize, the shapes without a tensor-core "
                      "path): d = 64, b1 = 2, m = 64, 2-bit values g = 32, bf16, 8 KV heads x 16384 "
                      "tokens per call",
    "quantize_sgemm_hadamard": "the same with the structured rotation (the per-row fast "
                               "Walsh-Hadamard transform instead of the rotation GEMM)",
    "quantize_tc_wide": "tcgen05 tile quantise on streamed operand pieces (k_operand_image, "
                        "k_quantize_tcg): the 262K wide-head shape (d = 256, b1 = 3, m = 256, 4-bit "
                        "values g = 64, bf16), 4 KV heads x 32768 tokens per call",
    "quantize_tc_aqjl": "the same kernel on the A-QJL shape of layers 0-7 (pure QJL, d = 128, "
                        "m = 512, fp16 keys, 2-bit values g = 32), 8 KV heads x 65536 tokens per call",
    "append_small": "single-token append (k_quantize_small, k_ring_write): the 32K GQA cache "
                    "(batch 8, 8 KV heads, d = 128, 16-token ring), one token per sequence per call",
    "prefill": "multi-token call (history partial, k_prefill_exact, merge) on the 32K GQA "
               "cache, 16-token chunk",
    "prefill64": "the same with a 64-token chunk",
}


def run_case(args):
    import torch
    import synth
    from compressed_attention_turboquantprod_b200 import (Codebook, CompressedKVCache, Projections,
                                                           native)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def timed(fn, reps=args.steps, warm=args.warmup):
        for _ in range(warm):
            flush_w.zero_()
            fn()
        tot = 0.0
        for _ in range(reps):
            flush_w.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            tot += e0.elapsed_time(e1)
        return tot / reps

    name = args.case
    out = {"case": name, "what": CASES[name]}
    if name == "decode_cuda_core":
        w = synth.Workload("decode_cuda_core", B=8, Hq=16, Hkv=8, d=64, T=32768, W=16, b1=2, m=64,
                           vbits=2, group=32, dtype="bf16", k_outlier_frac=0.02,
                           v_outlier_frac=0.02, outlier_scale=8.0)
        pj, cb = Projections(w.d, w.m, 0, device=dev), Codebook(w.d, w.b1, device=dev)
        cache = CompressedKVCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, w.W, w.T,
                                  dtype=w.torch_dtype, device=dev)
        K, V = synth.keys_values(w, device=dev)
        cache.append(K, V, pj, cb)
        del K, V
        Q = synth.queries(w, device=dev)
        o = torch.empty_like(Q)
        ws = cache.workspace(w.Hq)
        scale = 1.0 / math.sqrt(w.d)
        ms = timed(lambda: native.tq_decode_attention(cache.state, Q, scale, pj.Pi, pj.S,
                                                      cb.centroids, o, None, 0, ws))
        nb = w.B * w.Hkv * (cache.n_comp * cache.state.token_bytes + 2 * cache.n_ring * w.d * 2)
        out.update(ms=ms, packed_bytes=nb, GB_per_s=nb / (ms * 1e-3) / 1e9)
    elif name.startswith("quantize_"):
        if name.startswith("quantize_sgemm"):
            w = _sgemm_workload()
        elif name == "quantize_tc_wide":
            w = synth.WORKLOADS["wide"].scaled(B=1, T=32768)
        else:
            w = synth.WORKLOADS["aqjl"].scaled(B=1, T=65536, m=512)
        structured = name.endswith("hadamard")
        pj = Projections(w.d, w.m, 0, device=dev, rotation=w.b1 > 0, structured=structured)
        cb = Codebook(w.d, w.b1, device=dev) if w.b1 else None
        cache = CompressedKVCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, 0, w.T,
                                  dtype=w.torch_dtype, device=dev, structured=structured)
        K, V = synth.keys_values(w, device=dev)

        def call():
            cache.state.n_total = 0
            cache.append(K, V, pj, cb)
        ms = timed(call)
        keys = w.B * w.Hkv * w.T
        nbytes = keys * (2 * w.d * (4 if w.dtype == "f32" else 2) + cache.state.token_bytes)
        out.update(ms=ms, keys=keys, Mkeys_per_s=keys / (ms * 1e-3) / 1e6,
                   GB_per_s=nbytes / (ms * 1e-3) / 1e9)
    elif name == "append_small":
        w = synth.WORKLOADS["gqa32k"]
        pj, cb = Projections(w.d, w.m, 0, device=dev), Codebook(w.d, w.b1, device=dev)
        n_calls = args.warmup + args.steps
        cache = CompressedKVCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, w.W,
                                  w.T + n_calls + 64, dtype=w.torch_dtype, device=dev)
        K, V = synth.keys_values(w, device=dev)
        cache.append(K, V, pj, cb)
        del K, V
        _, Kn, Vn = synth.decode_stream(w, n_calls, device=dev)
        it = iter(range(n_calls))

        def call():
            i = next(it)
            cache.append(Kn[i], Vn[i], pj, cb)
        ms = timed(call)
        out.update(ms=ms, tokens_per_call=w.B * w.Hkv)
    elif name.startswith("prefill"):
        nq = 64 if name == "prefill64" else 16
        w = synth.WORKLOADS["gqa32k"]
        pj, cb = Projections(w.d, w.m, 0, device=dev), Codebook(w.d, w.b1, device=dev)
        cache = CompressedKVCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, w.W, w.T,
                                  dtype=w.torch_dtype, device=dev)
        K, V = synth.keys_values(w, device=dev)
        cache.append(K, V, pj, cb)
        del K, V
        Q, Kc, Vc = synth.prefill_chunk(w, nq, device=dev)
        o = torch.empty_like(Q)
        ws = torch.empty(native.tq_prefill_workspace_bytes(cache.state, w.Hq, nq, 0),
                         dtype=torch.uint8, device=dev)
        scale = 1.0 / math.sqrt(w.d)
        ms = timed(lambda: native.tq_prefill_attention(cache.state, Q, Kc, Vc, scale, pj.Pi, pj.S,
                                                       cb.centroids, o, 0, ws))
        native.tq_prefill_check(cache.state, w.Hq, nq, 0, ws)
        out.update(ms=ms, query_tokens=w.B * nq)
    torch.cuda.synchronize()
    print(json.dumps(out), flush=True)
    return 0


def main():
    args = parse_args()
    if args.case:
        return run_case(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
