#!/usr/bin/env python
"""Benchmark of the page indexer's hot path on B200.

One step = one ``score_topk_fused`` call over a whole batch of the ragged
decode workload: B=32 requests, Q=4 query heads, D=128, pages per request
uniform on 1024..65536 inside a padded N=65536, K=256 (seed 103; rank r of a
multi-GPU run draws its own batch from seed 103 + 1000 r).  Every valid page is
scored against its request's query heads and the top-K page indices of each
request are written.  The metric is valid pages scored+selected per second
(whole job) and the HBM bandwidth that implies.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                       [--workload ragged_decode|prefill_chunk|causal_decode|...]

The default workload is the headline one above.  The others are the indexer's
remaining workloads, for profiling: a prefill chunk (B=4, T=16, Q=8, N=131072,
K=512; every token row of 131072 pages selects its top 512) counts one unit per
(token row, page); a multi-token causal decode step (B=32 requests, 4 new
tokens each, per-token page counts, K=256) counts one unit per (token row,
valid page of that row).
For N > 1 launch under torch.distributed.run: requests are sharded across ranks
(each rank owns its batch; no collective on the data path), timing is the max
over ranks.  ``--impl reference`` times the CPU oracle (single-threaded C) on
a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "pages scored+selected/sec and HBM GB/s vs 8 TB/s at B=32,N=65536,K=256"
UNIT = "pages/s"
WORKLOAD = "ragged_decode"
NOMINAL_HBM_GBS = 8000.0
# The one kernel a step launches: tcgen05 scoring (D=128, query rows unrolled
# to 16), fused with the histogram-driven top-K select.
KERNEL = "decode_tc_kernel<D=128,NC=16,fused,hist>"
PREFILL_KERNEL = "prefill_kernel<Q=8> (tcgen05 score of a 16-token chunk)"
FALLBACK_HBM_GBS = 6650.0
# The ncu summary of the headline kernel records its DRAM bytes per valid page
# beside a digest of the library sources it was captured on; the traffic is
# reported only while the sources still have that digest.
L2_BYTES = 126 << 20
TRAFFIC_SUMMARY = os.path.join(ROOT, "profiles", "decode_fused_ragged_decode.md")
REPEATS = 11  # timed regions of exactly --steps steps; the median is reported


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=("ragged_decode", "prefill_chunk", "causal_decode", "pool_keys",
                             "paged_decode", "paged_sweep", "topk_sweep", "kmeans_assign",
                             "batch_decode_bias", "tiny_decode"))
    ap.add_argument("--dists", default="normal,levels16,neg_inf_90",
                    help="top-K sweep distributions (comma list, or 'all')")
    ap.add_argument("--topk-case", default=None,
                    help="top-K sweep: only the rows x N case given as ROWSxN (e.g. 128x262144)")
    ap.add_argument("--head-dim", type=int, default=None,
                    help="decode workloads: override D (64 and 128 take the tensor-core "
                         "kernel, other multiples of 8 the CUDA-core one)")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def workload_inputs(rank, name=WORKLOAD, head_dim=None):
    from page_scoring_top_b200 import dist as pdist
    from page_scoring_top_b200 import synth
    spec = dict(synth.WORKLOADS[name])
    seed = pdist.rank_seed(spec["seed"], rank)
    over = {} if head_dim is None else {"D": head_dim}
    return synth.workload(name, seed=seed, **over), spec, seed


def algorithmic_bytes(lengths, B, T, Q, D, K, with_values):
    pages = int(np.sum(lengths))
    b = pages * D * 2 + B * T * Q * D * 2 + B * 4 + B * T * K * 4
    if with_values:
        b += B * T * K * 4
    return pages, b


def source_digest():
    """sha256 (first 16 hex digits) over the library's CUDA sources and header."""
    import glob
    import hashlib
    h = hashlib.sha256()
    files = sorted(glob.glob(os.path.join(ROOT, "page_scoring_top_b200", "csrc", "*")))
    for f in files + [os.path.join(ROOT, "include", "idx.h")]:
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode() + b"\0" + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic_per_page():
    """(bytes per valid page, note) from the committed ncu summary, or (None,
    why) when the summary is missing or the sources changed since its capture."""
    import re
    try:
        with open(TRAFFIC_SUMMARY) as f:
            text = f.read()
    except OSError:
        return None, "no ncu summary"
    m = re.search(r"traffic_bytes_per_page\s*=\s*([0-9.]+)\s*;\s*sources\s*=\s*([0-9a-f]+)", text)
    if not m:
        return None, "no traffic record in the ncu summary"
    if m.group(2) != source_digest():
        return None, "kernel sources changed since the ncu capture"
    return float(m.group(1)), "ncu capture of this kernel build (dram read + write per page)"


def host_facts():
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


def timed_repeats(step, steps, stream, barrier, repeats=REPEATS):
    """``repeats`` timed regions of exactly ``steps`` steps, each bracketed by
    a barrier and a device synchronize on both sides and timed with CUDA
    events on the launching stream.  Returns the per-region milliseconds."""
    import torch
    out = []
    for _ in range(repeats):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        out.append(e0.elapsed_time(e1))
    return out


def soak(step, seconds):
    """Run untimed steps for about ``seconds`` (the clock sampler's window)."""
    import torch
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        for _ in range(50):
            step()
        torch.cuda.synchronize()


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, copy burst)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s earlier pool measurement)"


def measured_tensor_peak():
    """Dense bf16 TFLOP/s: the measured burst figure, else the recipe's fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops, burst)"
    except Exception:
        return 1590.0, "fallback (1.59 PFLOP/s earlier pool measurement, burst)"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"],
                    "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for name, flag in zip(names, parts[4:8]):
                if flag.lower() in ("active", "1"):
                    reasons.add(name)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": float(max(smax)) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def cpu_oracle_rate(d, K, seconds, max_requests=None):
    """Single-threaded oracle (scores in double + full sort per request) on a
    bounded sample of the workload: whole requests in order, repeated until
    ``seconds`` elapse (at least one request).  Returns (pages/s, description)."""
    import oracle
    q, c, lengths = d["q"], d["c"], d["lengths"]
    B = q.shape[0]
    pages = 0
    done = 0
    t0 = time.perf_counter()
    while True:
        b = done % B
        n = int(lengths[b])
        S, _ = oracle.scores(q[b:b + 1], c[b:b + 1, :max(n, 1)], np.array([n], np.int32))
        oracle.topk_rows(S[0], K, None)
        pages += n
        done += 1
        el = time.perf_counter() - t0
        if el >= seconds or (max_requests and done >= max_requests):
            break
    return pages / el, "%d requests of the workload in order (%d pages), %.1f s, 1 thread" % (
        done, pages, el)


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    d, spec, seed = workload_inputs(0)
    K = spec["K"]
    import oracle
    # Calibrate: one request's oracle time, then size each step's sample so the
    # whole --warmup + --steps run takes about two minutes.
    t0 = time.perf_counter()
    n0 = int(d["lengths"][0])
    S, _ = oracle.scores(d["q"][:1], d["c"][:1, :n0], d["lengths"][:1])
    oracle.topk_rows(S[0], K, None)
    per_page = (time.perf_counter() - t0) / n0
    budget = 120.0 / max(1, args.steps + args.warmup)
    sample_pages = int(max(1024, min(n0, budget / per_page)))
    total_pages = 0
    t_total = 0.0
    for step in range(args.warmup + args.steps):
        b = step % d["q"].shape[0]
        n = int(min(sample_pages, d["lengths"][b]))
        t0 = time.perf_counter()
        S, _ = oracle.scores(d["q"][b:b + 1], d["c"][b:b + 1, :n], np.array([n], np.int32))
        oracle.topk_rows(S[0], K, None)
        el = time.perf_counter() - t0
        if step >= args.warmup:
            total_pages += n
            t_total += el
    value = total_pages / t_total
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * t_total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": WORKLOAD, "B": 32, "T": 1, "Q": 4, "D": 128, "N": 65536, "K": K,
                   "seed": seed, "len_dist": "uniform 1024..65536"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": "per step: the first %d valid pages of one request "
                                   "(requests in turn), scores in double + full sort" %
                                   sample_pages, **host_facts()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch
    rank, world, local = dist_env()
    if world != args.gpus:
        print("warning: --gpus %d but WORLD_SIZE %d" % (args.gpus, world), file=sys.stderr)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist
    from page_scoring_top_b200 import binding

    d, spec, seed = workload_inputs(rank, args.workload, args.head_dim)
    B, T, Q, D = d["q"].shape
    N = d["c"].shape[1]
    K = spec["K"]
    pages, nbytes = algorithmic_bytes(d["lengths"], B, T, Q, D, K, with_values=False)
    units = pages * T  # (token row, valid page) pairs scored and selected
    tok = d.get("token_lengths")
    if tok is not None:
        units = int(np.sum(tok))

    q = torch.from_numpy(d["q"].view(np.int16)).to(dev)
    c = torch.from_numpy(d["c"].view(np.int16)).to(dev)
    ln = torch.from_numpy(d["lengths"]).to(dev)
    tokd = None if tok is None else torch.from_numpy(np.ascontiguousarray(tok)).to(dev)
    idx = torch.empty((B * T, K), dtype=torch.int32, device=dev)
    ctx = binding.Context(local, max_rows=B * T, max_n=N, max_k=K)
    stream = torch.cuda.current_stream(dev)

    # A centroid table below the L2 is replicated until the copies exceed
    # twice the L2, and the steps rotate over them: every step reads inputs
    # that are not L2-resident, back to back.
    small = c.numel() * 2 < L2_BYTES
    copies = [(q, c)]
    if small:
        ncopy = -(-2 * L2_BYTES // (c.numel() * 2))
        copies += [(q.clone(), c.clone()) for _ in range(ncopy - 1)]
    turn = [0]

    def step():
        qq, cc = copies[turn[0] % len(copies)]
        turn[0] += 1
        if tokd is not None:
            binding.score_topk_fused_tokens(ctx, qq, cc, tokd, K, idx, None, stream=stream)
        else:
            binding.score_topk_fused(ctx, qq, cc, ln, K, idx, None, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    rc, bits = binding.idx_get_status(ctx)
    if rc != 0:
        raise RuntimeError("device status %d after warm-up" % bits)

    def barrier():
        if pg is not None:
            pg.barrier()

    sampler = ClockSampler(local if "CUDA_VISIBLE_DEVICES" not in os.environ else
                           os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local])
    barrier()
    torch.cuda.synchronize(dev)
    # The sampler covers a window of load around the timed regions, so that
    # the clock record holds more than one reading even for short regions.
    sampler.start()
    time.sleep(0.15)  # let the sampler take its first reading
    soak(step, 0.3)
    reps = timed_repeats(step, args.steps, stream, barrier)
    soak(step, 0.3)
    clocks = sampler.stop()
    from page_scoring_top_b200 import dist as pdist
    reps_max = [pdist.reduce_timing(r, units, device=dev)[0] for r in reps]
    ms_max = float(np.median(reps_max))
    total_pages = pdist.reduce_timing(0.0, units, device=dev)[1]
    ms = float(np.median(reps))  # this rank's own median region
    ms_per_step = ms_max / args.steps
    value = total_pages * args.steps / (ms_max * 1e-3)
    repeats = {"regions": len(reps_max), "steps_each": args.steps,
               "ms_per_step": [r / args.steps for r in reps_max],
               "median_ms_per_step": ms_per_step,
               "spread": (max(reps_max) - min(reps_max)) / ms_max}
    rc, bits = binding.idx_get_status(ctx)
    if rc != 0:
        raise RuntimeError("device status %d after the timed region" % bits)

    # Roofline of the dominant kernel.  Decode: the fused tensor-core decode
    # kernel is the step's only launch, timed by the events above.  Prefill:
    # the step is the tcgen05 score kernel then the top-K kernel; the score
    # kernel (centroid_score alone) is timed the same way on the same stream.
    peak, peak_src = measured_peak()
    kernel, traffic, traffic_note = KERNEL, None, "no ncu capture for this workload"
    if args.head_dim is not None and args.head_dim not in (64, 128):
        kernel = "decode_kernel<D=%d,fused> (CUDA cores)" % args.head_dim
    elif args.workload == WORKLOAD and args.head_dim is None:
        per_page, traffic_note = recorded_traffic_per_page()
        traffic = None if per_page is None else per_page * pages
    launch_s = (ms / args.steps) * 1e-3
    score_bytes = nbytes
    tensor = None
    if tok is not None:
        kernel = "decode_tc_kernel<D=128,NC=16,fused> (4 token rows per request)"
    elif T > 1:
        kernel = PREFILL_KERNEL
        scores = torch.empty((B, T, N), dtype=torch.float32, device=dev)
        for _ in range(args.warmup):
            binding.centroid_score(ctx, q, c, ln, scores, stream=stream)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            binding.centroid_score(ctx, q, c, ln, scores, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        launch_s = e0.elapsed_time(e1) / args.steps * 1e-3
        # algorithmic bytes of the score kernel: valid centroids + q read,
        # every score written (padding included)
        score_bytes = pages * D * 2 + B * T * Q * D * 2 + B * T * N * 4
        flops = 2.0 * pages * T * Q * D
        tensor = {"achieved_tflops": flops / launch_s / 1e12, "score_kernel_us": launch_s * 1e6}
    achieved = score_bytes / launch_s / 1e9

    e2e = None
    if not args.no_e2e and args.workload == WORKLOAD:
        e2e = measure_e2e(binding, ctx, d, K, dev, stream, args.e2e_steps, barrier, pg)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.workload == WORKLOAD:
        rate, sample = cpu_oracle_rate(d, K, args.cpu_seconds)
        cpu = {"value": rate, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample,
               **host_facts()}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "accumulate": "f32",
            "data": "synthetic",
            "config": {"workload": args.workload, "B": B, "T": T, "Q": Q, "D": D, "N": N, "K": K,
                       "len_dist": ("uniform 1024..65536" if args.workload == WORKLOAD
                                    else "causal: context U{64*1024..64*65536-4} keys, "
                                         "64 keys per page" if tok is not None
                                    else "all pages valid"), "seed": seed,
                       "pages_per_step_per_gpu": pages, "bytes_per_step_per_gpu": nbytes,
                       "parallelism": "dp%d (requests sharded, no data-path collective)" % world,
                       "l2": ("centroid table of %.1f MB is below the 126 MB L2: the steps "
                              "rotate over %d copies of q and c (%.0f MB), back to back"
                              % (c.numel() * 2 / 1e6, len(copies),
                                 len(copies) * c.numel() * 2 / 1e6)) if small else
                             ("inputs larger than L2 (%.1f MB of centroids per step vs 126 MB); "
                              "no flush" % (pages * D * 2 / 1e6))},
            "hbm_gbs": achieved, "hbm_frac_of_8tbs": achieved / NOMINAL_HBM_GBS,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic, "traffic_source": traffic_note,
                         "peak_source": peak_src, "kernel": kernel},
            "gpu_launches": args.steps * (2 if (T > 1 and tok is None) else 1),
            "repeats": repeats,
            "clocks": clocks,
            "tensor": tensor,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    ctx.close()
    if pg is not None:
        pg.destroy_process_group()
    return 0


def measure_e2e(binding, ctx, d, K, dev, stream, steps, barrier, pg):
    """The same step through the public call with host buffers: pinned H2D of
    q, lengths and each request's valid centroid pages, the fused call, and a
    D2H read of the indices, all inside the timed region."""
    import torch
    B, T, Q, D = d["q"].shape
    N = d["c"].shape[1]
    q_h = torch.from_numpy(d["q"].view(np.int16)).pin_memory()
    c_h = torch.from_numpy(d["c"].view(np.int16)).pin_memory()
    ln_h = torch.from_numpy(d["lengths"]).pin_memory()
    idx_h = torch.empty((B * T, K), dtype=torch.int32).pin_memory()
    q = torch.empty_like(q_h, device=dev)
    c = torch.empty_like(c_h, device=dev)
    ln = torch.empty_like(ln_h, device=dev)
    idx = torch.empty((B * T, K), dtype=torch.int32, device=dev)
    lengths = [int(x) for x in d["lengths"]]
    h2d = q_h.numel() * 2 + ln_h.numel() * 4 + sum(lengths) * D * 2
    d2h = idx_h.numel() * 4

    def step():
        q.copy_(q_h, non_blocking=True)
        ln.copy_(ln_h, non_blocking=True)
        for b, n in enumerate(lengths):
            if n:
                c[b, :n].copy_(c_h[b, :n], non_blocking=True)
        binding.score_topk_fused(ctx, q, c, ln, K, idx, None, stream=stream)
        idx_h.copy_(idx, non_blocking=True)

    for _ in range(3):
        step()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ms = e0.elapsed_time(e1)
    from page_scoring_top_b200 import dist as pdist
    ms_max, total_pages = pdist.reduce_timing(ms, sum(lengths), device=dev)
    value = total_pages * steps / (ms_max * 1e-3)
    return {"value": value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": steps, "ms_per_step": ms_max / steps}


def run_pool(args):
    """Page centroids by key mean-pooling (the producer of the centroid
    table): 4 requests x 131072 keys of D=128 in pages of 64, one
    centroid_pool call per step; units are pages pooled."""
    import torch
    from page_scoring_top_b200 import binding, synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    B, P, N, D = 4, 64, 2048, 128
    keys = synth.normal_bf16(107, 1, 0, B * N * P * D).reshape(B, N * P, D)
    counts = np.full(B, N * P, np.int32)
    kd = torch.from_numpy(keys.view(np.int16)).to(dev)
    kc = torch.from_numpy(counts).to(dev)
    cd = torch.empty((B, N, D), dtype=torch.int16, device=dev)
    ctx = binding.Context(0, max_rows=B, max_n=N, max_k=1)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        binding.centroid_pool(ctx, kd, kc, P, cd, stream=stream)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(0)
    sampler.start()
    time.sleep(0.15)
    e0.record(stream)
    for _ in range(args.steps):
        binding.centroid_pool(ctx, kd, kc, P, cd, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1)
    rc, bits = binding.idx_get_status(ctx)
    if rc != 0:
        raise RuntimeError("device status %d" % bits)
    pages = B * N
    nbytes = B * N * P * D * 2 + B * N * D * 2 + B * 4
    launch_s = ms / args.steps * 1e-3
    achieved = nbytes / launch_s / 1e9
    peak, peak_src = measured_peak()
    line = {
        "metric": "pages pooled/sec (key mean-pooling into centroids)", "value": pages / launch_s,
        "unit": "pages/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "accumulate": "f32", "data": "synthetic",
        "config": {"workload": "pool_keys", "B": B, "keys_per_page": P, "pages": N, "D": D,
                   "bytes_per_step": nbytes,
                   "l2": "inputs larger than L2 (%.1f MB of keys per step); no flush" %
                         (B * N * P * D * 2 / 1e6)},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": None, "peak_source": peak_src,
                     "kernel": "pool_kernel"},
        "gpu_launches": args.steps, "clocks": clocks, "e2e": None, "cpu_baseline": None,
    }
    print(json.dumps(line), flush=True)
    ctx.close()
    return 0


def run_paged(args):
    """Paged decode: 32 requests whose page lists (page counts ~ N(4096, 1024),
    clipped to 1..8192) index a shared pool of 16384 centroid blocks; one
    score_topk_fused_paged call per step, K=256; units are valid pages."""
    import torch
    from page_scoring_top_b200 import binding, synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    B, Q, D, N, K, NB = 32, 4, 128, 8192, 256, 16384
    seed = 108
    z = synth.normal(seed, 0, 0, B)
    lengths = np.clip(np.round(4096 + 1024 * z), 1, N).astype(np.int32)
    ids = (synth.u64(seed, 3, 0, B * N) % np.uint64(NB)).astype(np.int32).reshape(B, N)
    pool = synth.normal_bf16(seed, 2, 0, NB * D).reshape(NB, D)
    q = synth.normal_bf16(seed, 1, 0, B * Q * D).reshape(B, 1, Q, D)
    qd = torch.from_numpy(q.view(np.int16)).to(dev)
    pd = torch.from_numpy(pool.view(np.int16)).to(dev)
    ptd = torch.from_numpy(ids).to(dev)
    ld = torch.from_numpy(lengths).to(dev)
    idx = torch.empty((B, K), dtype=torch.int32, device=dev)
    ctx = binding.Context(0, max_rows=B, max_n=N, max_k=K)
    stream = torch.cuda.current_stream(dev)
    step = lambda: binding.score_topk_fused_paged(ctx, qd, pd, ptd, ld, K, idx, None,
                                                  stream=stream)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(0)
    sampler.start()
    time.sleep(0.15)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1)
    rc, bits = binding.idx_get_status(ctx)
    if rc != 0:
        raise RuntimeError("device status %d" % bits)
    pages = int(lengths.sum())
    nbytes = pages * (D * 2 + 4) + B * Q * D * 2 + B * 4 + B * K * 4
    launch_s = ms / args.steps * 1e-3
    achieved = nbytes / launch_s / 1e9
    peak, peak_src = measured_peak()
    line = {
        "metric": "paged pages scored+selected/sec", "value": pages / launch_s, "unit": "pages/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "accumulate": "f32", "data": "synthetic",
        "config": {"workload": "paged_decode", "B": B, "Q": Q, "D": D, "N": N, "K": K,
                   "n_blocks": NB, "len_dist": "N(4096, 1024) clipped to 1..8192",
                   "pages_per_step": pages, "bytes_per_step": nbytes,
                   "l2": "the 4.2 MB block pool stays in L2; page ids and gathers stream"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": None, "peak_source": peak_src,
                     "kernel": "decode_tc_kernel<128,16,fused,hist,paged> (tile::gather4 producer)"},
        "gpu_launches": args.steps, "clocks": clocks, "e2e": None, "cpu_baseline": None,
    }
    print(json.dumps(line), flush=True)
    ctx.close()
    return 0


PAGED_REGIMES = ((256, 64), (512, 128), (1024, 256), (2048, 512), (4096, 1024))
PAGED_BATCHES = (1, 4, 16, 32, 64)


def run_paged_sweep(args):
    """The paged table's own protocol: page counts from five regimes N(256, 64)
    .. N(4096, 1024) (means doubling, sd a quarter of the mean; counts clipped
    to 1 .. 2 x mean) x batch {1, 4, 16, 32, 64}, ids uniform over a shared
    pool of 16384 blocks, head_dim 128, Q = 4.  Each case times
    centroid_score_paged (score only) and score_topk_fused_paged (K = 256),
    every call alone with CUDA events after a 256 MB L2 flush (all cases are
    far below the L2).  Prints one line with every case."""
    import torch
    from page_scoring_top_b200 import binding, synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    Q, D, K, NB, seed = 4, 128, 256, 16384, 110
    peak, peak_src = measured_peak()
    pool = synth.normal_bf16(seed, 2, 0, NB * D).reshape(NB, D)
    pd = torch.from_numpy(pool.view(np.int16)).to(dev)
    nmax = 2 * PAGED_REGIMES[-1][0]
    ctx = binding.Context(0, max_rows=max(PAGED_BATCHES), max_n=nmax, max_k=K)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    steps = max(3, min(args.steps, 100))

    def time_alone(call):
        for _ in range(3):
            call()
        per = []
        for _ in range(steps):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            call()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            per.append(e0.elapsed_time(e1))
        return float(np.median(per))

    cases = []
    sampler = ClockSampler(0)
    sampler.start()
    time.sleep(0.15)
    for ri, (mu, sd) in enumerate(PAGED_REGIMES):
        N = 2 * mu
        for B in PAGED_BATCHES:
            cs = seed + 10 * ri + PAGED_BATCHES.index(B)
            z = synth.normal(cs, 0, 0, B)
            lengths = np.clip(np.round(mu + sd * z), 1, N).astype(np.int32)
            ids = (synth.u64(cs, 3, 0, B * N) % np.uint64(NB)).astype(np.int32).reshape(B, N)
            q = synth.normal_bf16(cs, 1, 0, B * Q * D).reshape(B, 1, Q, D)
            qd = torch.from_numpy(q.view(np.int16)).to(dev)
            ptd = torch.from_numpy(ids).to(dev)
            ld = torch.from_numpy(lengths).to(dev)
            sc = torch.empty((B, 1, N), dtype=torch.float32, device=dev)
            idx = torch.empty((B, K), dtype=torch.int32, device=dev)
            ms_s = time_alone(lambda: binding.centroid_score_paged(ctx, qd, pd, ptd, ld, sc,
                                                                   stream=stream))
            ms_f = time_alone(lambda: binding.score_topk_fused_paged(ctx, qd, pd, ptd, ld, K, idx,
                                                                     None, stream=stream))
            rc, bits = binding.idx_get_status(ctx)
            if rc != 0:
                raise RuntimeError("device status %d" % bits)
            pages = int(lengths.sum())
            nbytes = pages * (D * 2 + 4) + B * Q * D * 2 + B * 4
            cases.append({"regime": "N(%d,%d)" % (mu, sd), "B": B, "pages": pages,
                          "us_score": ms_s * 1e3, "us_fused": ms_f * 1e3,
                          "pages_per_s_score": pages / (ms_s * 1e-3),
                          "pages_per_s_fused": pages / (ms_f * 1e-3),
                          "gbs_score": nbytes / (ms_s * 1e-3) / 1e9})
    clocks = sampler.stop()
    head = max(cases, key=lambda c: c["pages"])
    line = {
        "metric": "paged pages scored/sec (centroid_score_paged, regime x batch sweep)",
        "value": head["pages_per_s_score"], "unit": "pages/s", "n_gpus": 1, "steps": steps,
        "warmup": 3, "ms_per_step": head["us_score"] * 1e-3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "accumulate": "f32",
        "data": "synthetic",
        "config": {"workload": "paged_sweep", "Q": Q, "D": D, "K": K, "n_blocks": NB,
                   "regimes": ["N(%d,%d)" % r for r in PAGED_REGIMES],
                   "batches": list(PAGED_BATCHES),
                   "value_case": "%s B=%d" % (head["regime"], head["B"]),
                   "l2": "flush (256 MB write) before every timed call"},
        "roofline": {"bound": "hbm", "achieved": head["gbs_score"], "peak": peak, "unit": "GB/s",
                     "frac": head["gbs_score"] / peak, "traffic": None, "peak_source": peak_src,
                     "kernel": "decode_tc_kernel<128,16,score,paged> (tile::gather4 producer)"},
        "geomean_us_score": float(np.exp(np.mean(np.log([c["us_score"] for c in cases])))),
        "geomean_us_fused": float(np.exp(np.mean(np.log([c["us_fused"] for c in cases])))),
        "gpu_launches": None, "clocks": clocks, "e2e": None, "cpu_baseline": None,
        "cases": cases,
    }
    print(json.dumps(line), flush=True)
    ctx.close()
    return 0


def run_topk_sweep(args):
    """The standalone top-K sweep: fp32 score rows, rows in {1, 8, 32, 128} x
    N in {4096, 16384, 65536, 262144}, K = 256, each case with its own seed
    (104 + case number).  One topk_select call per step.  Cases whose rows
    fit in L2 get a 256 MB L2 flush before every timed call (each call timed
    alone with CUDA events); larger ones run back to back.  Prints one line
    with every case's time and HBM fraction (rows * (N + K) * 4 bytes)."""
    import torch
    from page_scoring_top_b200 import binding, synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    K = 256
    dists = synth.DISTRIBUTIONS if args.dists == "all" else tuple(args.dists.split(","))
    peak, peak_src = measured_peak()
    ctx = binding.Context(0, max_rows=max(synth.SWEEP_ROWS), max_n=max(synth.SWEEP_N), max_k=K)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    l2_bytes = 126 << 20
    steps = max(3, min(args.steps, 200))
    cases = []
    sampler = ClockSampler(0)
    sampler.start()
    time.sleep(0.15)
    only = None if args.topk_case is None else tuple(int(x) for x in args.topk_case.split("x"))
    for case, rows, n, dist in synth.sweep_cases():
        if dist not in dists or (only is not None and (rows, n) != only):
            continue
        s = torch.from_numpy(synth.score_rows(104 + case, rows, n, dist)).to(dev)
        idx = torch.empty((rows, K), dtype=torch.int32, device=dev)
        call = lambda: binding.topk_select(ctx, s, None, K, idx, None, stream=stream)
        for _ in range(max(3, args.warmup)):
            call()
        nbytes = rows * (n + K) * 4
        per = []
        if nbytes < l2_bytes:
            for _ in range(steps):
                flush.zero_()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                call()
                e1.record(stream)
                torch.cuda.synchronize(dev)
                per.append(e0.elapsed_time(e1))
            ms = float(np.median(per))
        else:
            ms = float(np.median(timed_repeats(call, steps, stream, lambda: None, 5))) / steps
        rc, bits = binding.idx_get_status(ctx)
        if rc != 0:
            raise RuntimeError("device status %d" % bits)
        gbs = nbytes / (ms * 1e-3) / 1e9
        cases.append({"case": case, "rows": rows, "N": n, "dist": dist, "us": ms * 1e3,
                      "rows_per_s": rows / (ms * 1e-3), "hbm_gbs": gbs, "frac": gbs / peak,
                      "l2": "flushed" if nbytes < l2_bytes else "larger than L2"})
        del s, idx
    clocks = sampler.stop()
    big = [c for c in cases if c["rows"] * c["N"] * 4 >= (32 << 20)]
    head = max(cases, key=lambda c: (c["rows"] * c["N"], c["frac"]))
    line = {
        "metric": "top-K rows selected/sec (standalone select, fp32 rows, K=256)",
        "value": head["rows_per_s"], "unit": "rows/s", "n_gpus": 1, "steps": steps,
        "warmup": args.warmup, "ms_per_step": head["us"] * 1e-3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": "topk_sweep", "K": K, "dists": list(dists),
                   "value_case": "rows=%d N=%d %s" % (head["rows"], head["N"], head["dist"]),
                   "l2": "flush (256 MB write) before each call below 126 MB; larger cases "
                         "back to back"},
        "roofline": {"bound": "hbm", "achieved": head["hbm_gbs"], "peak": peak, "unit": "GB/s",
                     "frac": head["frac"], "traffic": None, "peak_source": peak_src,
                     "kernel": "topk select (standalone)",
                     "median_frac_cases_ge_32MB": float(np.median([c["frac"] for c in big]))
                     if big else None},
        "gpu_launches": None, "clocks": clocks, "e2e": None, "cpu_baseline": None,
        "cases": cases,
    }
    print(json.dumps(line), flush=True)
    ctx.close()
    return 0


def run_kmeans(args):
    """KMeans assignment, the second workload: 262144 clustered points, 1024
    centroids, D=128 (seed 109), one kmeans_assign call per step (the h
    pre-pass and the tcgen05 assignment kernel).  Units are points assigned;
    the roofline is the tensor pipe (2 M C D flops per step)."""
    import torch
    from page_scoring_top_b200 import binding, synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    spec = synth.KMEANS
    M, C, D = spec["M"], spec["C"], spec["D"]
    d = synth.kmeans_inputs(spec["seed"], M, C, D)
    xd = torch.from_numpy(d["x"].view(np.int16)).to(dev)
    cd = torch.from_numpy(d["centroids"].view(np.int16)).to(dev)
    assign = torch.empty(M, dtype=torch.int32, device=dev)
    ctx = binding.Context(0, max_rows=1, max_n=C, max_k=1)
    stream = torch.cuda.current_stream(dev)
    step = lambda: binding.kmeans_assign(ctx, xd, cd, assign, None, stream=stream)
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(0)
    sampler.start()
    time.sleep(0.15)
    soak(step, 0.3)
    reps = timed_repeats(step, args.steps, stream, lambda: None)
    clocks = sampler.stop()
    ms = float(np.median(reps)) / args.steps
    rc, bits = binding.idx_get_status(ctx)
    if rc != 0:
        raise RuntimeError("device status %d" % bits)
    flops = 2.0 * M * C * D
    tflops = flops / (ms * 1e-3) / 1e12
    peak, peak_src = measured_tensor_peak()
    nbytes = M * D * 2 + C * D * 2 + M * 4
    line = {
        "metric": "points assigned/sec (KMeans assignment, nearest of 1024 centroids)",
        "value": M / (ms * 1e-3), "unit": "points/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "accumulate": "f32", "data": "synthetic",
        "config": {"workload": "kmeans_assign", "M": M, "C": C, "D": D, "seed": spec["seed"],
                   "points": "clustered: a uniform centroid + 0.5 N(0,1)",
                   "l2": "inputs (%.0f MB of points) larger than half the L2, back to back"
                         % (M * D * 2 / 1e6)},
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": tflops / peak, "traffic": None, "peak_source": peak_src,
                     "kernel": "kmeans_kernel (tcgen05 M128 N256, argmax epilogue)",
                     "hbm_gbs": nbytes / (ms * 1e-3) / 1e9},
        "repeats": {"regions": len(reps), "ms_per_step": [r / args.steps for r in reps]},
        "gpu_launches": 2 * args.steps, "clocks": clocks, "e2e": None, "cpu_baseline": None,
    }
    print(json.dumps(line), flush=True)
    ctx.close()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "pool_keys":
        return run_pool(args)
    if args.workload == "paged_decode":
        return run_paged(args)
    if args.workload == "paged_sweep":
        return run_paged_sweep(args)
    if args.workload == "topk_sweep":
        return run_topk_sweep(args)
    if args.workload == "kmeans_assign":
        return run_kmeans(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
