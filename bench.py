"""Benchmark of the multi-LoRA delta path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]
                    [--workload q_proj|tiny|prefill|mlp|paged|qkv|swapin|linear|moe]

Default workload: the largest single-GPU configuration, the S-LoRA-style
paged step -- 1000 rank-16 adapters on q/k/v/o of 32 layers at hidden 4096
(a 31.25 GiB pool of 1 MiB pages scattered by a seeded permutation), a decode
batch of 512 tokens over 64 distinct adapters drawn Zipf(1.1), and all 128
layer x projection deltas per step: one plan (lora_plan_ids) and 128
lora_apply_plan calls, bf16 inputs, fp32 accumulation.  The pool and the
step's 1 GiB of activations exceed the 126 MB L2, so every matrix reads its
adapters and activations from HBM.

Other workloads (--workload): q_proj (Llama-2-7B q_proj-shaped decode,
d_in = d_out = 4096, rank 16, 32 adapters in a contiguous pool, 64 tokens;
one fused launch per batch; steps rotate over up to 64 buffer sets, > 4x the
L2), tiny, prefill (segmented tensor-core path), mlp (mixed ranks padded to
64, 4096 -> 11008), qkv, linear, moe and swapin.

Printed: one JSON line (rank 0).  value = tokens/s over all ranks; roofline =
algorithmic bytes of the dominant kernel / its mean launch time (CUDA events
on the launching stream) against the measured HBM copy bandwidth;
cpu_baseline = the fp64 oracle on the host cores on a bounded sample; e2e =
the same metric through the C ABI with pinned host buffers copied in and the
result copied out inside the timed region.

With N > 1 (torchrun) every rank runs an independent replica on its own
batches (tokens are independent; the path has no data exchange): weak scaling,
timed per rank with CUDA events and reduced with a max over ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "LoRA-delta tokens/sec and achieved HBM GB/s (% of B200 peak), 1 GPU"
WORKLOADS = {"tiny": 1, "q_proj": 2, "prefill": 3, "mlp": 4, "paged": 5, "qkv": 2, "swapin": 5, "linear": 2,
             "moe": 2}
LINEAR_WORKLOAD = "q_proj layer with its delta fused: y = x W^T + delta, d4096 r16 32 adapters 64 tokens"
MOE_WORKLOAD = ("routed expert pairs: 64 tokens x top-4 of 32 experts, 8 adapters (256 slots), rank 16, "
                "expert projection 2880 -> 2880")
MOE_SHAPE = dict(T=64, k=4, E=32, n_ad=8, d=2880, r=16)
L2_BYTES = 126 * 2 ** 20
FUSED_MAX_T = 256   # batches up to this size are grouped inside the decode kernel (one launch)


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def algorithmic_bytes(w, target: int, ids) -> int:
    """Bytes the delta must move for one call: each distinct adapter's A and B
    at its own rank, x of every adapted row, and y of every adapted row read
    and written."""
    d_in, d_out = w.targets[target]
    act = ids[ids >= 0]
    act = act[w.rank[act] > 0]
    distinct = np.unique(act)
    adapters = int(sum(int(w.rank[a]) * (d_in + d_out) * 2 for a in distinct))
    return adapters + act.size * d_in * 2 + act.size * d_out * 4


def traffic_from_profile(kernel: str, kernel_file: str, workload: str):
    """DRAM bytes per launch recorded from an ncu capture, if it was taken on
    the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "%s_%s.txt" % (kernel, workload))
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    kv = {}
    for ln in lines:
        if ":" in ln:
            k, v = ln.split(":", 1)
            kv[k.strip()] = v.strip()
    try:
        src = open(os.path.join(ROOT, "adapter_deltas_b200", "csrc", kernel_file), "rb").read()
    except OSError:
        return None
    if kv.get("source_sha256") != hashlib.sha256(src).hexdigest():
        return None
    try:
        return int(kv["traffic_bytes_per_launch"].split()[0])
    except (KeyError, ValueError, IndexError):
        return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.QUERY, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        pass

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in out.splitlines():
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- CPU arms


def oracle_inputs(w, target: int, layer: bool = False):
    """The oracle's inputs for one batch of one target (drawn once, outside
    any timed region); layer: the whole projection (base weight W instead of
    a given y)."""
    slots = [int(s) for s in np.unique(w.ids[w.ids >= 0])]
    inp = dict(x=w.x(target), adapters={s: w.adapter(s, target) for s in slots})
    if layer:
        inp["W"] = w.W(target)
    else:
        inp["y"] = w.y_in(target)
    return inp


def time_oracle(w, inp, min_seconds: float, threads: int, max_calls: int = 1 << 30):
    """Run the oracle on whole batches of one target until min_seconds passed
    (or max_calls calls); returns (calls, seconds)."""
    import oracle
    n, t0 = 0, time.perf_counter()
    while True:
        if "W" in inp:
            oracle.lora_linear(inp["x"], inp["W"], w.ids, w.n_slots, inp["adapters"], w.alpha, threads=threads)
        else:
            oracle.lora_apply(inp["x"], inp["y"], w.ids, w.n_slots, inp["adapters"], w.alpha, threads=threads)
        n += 1
        el = time.perf_counter() - t0
        if (min_seconds > 0 and el >= min_seconds) or n >= max_calls:
            break
    return n, el


def cpu_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def run_reference(args, rank: int, world: int):
    """The oracle, timed on the host cores, on the same workload and metric.
    A step is one batch of one target; where the workload's step covers
    several targets of one shape (the paged workload's 128 deltas), the value
    is scaled by their count."""
    if rank != 0:
        return
    if args.workload == "moe":
        return run_reference_moe(args)
    import synth
    w = synth.config(WORKLOADS[args.workload])
    n_t = len(w.targets) if args.workload == "paged" else 3 if args.workload == "qkv" else 1
    threads = min(cpu_threads(), w.T)
    inp = oracle_inputs(w, 0, layer=args.workload == "linear")
    time_oracle(w, inp, 0.0, threads, max_calls=args.warmup)
    n, el = time_oracle(w, inp, 0.0, threads, max_calls=args.steps)
    per_call = el / n
    value = w.T / (per_call * n_t)
    sample = "%d whole batches of %d tokens on target 0" % (n, w.T)
    if args.workload == "linear":
        sample += ", whole layer (x W^T + delta)"
    if n_t > 1:
        sample += " (1 of the %d same-shape deltas of a step; value scaled by %d)" % (n_t, n_t)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * per_call * n_t,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": LINEAR_WORKLOAD if args.workload == "linear" else w.name, "global_batch": w.T,
                   "seq_len": 1, "parallelism": "oracle on host cores"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_reference_moe(args):
    """The oracle on the routed-pair workload: warm-up calls, then K timed."""
    moe_cpu_baseline(0.0, max_calls=args.warmup)
    cb = moe_cpu_baseline(0.0, max_calls=args.steps)
    value = cb["value"]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * MOE_SHAPE["T"] / value,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": MOE_WORKLOAD, "global_batch": MOE_SHAPE["T"], "seq_len": 1,
                   "parallelism": "oracle on host cores"},
        "cpu_baseline": cb,
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline(w, n_targets: int, seconds: float, layer: bool = False):
    """The oracle on a bounded sample of the workload (rank 0, N = 1)."""
    threads = min(cpu_threads(), w.T)
    inp = oracle_inputs(w, 0, layer)
    n, el = time_oracle(w, inp, seconds, threads)
    sample = "%d whole batches of %d tokens on target 0%s (%.1f s)" % (
        n, w.T, ", whole layer (x W^T + delta)" if layer else "", el)
    if n_targets > 1:
        sample += ", value scaled by the %d same-shape deltas of a step" % n_targets
    return {"value": n * w.T / el / n_targets, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": sample}


# ---------------------------------------------------------------- GPU arm


def run_b200(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    import adapter_deltas_b200 as L
    import synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = synth.config(WORKLOADS[args.workload], seed=1000 + WORKLOADS[args.workload] + 1000 * rank)

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    scales_np = np.zeros(w.n_slots, np.float32)
    nz = w.rank > 0
    scales_np[nz] = (w.alpha[nz] / w.rank[nz]).astype(np.float32)
    scales = torch.from_numpy(scales_np).to(dev)
    if args.workload == "paged":
        return run_paged(args, rank, world, dev, w, scales, bf16)
    if args.workload == "qkv":
        return run_qkv(args, rank, world, dev, w, scales, bf16)
    if args.workload == "swapin":
        return run_swapin(args, rank, world, dev, bf16)
    if args.workload == "linear":
        return run_linear(args, rank, world, dev, w, scales, bf16)
    if args.workload == "moe":
        return run_moe(args, rank, world, dev, bf16)

    # one buffer set: pool (all slots loaded), x, y, ids, workspace
    pool_bytes = L.lora_pool_bytes_required(w.targets, w.r_max, w.n_slots, w.page_bytes)
    act_bytes = w.T * sum(d_in + d_out for d_in, d_out in w.targets) * 2
    set_bytes = pool_bytes + act_bytes
    n_sets = max(2, min(64, -(-4 * L2_BYTES // set_bytes)))
    target = 0
    adapters = {}
    for s in range(w.n_slots):
        if w.rank[s] > 0:
            A, B = w.adapter(s, target)
            adapters[s] = (bf16(A), bf16(B))
    x0, y0 = bf16(w.x(target)), bf16(w.y_in(target))
    ids0 = torch.from_numpy(w.ids).to(dev)
    # the prefill workload enters through its segment offsets (the tensor-core path)
    segmented = args.workload == "prefill"
    off0 = torch.from_numpy(w.seg_offsets).to(dev) if segmented else None
    sl0 = torch.from_numpy(w.seg_slot).to(dev) if segmented else None
    sets = []
    for k in range(n_sets):
        mem = torch.empty(pool_bytes, dtype=torch.uint8, device=dev)
        pool = L.lora_pool_create(local_rank, w.targets, w.r_max, w.n_slots, w.page_bytes, mem, w.scatter_seed)
        for s, (A, B) in adapters.items():
            L.lora_pool_load(pool, s, target, int(w.rank[s]), A, B)
        ws = torch.zeros(L.lora_workspace_bytes(pool, target, w.T), dtype=torch.uint8, device=dev)
        sets.append(dict(pool=pool, x=x0.clone(), y=y0.clone(), ids=ids0.clone(), ws=ws,
                         off=off0.clone() if segmented else None, sl=sl0.clone() if segmented else None))
    torch.cuda.synchronize()

    def call(s):
        if segmented:
            L.lora_apply_segments(s["pool"], target, s["x"], s["y"], s["off"], s["sl"], scales, s["ws"])
        else:
            L.lora_apply(s["pool"], target, s["x"], s["y"], s["ids"], scales, s["ws"])

    def step(k):
        call(sets[k % n_sets])

    def barrier():
        sync_ranks(world)

    # ---- timed region: a CUDA graph of exactly K whole steps
    g_warm, _ = capture_graph(dev, step, range(args.warmup))
    g_main, launches = capture_graph(dev, step, range(args.warmup, args.warmup + args.steps))
    g_warm.replay()
    torch.cuda.synchronize()
    barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local_rank)
    with sampler:
        torch.cuda.synchronize()
        ev0.record()
        g_main.replay()
        ev1.record()
        torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier()
    ms = ev0.elapsed_time(ev1) / args.steps
    ms = reduce_max(ms, world, dev)

    # ---- dominant kernel alone.  Batches of at most 256 rows are one launch
    # (rows grouped inside the delta kernel), so the kernel is the step; larger
    # ones time the delta launches on prebuilt plans.
    one_launch = (not segmented) and w.T <= FUSED_MAX_T
    if not one_launch:
        for s in sets:
            if segmented:
                L.lora_plan_segments(s["pool"], s["off"], s["sl"], w.T, s["ws"])
            else:
                L.lora_plan_ids(s["pool"], s["ids"], s["ws"])
    reps = max(args.steps, 3 * n_sets)

    def apply_only(k):
        s = sets[k % n_sets]
        if one_launch:
            call(s)
        else:
            L.lora_apply_plan(s["pool"], target, s["x"], s["y"], scales, s["ws"])

    g_kw, _ = capture_graph(dev, apply_only, range(n_sets))
    g_k, _ = capture_graph(dev, apply_only, range(reps))
    g_kw.replay()
    torch.cuda.synchronize()
    ev0.record()
    g_k.replay()
    ev1.record()
    torch.cuda.synchronize()
    kernel_ms = ev0.elapsed_time(ev1) / reps

    # ---- end to end through the C ABI with pinned host buffers: each step
    # copies its inputs (ids or segment table, x, y) in from one packed
    # pinned buffer with one copy, runs the call on views of the device copy,
    # and copies y back out
    idx_host = (torch.cat([off0, sl0]) if segmented else ids0).cpu()
    parts = [idx_host.view(torch.uint8), x0.cpu().view(torch.uint8).reshape(-1), y0.cpu().view(torch.uint8).reshape(-1)]
    offs, total = [], 0
    for t_ in parts:
        offs.append(total)
        total += -(-t_.numel() // 256) * 256
    packed_h = torch.zeros(total, dtype=torch.uint8).pin_memory()
    for o, t_ in zip(offs, parts):
        packed_h[o:o + t_.numel()] = t_
    yout = torch.empty(y0.shape, dtype=torch.bfloat16).pin_memory()
    h2d = total
    d2h = yout.numel() * 2
    packed_d = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(n_sets)]

    def views(k):
        buf = packed_d[k % n_sets]
        n_idx = idx_host.numel()
        idx = buf[offs[0]:offs[0] + n_idx * 4].view(torch.int32)
        x = buf[offs[1]:offs[1] + x0.numel() * 2].view(torch.bfloat16).view(x0.shape)
        y = buf[offs[2]:offs[2] + y0.numel() * 2].view(torch.bfloat16).view(y0.shape)
        return idx, x, y

    def e2e_step(k):
        s = sets[k % n_sets]
        packed_d[k % n_sets].copy_(packed_h, non_blocking=True)
        idx, x, y = views(k)
        if segmented:
            n_off = off0.numel()
            L.lora_apply_segments(s["pool"], target, x, y, idx[:n_off], idx[n_off:], scales, s["ws"])
        else:
            L.lora_apply(s["pool"], target, x, y, idx, scales, s["ws"])
        yout.copy_(y, non_blocking=True)

    g_ew, _ = capture_graph(dev, e2e_step, range(args.warmup))
    g_e, _ = capture_graph(dev, e2e_step, range(args.steps))
    g_ew.replay()
    torch.cuda.synchronize()
    barrier()
    ev0.record()
    g_e.replay()
    ev1.record()
    torch.cuda.synchronize()
    e2e_ms = reduce_max(ev0.elapsed_time(ev1) / args.steps, world, dev)
    del g_warm, g_main, g_kw, g_k, g_ew, g_e

    for s in sets:
        L.lora_pool_destroy(s["pool"])
    if rank != 0:
        return

    peak, peak_kind = load_peaks()
    alg = algorithmic_bytes(w, target, w.ids)
    achieved = alg / (kernel_ms * 1e-3) / 1e9
    tokens = w.T * world
    value = job_value(w.T, world, ms)
    if segmented:
        kernel_name = "prefill_kernels"
        kernel_desc = ("prefill kernels (tcgen05 shrink + expand) for every segment (%d segments)" % len(w.seg_slot)
                       if L.lora_mma_min_rows_for(len(w.seg_slot), w.T) == 1 else
                       "prefill kernels (tcgen05) + decode_kernel launch for segments under %d rows"
                       % L.lora_mma_min_rows())
    elif one_launch:
        kernel_name, kernel_desc = "decode_kernel", "decode_kernel<fused> grouping the batch in-kernel (the whole step)"
    else:
        kernel_name, kernel_desc = "decode_kernel", "decode_kernel<fused> on a prebuilt plan"
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "global_batch": tokens, "seq_len": 1,
                   "parallelism": "replicas%d" % world if world > 1 else "single",
                   "adapters_in_batch": int(np.unique(w.ids[w.ids >= 0]).size),
                   "l2": "%d rotating buffer sets, %.0f MB > 4x L2" % (n_sets, n_sets * set_bytes / 1e6),
                   "timing": "CUDA graph of the K steps, CUDA events around its replay"},
        "hbm_gbs_step": alg * world / (ms * 1e-3) / 1e9 / world,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind,
                     "traffic": traffic_from_profile(kernel_name, "prefill.cu" if segmented else "decode.cu",
                                                     args.workload),
                     "traffic_note": "DRAM bytes of one launch (prefill: shrink + expand launches) from the ncu "
                                     "summary in profiles/, while its source hash matches",
                     "kernel": kernel_desc, "kernel_us": kernel_ms * 1e3,
                     "algorithmic_bytes_per_launch": alg, "frac_of_8TBps_datasheet": achieved / 8000.0},
        "e2e": {"value": job_value(w.T, world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "clocks": clocks,
        "delta_vs_base_w_read": (kernel_ms * 1e-3) / (sum(a * b for a, b in w.targets[:1]) * 2 / (peak * 1e9)),
    }
    if segmented:
        # the contraction's own rate, for context: 2 flops per multiply-add of
        # the shrink (r x d_in per row) and the expand (d_out x r per row)
        d_in, d_out = w.targets[target]
        rows = w.ids >= 0
        flops = float(sum(2.0 * int(w.rank[w.ids[t]]) * (d_in + d_out) for t in np.nonzero(rows)[0]))
        line["tensor_tflops"] = flops / (kernel_ms * 1e-3) / 1e12
    if world == 1:
        line["cpu_baseline"] = cpu_baseline(w, 1, args.cpu_seconds)
    print(json.dumps(line), flush=True)


def run_paged(args, rank, world, dev, w, scales, bf16):
    """All 128 layer x projection deltas of one decode step over the 31.25 GiB
    paged pool: one plan, then one lora_apply_plan per matrix."""
    import torch

    import adapter_deltas_b200 as L
    T, n_t = w.T, len(w.targets)
    active = [int(s) for s in w.active_slots]
    # --pool active: pages for the batch's active slots only (a few GB, for
    # profiler captures); the kernels read the same bytes per matrix
    n_pages_slots = len(active) if args.pool == "active" else w.n_slots
    pool_bytes = L.lora_pool_bytes_required(w.targets, w.r_max, n_pages_slots, w.page_bytes)
    mem = torch.empty(pool_bytes, dtype=torch.uint8, device=dev)
    pool = L.lora_pool_create(dev.index, w.targets, w.r_max, w.n_slots, w.page_bytes, mem, w.scatter_seed)
    w.prefetch(active, range(n_t))
    for s in active:
        for t in range(n_t):
            A, B = w.adapter(s, t)
            L.lora_pool_load(pool, s, t, int(w.rank[s]), bf16(A), bf16(B))
    g = torch.Generator(device=dev).manual_seed(7)
    fa = (torch.randn(16, 4096, generator=g, device=dev) / 64).to(torch.bfloat16)
    fb = (torch.randn(4096, 16, generator=g, device=dev) * 0.14).to(torch.bfloat16)
    act = set(active)
    for s in range(w.n_slots if args.pool == "full" else 0):
        if s not in act:
            for t in range(n_t):
                L.lora_pool_load(pool, s, t, 16, fa, fb)
    xs = [bf16(w.x(t)) for t in range(n_t)]
    ys = [bf16(w.y_in(t)) for t in range(n_t)]
    w.drop()
    ids = torch.from_numpy(w.ids).to(dev)
    ws = torch.zeros(L.lora_workspace_bytes(pool, 0, T), dtype=torch.uint8, device=dev)

    def step(_k):
        L.lora_plan_ids(pool, ids, ws)
        for t in range(n_t):
            L.lora_apply_plan(pool, t, xs[t], ys[t], scales, ws)

    g_warm, _ = capture_graph(dev, step, range(args.warmup))
    g_main, launches = capture_graph(dev, step, range(args.steps))
    g_warm.replay()
    torch.cuda.synchronize()
    sync_ranks(world)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index)
    with sampler:
        torch.cuda.synchronize()
        ev0.record()
        g_main.replay()
        ev1.record()
        torch.cuda.synchronize()
    clocks = sampler.stop()
    sync_ranks(world)
    ms = reduce_max(ev0.elapsed_time(ev1) / args.steps, world, dev)

    # kernel alone: the 128 applies without the plan
    def applies(_k):
        for t in range(n_t):
            L.lora_apply_plan(pool, t, xs[t], ys[t], scales, ws)

    g_k, _ = capture_graph(dev, applies, range(args.steps))
    ev0.record()
    g_k.replay()
    ev1.record()
    torch.cuda.synchronize()
    kernel_ms = ev0.elapsed_time(ev1) / (args.steps * n_t)

    # end to end: each step copies the ids and every matrix's x and y in from
    # pinned host memory and every y back out (one staging buffer each,
    # reused across the matrices)
    xh = xs[0].cpu().pin_memory()
    yh = ys[0].cpu().pin_memory()
    idh = ids.cpu().pin_memory()
    yout = torch.empty_like(yh).pin_memory()
    h2d = idh.numel() * 4 + n_t * (xh.numel() + yh.numel()) * 2
    d2h = n_t * yout.numel() * 2

    def e2e_step(_k):
        ids.copy_(idh, non_blocking=True)
        L.lora_plan_ids(pool, ids, ws)
        for t in range(n_t):
            xs[t].copy_(xh, non_blocking=True)
            ys[t].copy_(yh, non_blocking=True)
            L.lora_apply_plan(pool, t, xs[t], ys[t], scales, ws)
            yout.copy_(ys[t], non_blocking=True)

    e2e_steps = max(1, min(args.steps, 20))
    g_e, _ = capture_graph(dev, e2e_step, range(e2e_steps))
    g_e.replay()
    torch.cuda.synchronize()
    sync_ranks(world)
    ev0.record()
    g_e.replay()
    ev1.record()
    torch.cuda.synchronize()
    sync_ranks(world)
    e2e_ms = reduce_max(ev0.elapsed_time(ev1) / e2e_steps, world, dev)
    del g_warm, g_main, g_k, g_e
    L.lora_pool_destroy(pool)
    if rank != 0:
        return
    peak, peak_kind = load_peaks()
    alg = algorithmic_bytes(w, 0, w.ids)
    achieved = alg / (kernel_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": job_value(T, world, ms), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "global_batch": T * world, "seq_len": 1,
                   "parallelism": "replicas%d" % world if world > 1 else "single",
                   "deltas_per_step": n_t,
                   "pool": ("31.25 GiB, every slot loaded" if args.pool == "full"
                            else "pages of the %d active slots only" % len(active)),
                   "l2": "pool and 1 GiB of activations per step > L2",
                   "timing": "CUDA graph of the K steps, CUDA events around its replay"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_kind": peak_kind, "traffic": traffic_from_profile("decode_kernel", "decode.cu", "paged"),
                     "kernel": "decode_kernel<fused>", "kernel_us": kernel_ms * 1e3,
                     "algorithmic_bytes_per_launch": alg},
        "e2e": {"value": job_value(T, world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": launches, "clocks": clocks,
    }
    if world == 1:
        line["cpu_baseline"] = cpu_baseline(w, n_t, args.cpu_seconds)
    print(json.dumps(line), flush=True)


def run_qkv(args, rank, world, dev, w2, scales, bf16):
    """The q_proj decode batch (64 tokens, 32 rank-16 adapters, ids of the
    q_proj workload) on the q, k and v projections of one layer (three
    4096 x 4096 targets with their own adapter weights) that share x: one
    lora_apply_multi per step into a fused [64, 3 x 4096] y, against three
    lora_apply calls for context."""
    import torch

    import adapter_deltas_b200 as L
    import synth
    d = 4096
    w = synth.custom(2000 + rank, w2.T, [(d, d)] * 3, [int(r) for r in w2.rank], int(w2.r_max), ids=w2.ids)
    T, n_t = w.T, 3
    cols = [0, d, 2 * d]
    pool_bytes = L.lora_pool_bytes_required(w.targets, w.r_max, w.n_slots, 0)
    act_bytes = T * (d + 3 * d) * 2
    n_sets = max(2, min(64, -(-4 * L2_BYTES // (pool_bytes + act_bytes))))
    adapters = {}
    for s_ in range(w.n_slots):
        for t in range(n_t):
            A, B = w.adapter(s_, t)
            adapters[(s_, t)] = (bf16(A), bf16(B))
    x0 = bf16(w.x(0))
    y0 = torch.cat([bf16(w.y_in(t)) for t in range(n_t)], dim=1).contiguous()
    ids0 = torch.from_numpy(w.ids).to(dev)
    sets = []
    for k in range(n_sets):
        mem = torch.empty(pool_bytes, dtype=torch.uint8, device=dev)
        pool = L.lora_pool_create(dev.index, w.targets, w.r_max, w.n_slots, 0, mem, 0)
        for (s_, t), (A, B) in adapters.items():
            L.lora_pool_load(pool, s_, t, int(w.rank[s_]), A, B)
        ws = torch.zeros(L.lora_workspace_bytes(pool, 0, T), dtype=torch.uint8, device=dev)
        sets.append(dict(pool=pool, mem=mem, x=x0.clone(), y=y0.clone(), ids=ids0.clone(), ws=ws))
    torch.cuda.synchronize()

    def step(k):
        s_ = sets[k % n_sets]
        L.lora_apply_multi(s_["pool"], [0, 1, 2], s_["x"], s_["y"], cols, s_["ids"], scales, s_["ws"])

    def step_separate(k):
        s_ = sets[k % n_sets]
        for t in range(n_t):
            L.lora_apply(s_["pool"], t, s_["x"], s_["y"][:, cols[t]:cols[t] + d], s_["ids"], scales, s_["ws"])

    def timed(fn, n):
        g_w, _ = capture_graph(dev, fn, range(args.warmup))
        g, launches = capture_graph(dev, fn, range(n))
        g_w.replay()
        torch.cuda.synchronize()
        sync_ranks(world)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record()
        g.replay()
        ev1.record()
        torch.cuda.synchronize()
        sync_ranks(world)
        return ev0.elapsed_time(ev1) / n, launches, (g, g_w)

    sampler = ClockSampler(dev.index)
    with sampler:
        ms, launches, keep = timed(step, args.steps)
    clocks = sampler.stop()
    ms = reduce_max(ms, world, dev)
    sep_ms, _, keep2 = timed(step_separate, args.steps)
    sep_ms = reduce_max(sep_ms, world, dev)
    del keep, keep2
    for s_ in sets:
        L.lora_pool_destroy(s_["pool"])
    if rank != 0:
        return
    peak, peak_kind = load_peaks()
    # algorithmic bytes: each distinct adapter's A and B on the three targets,
    # x of the adapted rows once (shared), y of the adapted rows read and
    # written on each target
    act = w.ids[w.ids >= 0]
    distinct = np.unique(act)
    alg = int(sum(int(w.rank[a]) * 2 * d * 2 for a in distinct)) * n_t + act.size * d * 2 + n_t * act.size * d * 4
    achieved = alg / (ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": job_value(T, world, ms), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "qkv decode: q_proj batch on 3 targets sharing x, d4096 r16 32 adapters 64 tokens",
                   "global_batch": T * world, "seq_len": 1,
                   "parallelism": "replicas%d" % world if world > 1 else "single", "deltas_per_step": n_t,
                   "l2": "%d rotating buffer sets > 4x L2" % n_sets,
                   "timing": "CUDA graph of the K steps, CUDA events around its replay"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_kind": peak_kind, "traffic": None, "kernel": "decode_kernel<fused>, 3 targets per launch",
                     "kernel_us": ms * 1e3, "algorithmic_bytes_per_launch": alg},
        "separate_launches": {"ms_per_step": sep_ms, "value": job_value(T, world, sep_ms),
                              "note": "the same three deltas as three lora_apply calls"},
        "gpu_launches": launches, "clocks": clocks,
    }
    if world == 1:
        line["cpu_baseline"] = cpu_baseline(w, n_t, args.cpu_seconds)
    print(json.dumps(line), flush=True)


def run_linear(args, rank, world, dev, w, scales, bf16):
    """The q_proj decode batch as a whole projection layer: y = x W^T + each
    row's delta, W a 4096 x 4096 bf16 base weight.  A step is one
    lora_linear call (the shrink launch, then the tensor-core layer kernel
    that streams W and adds the delta inside its accumulator; y written
    once).  Timed in the same run for context: the base product alone
    (torch.matmul, cuBLAS) and the unfused layer (that product, then
    lora_apply adding the delta to y in place)."""
    import torch

    import adapter_deltas_b200 as L
    target = 0
    d_in, d_out = w.targets[target]
    T = w.T
    pool_bytes = L.lora_pool_bytes_required(w.targets, w.r_max, w.n_slots, w.page_bytes)
    set_bytes = pool_bytes + d_out * d_in * 2 + T * (d_in + d_out) * 2
    n_sets = max(2, min(32, -(-4 * L2_BYTES // set_bytes)))
    adapters = {}
    for s_ in range(w.n_slots):
        if w.rank[s_] > 0:
            A, B = w.adapter(s_, target)
            adapters[s_] = (bf16(A), bf16(B))
    W0, x0, ids0 = bf16(w.W(target)), bf16(w.x(target)), torch.from_numpy(w.ids).to(dev)
    sets = []
    for k in range(n_sets):
        mem = torch.empty(pool_bytes, dtype=torch.uint8, device=dev)
        pool = L.lora_pool_create(dev.index, w.targets, w.r_max, w.n_slots, w.page_bytes, mem, w.scatter_seed)
        for s_, (A, B) in adapters.items():
            L.lora_pool_load(pool, s_, target, int(w.rank[s_]), A, B)
        sets.append(dict(pool=pool, mem=mem, W=W0.clone(), x=x0.clone(), ids=ids0.clone(),
                         y=torch.empty(T, d_out, dtype=torch.bfloat16, device=dev),
                         v=torch.zeros(T, w.r_max, dtype=torch.float32, device=dev),
                         ws=torch.zeros(L.lora_linear_workspace_bytes(pool, target, T), dtype=torch.uint8,
                                        device=dev),
                         ws_apply=torch.zeros(L.lora_workspace_bytes(pool, target, T), dtype=torch.uint8,
                                              device=dev)))
    for s_ in sets:   # v of each set, for the layer kernel timed alone
        L.lora_shrink(s_["pool"], target, s_["x"], s_["ids"], s_["v"], s_["ws_apply"])
    torch.cuda.synchronize()

    def step(k):
        s_ = sets[k % n_sets]
        L.lora_linear(s_["pool"], target, s_["x"], s_["W"], s_["y"], s_["ids"], scales, s_["ws"])

    def layer_kernel(k):
        s_ = sets[k % n_sets]
        L.lora_linear_expand(s_["pool"], target, s_["x"], s_["W"], s_["v"], s_["y"], s_["ids"], scales)

    def base_only(k):
        s_ = sets[k % n_sets]
        torch.matmul(s_["x"], s_["W"].t(), out=s_["y"])

    def unfused(k):
        s_ = sets[k % n_sets]
        torch.matmul(s_["x"], s_["W"].t(), out=s_["y"])
        L.lora_apply(s_["pool"], target, s_["x"], s_["y"], s_["ids"], scales, s_["ws_apply"])

    def timed(fn, n):
        g_w, _ = capture_graph(dev, fn, range(args.warmup))
        g, launches = capture_graph(dev, fn, range(n))
        g_w.replay()
        torch.cuda.synchronize()
        sync_ranks(world)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record()
        g.replay()
        ev1.record()
        torch.cuda.synchronize()
        sync_ranks(world)
        del g, g_w
        return reduce_max(ev0.elapsed_time(ev1) / n, world, dev), launches

    # cuBLAS creates its handle on first use, which a graph capture refuses
    side = torch.cuda.Stream(dev)
    with torch.cuda.stream(side):
        unfused(0)
    torch.cuda.synchronize()

    sampler = ClockSampler(dev.index)
    with sampler:
        ms, launches = timed(step, args.steps)
    clocks = sampler.stop()
    reps = max(args.steps, 3 * n_sets)
    kernel_ms, _ = timed(layer_kernel, reps)
    base_ms, _ = timed(base_only, reps)
    unfused_ms, _ = timed(unfused, args.steps)

    # end to end through the C ABI: x and ids in from one packed pinned
    # buffer, y out, every step (W and the adapters stay resident)
    parts = [ids0.cpu().view(torch.uint8), x0.cpu().view(torch.uint8).reshape(-1)]
    offs, total = [], 0
    for t_ in parts:
        offs.append(total)
        total += -(-t_.numel() // 256) * 256
    packed_h = torch.zeros(total, dtype=torch.uint8).pin_memory()
    for o, t_ in zip(offs, parts):
        packed_h[o:o + t_.numel()] = t_
    yout = torch.empty(T, d_out, dtype=torch.bfloat16).pin_memory()
    packed_d = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(n_sets)]

    def e2e_step(k):
        s_ = sets[k % n_sets]
        buf = packed_d[k % n_sets]
        buf.copy_(packed_h, non_blocking=True)
        ids = buf[offs[0]:offs[0] + T * 4].view(torch.int32)
        x = buf[offs[1]:offs[1] + T * d_in * 2].view(torch.bfloat16).view(T, d_in)
        L.lora_linear(s_["pool"], target, x, s_["W"], s_["y"], ids, scales, s_["ws"])
        yout.copy_(s_["y"], non_blocking=True)

    e2e_ms, _ = timed(e2e_step, args.steps)
    for s_ in sets:
        L.lora_pool_destroy(s_["pool"])
    if rank != 0:
        return
    peak, peak_kind = load_peaks()
    act = w.ids[w.ids >= 0]
    distinct = np.unique(act)
    # the layer kernel: W, x, y written once, B of each distinct adapter and
    # v of the adapted rows; the whole step adds each adapter's A, x again
    # for the shrink and v written
    w_bytes = d_out * d_in * 2
    b_bytes = int(sum(int(w.rank[a]) * d_out * 2 for a in distinct))
    a_bytes = int(sum(int(w.rank[a]) * d_in * 2 for a in distinct))
    v_bytes = int(sum(int(w.rank[a]) * 4 for a in act))
    alg_kernel = w_bytes + T * d_in * 2 + T * d_out * 2 + b_bytes + v_bytes
    alg_step = alg_kernel + a_bytes + act.size * d_in * 2 + v_bytes
    achieved = alg_kernel / (kernel_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": job_value(T, world, ms), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": LINEAR_WORKLOAD, "global_batch": T * world, "seq_len": 1,
                   "parallelism": "replicas%d" % world if world > 1 else "single",
                   "l2": "%d rotating buffer sets (own W, pool, x, y), %.0f MB > 4x L2" % (
                       n_sets, n_sets * set_bytes / 1e6),
                   "timing": "CUDA graph of the K steps, CUDA events around its replay"},
        "hbm_gbs_step": alg_step / (ms * 1e-3) / 1e9,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_kind": peak_kind, "traffic": traffic_from_profile("linear_kernel", "linear.cu", "linear"),
                     "traffic_note": "DRAM bytes of one launch from the ncu summary in profiles/, while its "
                                     "source hash matches",
                     "kernel": "linear_kernel (tcgen05: W streamed by TMA, delta in the accumulator), "
                               "timed alone on a precomputed v",
                     "kernel_us": kernel_ms * 1e3, "algorithmic_bytes_per_launch": alg_kernel},
        "base_gemm_only": {"ms_per_step": base_ms, "note": "torch.matmul (cuBLAS) of x W^T alone, no delta"},
        "unfused_layer": {"ms_per_step": unfused_ms, "value": job_value(T, world, unfused_ms),
                          "note": "torch.matmul (cuBLAS) then lora_apply adding the delta to y in place"},
        "e2e": {"value": job_value(T, world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": total,
                "d2h_bytes_per_step": T * d_out * 2},
        "gpu_launches": launches, "clocks": clocks,
    }
    if world == 1:
        line["cpu_baseline"] = cpu_baseline(w, 1, args.cpu_seconds, layer=True)
    print(json.dumps(line), flush=True)


def moe_workload(seed: int):
    """The routed workload: a synth pool of n_ad * E slots (adapter a's
    matrices for expert e in slot a * E + e), each token's adapter uniform
    over the adapters (10 % none) and top_k distinct experts per token."""
    import synth
    m = MOE_SHAPE
    w = synth.custom(seed, m["T"], [(m["d"], m["d"])], [m["r"]] * (m["n_ad"] * m["E"]), m["r"])
    g = np.random.default_rng(seed + 1)
    lora = g.integers(0, m["n_ad"], size=m["T"]).astype(np.int32)
    lora[g.permutation(m["T"])[:round(0.1 * m["T"])]] = -1
    topk = np.stack([g.permutation(m["E"])[:m["k"]] for _ in range(m["T"])]).astype(np.int32)
    y = synth.normal_bf16(np.random.default_rng(seed + 2), (m["T"] * m["k"], m["d"]), 1.0)
    return w, lora, topk, y


def run_moe(args, rank, world, dev, bf16):
    """The delta inside expert routing: one lora_apply_moe per step over the
    256 (token, expert) pairs of 64 tokens routed to 4 of 32 experts, each
    pair taking its own (adapter, expert) slot (one launch: the pairs' slots
    are formed and grouped inside the delta kernel)."""
    import torch

    import adapter_deltas_b200 as L
    m = MOE_SHAPE
    w, lora, topk, y_np = moe_workload(4000 + rank)
    T, k, E, d = m["T"], m["k"], m["E"], m["d"]
    pool_bytes = L.lora_pool_bytes_required(w.targets, w.r_max, w.n_slots, 0)
    set_bytes = pool_bytes + (T * d + T * k * d) * 2
    n_sets = max(2, min(32, -(-4 * L2_BYTES // set_bytes)))
    w.prefetch(range(w.n_slots), [0])
    adapters = {s_: tuple(bf16(t) for t in w.adapter(s_, 0)) for s_ in range(w.n_slots)}
    sc_np = (w.alpha / w.rank).astype(np.float32)
    scales = torch.from_numpy(sc_np).to(dev)
    x0, y0 = bf16(w.x(0)), bf16(y_np)
    lo0, tk0 = torch.from_numpy(lora).to(dev), torch.from_numpy(topk).to(dev)
    sets = []
    for _ in range(n_sets):
        mem = torch.empty(pool_bytes, dtype=torch.uint8, device=dev)
        pool = L.lora_pool_create(dev.index, w.targets, w.r_max, w.n_slots, 0, mem, 0)
        for s_, (A, B) in adapters.items():
            L.lora_pool_load(pool, s_, 0, int(w.rank[s_]), A, B)
        sets.append(dict(pool=pool, mem=mem, x=x0.clone(), y=y0.clone(), lo=lo0.clone(), tk=tk0.clone(),
                         ws=torch.zeros(max(256, L.lora_moe_workspace_bytes(pool, 0, T * k)), dtype=torch.uint8,
                                        device=dev)))
    torch.cuda.synchronize()

    def step(i):
        s_ = sets[i % n_sets]
        L.lora_apply_moe(s_["pool"], 0, s_["x"], s_["y"], s_["lo"], s_["tk"], E, scales, s_["ws"])

    def timed(fn, n):
        g_w, _ = capture_graph(dev, fn, range(args.warmup))
        g, launches = capture_graph(dev, fn, range(n))
        g_w.replay()
        torch.cuda.synchronize()
        sync_ranks(world)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record()
        g.replay()
        ev1.record()
        torch.cuda.synchronize()
        sync_ranks(world)
        del g, g_w
        return reduce_max(ev0.elapsed_time(ev1) / n, world, dev), launches

    sampler = ClockSampler(dev.index)
    with sampler:
        ms, launches = timed(step, args.steps)
    clocks = sampler.stop()

    # end to end: x, adapter ids and routing in from one packed pinned buffer,
    # the pairs' output rows in and out, every step
    parts = [lo0.cpu().view(torch.uint8), tk0.cpu().view(torch.uint8).reshape(-1),
             x0.cpu().view(torch.uint8).reshape(-1), y0.cpu().view(torch.uint8).reshape(-1)]
    offs, total = [], 0
    for t_ in parts:
        offs.append(total)
        total += -(-t_.numel() // 256) * 256
    packed_h = torch.zeros(total, dtype=torch.uint8).pin_memory()
    for o, t_ in zip(offs, parts):
        packed_h[o:o + t_.numel()] = t_
    yout = torch.empty(T * k, d, dtype=torch.bfloat16).pin_memory()
    packed_d = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(n_sets)]

    def e2e_step(i):
        s_ = sets[i % n_sets]
        buf = packed_d[i % n_sets]
        buf.copy_(packed_h, non_blocking=True)
        lo = buf[offs[0]:offs[0] + T * 4].view(torch.int32)
        tk = buf[offs[1]:offs[1] + T * k * 4].view(torch.int32).view(T, k)
        x = buf[offs[2]:offs[2] + T * d * 2].view(torch.bfloat16).view(T, d)
        y = buf[offs[3]:offs[3] + T * k * d * 2].view(torch.bfloat16).view(T * k, d)
        L.lora_apply_moe(s_["pool"], 0, x, y, lo, tk, E, scales, s_["ws"])
        yout.copy_(y, non_blocking=True)

    e2e_ms, _ = timed(e2e_step, args.steps)
    for s_ in sets:
        L.lora_pool_destroy(s_["pool"])
    if rank != 0:
        return
    peak, peak_kind = load_peaks()
    import oracle
    slots = oracle.moe_pair_slots(lora, topk, E, w.n_slots)
    act = slots[slots >= 0]
    distinct = np.unique(act)
    # each distinct slot's A and B, the adapted tokens' x once, the adapted
    # pairs' y read and written
    alg = (int(sum(int(w.rank[s_]) * 2 * d * 2 for s_ in distinct)) + int((lora >= 0).sum()) * d * 2
           + act.size * d * 4)
    achieved = alg / (ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": job_value(T, world, ms), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": MOE_WORKLOAD, "global_batch": T * world, "seq_len": 1,
                   "parallelism": "replicas%d" % world if world > 1 else "single",
                   "pairs": T * k, "slots_in_batch": int(distinct.size),
                   "l2": "%d rotating buffer sets, %.0f MB > 4x L2" % (n_sets, n_sets * set_bytes / 1e6),
                   "timing": "CUDA graph of the K steps, CUDA events around its replay"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_kind": peak_kind, "traffic": traffic_from_profile("decode_kernel", "decode.cu", "moe"),
                     "traffic_note": "DRAM bytes of one launch from the ncu summary in profiles/, while its "
                                     "source hash matches",
                     "kernel": "decode_kernel<fused> forming and grouping the pairs' slots in-kernel (the whole step)",
                     "kernel_us": ms * 1e3, "algorithmic_bytes_per_launch": alg},
        "e2e": {"value": job_value(T, world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": total,
                "d2h_bytes_per_step": T * k * d * 2},
        "gpu_launches": launches, "clocks": clocks,
    }
    if world == 1:
        line["cpu_baseline"] = moe_cpu_baseline(args.cpu_seconds)
    print(json.dumps(line), flush=True)


def moe_cpu_baseline(seconds: float, max_calls: int = 1 << 30):
    """The oracle's routed-pair delta on the host cores, whole batches."""
    import oracle
    m = MOE_SHAPE
    w, lora, topk, y = moe_workload(4000)
    slots = oracle.moe_pair_slots(lora, topk, m["E"], w.n_slots)
    adapters = {int(s_): w.adapter(int(s_), 0) for s_ in np.unique(slots[slots >= 0])}
    threads = min(cpu_threads(), m["T"] * m["k"])
    x = w.x(0)
    n, t0 = 0, time.perf_counter()
    while True:
        oracle.moe_lora_apply(x, y, lora, topk, m["E"], w.n_slots, adapters, w.alpha, threads=threads)
        n += 1
        el = time.perf_counter() - t0
        if (seconds > 0 and el >= seconds) or n >= max_calls:
            break
    return {"value": n * m["T"] / el, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": "%d whole batches of %d tokens (%d pairs) (%.1f s)" % (n, m["T"], m["T"] * m["k"], el)}


def run_swapin(args, rank, world, dev, bf16):
    """Adapter swap-in at the paged workload's geometry: one rank-16 adapter on
    the q/k/v/o of 32 layers (128 targets of 4096 x 4096, 32 MiB) from pinned
    host memory into 1 MiB pages, K swaps per measurement.  Reported against a
    plain pinned host-to-device copy of the same bytes timed in the same run
    (the link's measured rate), and against q_proj-shaped decode steps on
    other slots run alone and beside the swap-ins on a second stream."""
    import torch

    import adapter_deltas_b200 as L
    import synth
    d, n_t, r, n_swap, n_res = 4096, 128, 16, 8, 4
    ids = synth.config(2).ids % n_res + n_swap      # decode batch over the resident slots
    w = synth.custom(3000 + rank, len(ids), [(d, d)] * n_t, [r] * (n_swap + n_res), r, ids=ids,
                     page_bytes=1 << 20, scatter_seed=5)
    pool_bytes = L.lora_pool_bytes_required(w.targets, w.r_max, w.n_slots, w.page_bytes)
    mem = torch.zeros(pool_bytes, dtype=torch.uint8, device=dev)
    pool = L.lora_pool_create(dev.index, w.targets, w.r_max, w.n_slots, w.page_bytes, mem, w.scatter_seed)
    ranks = [r] * n_t
    # one packed adapter (slot 0's weights) in pinned memory
    parts = []
    for t in range(n_t):
        A, B = w.adapter(0, t)
        parts += [np.ascontiguousarray(A).ravel(), np.ascontiguousarray(B).ravel()]
    flat = np.concatenate(parts)
    src = torch.empty(flat.size * 2, dtype=torch.uint8).pin_memory()
    src.numpy()[:] = flat.view(np.uint8)
    nbytes = src.numel()
    staging = torch.empty(L.lora_swap_staging_bytes(pool, ranks), dtype=torch.uint8, device=dev)
    plain_dst = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    for s_ in range(n_swap, n_swap + n_res):           # resident slots for the decode steps
        L.lora_pool_swap_in(pool, s_, ranks, src, staging)
    torch.cuda.synchronize()
    s_swap, s_dec = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    x = bf16(w.x(0))
    y = bf16(w.y_in(0))
    d_ids = torch.from_numpy(w.ids).to(dev)
    sc = torch.full((w.n_slots,), 2.0, dtype=torch.float32, device=dev)
    ws = torch.zeros(L.lora_workspace_bytes(pool, 0, w.T), dtype=torch.uint8, device=dev)

    def swaps():
        for k in range(n_swap):
            L.lora_pool_swap_in(pool, k, ranks, src, staging, s_swap)

    def plain():
        for k in range(n_swap):
            plain_dst.copy_(src, non_blocking=True)

    def decode_steps(n):
        with torch.cuda.stream(s_dec):
            for k in range(n):
                L.lora_apply(pool, k % 4, x, y, d_ids, sc, ws)

    def timed(stream, fn):
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        with torch.cuda.stream(stream):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    n_dec = 400
    for _ in range(max(1, args.warmup)):
        timed(s_swap, swaps)
        timed(s_swap, plain)
        timed(s_dec, lambda: decode_steps(n_dec))
    launches0 = L.lora_kernel_launches()
    sampler = ClockSampler(dev.index)
    with sampler:
        swap_ms = min(timed(s_swap, swaps) for _ in range(args.steps))
        plain_ms = min(timed(s_swap, plain) for _ in range(args.steps))
        dec_ms = min(timed(s_dec, lambda: decode_steps(n_dec)) for _ in range(args.steps))
        # both at once: decode steps on one stream, swap-ins on the other
        both = []
        for _ in range(args.steps):
            torch.cuda.synchronize()
            e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            e[0].record(s_dec)
            e[2].record(s_swap)
            decode_steps(n_dec)
            with torch.cuda.stream(s_swap):
                swaps()
            e[1].record(s_dec)
            e[3].record(s_swap)
            torch.cuda.synchronize()
            both.append((e[0].elapsed_time(e[1]), e[2].elapsed_time(e[3])))
    clocks = sampler.stop()
    launches = (L.lora_kernel_launches() - launches0) // max(1, args.steps)
    L.lora_pool_destroy(pool)
    if rank != 0:
        return
    dec_both = min(b[0] for b in both)
    swap_both = min(b[1] for b in both)
    gbs = n_swap * nbytes / (swap_ms * 1e-3) / 1e9
    plain_gbs = n_swap * nbytes / (plain_ms * 1e-3) / 1e9
    line = {
        "metric": "adapter swap-in GB/s, pinned host to paged pool, 1 GPU", "value": gbs, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": swap_ms / n_swap,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "swap-in of one rank-16 adapter on 128 targets of 4096x4096 (%d MiB), 1 MiB pages"
                               % (nbytes >> 20), "swaps_per_measurement": n_swap, "parallelism": "single",
                   "timing": "CUDA events on the swap stream, best of the steps"},
        "roofline": {"bound": "h2d", "achieved": gbs, "peak": plain_gbs, "unit": "GB/s", "frac": gbs / plain_gbs,
                     "peak_kind": "measured in this run: plain pinned host-to-device copy of the same bytes",
                     "traffic": None, "kernel": "copy + swap_in_kernel"},
        "overlap": {"decode_step_us_alone": dec_ms * 1e3 / n_dec, "decode_step_us_beside_swaps": dec_both * 1e3 / n_dec,
                    "swap_ms_alone": swap_ms / n_swap, "swap_ms_beside_decode": swap_both / n_swap,
                    "decode": "q_proj-shaped lora_apply on resident slots, %d steps" % n_dec},
        "gpu_launches": launches, "clocks": clocks,
        "cpu_baseline": {"value": None, "unit": "GB/s", "cores": 0, "kind": "none",
                         "sample": "a host-to-device copy has no CPU oracle; the plain copy is the baseline"},
    }
    print(json.dumps(line), flush=True)


def capture_graph(dev, fn, ks):
    """Capture fn(k) for k in ks into one CUDA graph; also return how many of
    the library's kernels the captured calls launch."""
    import torch

    import adapter_deltas_b200 as L
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    n0 = L.lora_kernel_launches()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for k in ks:
                fn(k)
    torch.cuda.current_stream(dev).wait_stream(s)
    torch.cuda.synchronize(dev)
    return g, L.lora_kernel_launches() - n0


def reduce_max(x: float, world: int, dev=None) -> float:
    """Max of a per-rank value over all ranks (the slowest rank sets the
    step time); dev None reduces a host tensor (gloo)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sync_ranks(world: int) -> None:
    """Barrier of all ranks (no-op on one)."""
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def job_value(tokens_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job tokens/s: every rank's batch, over the slowest rank's time."""
    return tokens_per_rank * world / (ms_max * 1e-3)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--workload", default="paged", choices=sorted(WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--pool", default="full", choices=["full", "active"],
                    help="paged workload: a pool for all 1000 slots, or pages for the active slots only")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        if args.impl == "reference":
            if rank != 0:
                return
        else:
            torch.cuda.set_device(local_rank)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local_rank))
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_b200(args, rank, world, local_rank)
    finally:
        if world > 1 and args.impl != "reference":
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
