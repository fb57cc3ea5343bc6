"""Benchmark of the B200 MLA-absorb tree-verify attention.

One step = one verify call (split kernel + LSE-merge reduce) over the
65k-context workload: 1 request, 64 heads, a 64-node random tree (depth
<= 16), 65,536-token prefix, scattered slots in a 262,144-slot bf16 latent
pool. The call is captured in CUDA graphs with a static workspace and
replayed; L2 is flushed (256 MiB write) before every timed step and the
flush is outside the timed events.

Prints one JSON line (rank 0). ``value`` is KV tokens per second (sum of the
requests' KV lengths per call / device time per call), whole job over all
ranks; ``--gpus N`` runs N independent replicas (the path needs no
collective). ``--impl reference`` times the float64 CPU oracle instead, on a
bounded sample of the same workload.

``--op defrag`` (KV relocation), ``--op split-verify`` (tree block + dense
pass + merge) and ``--op sequence-shard`` (the KV split over the ranks, NCCL
all-gather and stacked merge) print lines of their own on the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import WORKLOADS, generate  # noqa: E402

METRIC = "tree-verify attn µs/call, KV tok/s & HBM GB/s (% roofline) at 65k ctx"
UNIT = "KV tok/s"
WORKLOAD = "long"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def workload_config(wl, extra=None):
    cfg = {
        "workload": "long: 1 request, H=64 heads, T=64 random tree (depth<=16), prefix L=65536, "
                    "q_latent 512 + q_rope 64, c_kv 512 + k_rope 64 bf16, scattered slots in a "
                    "262144-slot page_size=1 pool, scale 192^-0.5",
        "batch": wl.batch, "num_heads": wl.num_heads, "tree_nodes": list(wl.tree_sizes),
        "prefix": list(wl.prefixes), "kv_per_call": wl.total_kv, "pool_slots": wl.pool_slots,
        "kv_layout": wl.layout, "l2": "flushed before every timed step (256 MiB write, outside the events)",
    }
    if extra:
        cfg.update(extra)
    return cfg


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def algorithmic_work(inp, anc):
    """(flops, bytes) the method must do: every visible (row, key) pair costs
    2*(576+512) flops; every KV row, q row and output row moves once."""
    H = inp.q_latent.shape[1]
    visible = 0
    for b in range(len(inp.qo_indptr) - 1):
        q0, q1 = int(inp.qo_indptr[b]), int(inp.qo_indptr[b + 1])
        L = int(inp.kv_indptr[b + 1] - inp.kv_indptr[b]) - (q1 - q0)
        visible += sum(L + bin(int(a)).count("1") for a in anc[q0:q1])
    rows = inp.q_latent.shape[0] * H
    total_kv = int(inp.kv_indptr[-1])
    flops = 2.0 * H * visible * (576 + 512)
    nbytes = total_kv * 1152 + rows * 1152 + rows * 1024 + total_kv * 4
    return flops, nbytes


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled while the timed loop runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            lines = open(self.path).read().strip().splitlines()
        except OSError:
            lines = []
        for line in lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if self.path:
            os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def cpu_baseline(inp, anc_oracle, budget_s: float = 12.0):
    """Time the float64 oracle on whole query rows of the same workload until
    about `budget_s` seconds of work are done; scale to the full call."""
    import oracle

    H = inp.q_latent.shape[1]
    rows_total = inp.q_latent.shape[0] * H
    cores = len(os.sched_getaffinity(0))
    order = np.random.default_rng(0).permutation(rows_total).astype(np.int64)
    chunk = max(cores, 1)
    done, t0 = 0, time.perf_counter()
    while done < rows_total:
        oracle.verify_rows(inp, anc_oracle, rows=order[done:done + chunk], threads=cores)
        done += chunk
        spent = time.perf_counter() - t0
        left = budget_s - spent
        if left <= 0:
            break
        # next chunk: what fits in the remaining budget at the rate seen so far
        fit = int(left / (spent / done))
        if fit < cores:
            break
        chunk = min(max(cores, (fit // cores) * cores), rows_total - done)
    elapsed = time.perf_counter() - t0
    full_call_s = elapsed * rows_total / done
    value = int(inp.kv_indptr[-1]) / full_call_s
    return {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{done} of {rows_total} (token, head) query rows of the {WORKLOAD} workload, each over its "
                      f"full 65.6k-key visible set, float64 C oracle with OpenMP; {elapsed:.1f} s scaled to the "
                      f"full call by rows"}


def run_reference(args):
    """The reference arm: the CPU oracle as it stands, rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle

    wl = WORKLOADS[WORKLOAD]
    inp = generate(wl)
    anc = oracle.ancestor_masks(inp.parents, inp.qo_indptr)
    H = inp.q_latent.shape[1]
    rows_total = inp.q_latent.shape[0] * H
    cores = len(os.sched_getaffinity(0))
    rows_per_step = max(cores, 8)
    order = np.random.default_rng(1).permutation(rows_total).astype(np.int64)
    pos = 0

    def step():
        nonlocal pos
        sel = order[pos:pos + rows_per_step]
        if sel.shape[0] < rows_per_step:
            pos = 0
            sel = order[:rows_per_step]
        pos += rows_per_step
        oracle.verify_rows(inp, anc, rows=sel, threads=cores)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    elapsed = time.perf_counter() - t0
    per_call = elapsed / args.steps * rows_total / rows_per_step
    value = wl.total_kv / per_call
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, {"step": f"{rows_per_step} query rows of {rows_total} per step",
                                        "l2": "not applicable (float64 oracle on the host cores)"}),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{rows_per_step} of {rows_total} query rows per step, scaled by rows"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_gpu(args):
    import torch

    import mla_speculative_verify_absorb_b200 as va
    from workloads import device as wdev

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    wl = WORKLOADS[WORKLOAD]
    inp = generate(wl)
    anc = np.concatenate([va.verify_attn_build_tree_mask(inp.parents[int(inp.qo_indptr[b]):int(inp.qo_indptr[b + 1])])
                          for b in range(wl.batch)])
    flops, nbytes = algorithmic_work(inp, anc)
    peaks, peak_kind = load_peaks()

    attn = va.VerifyAttention(max_batch=wl.batch, num_heads=wl.num_heads, max_tree=max(wl.tree_sizes),
                              max_kv_per_req=max(wl.kv_lens), max_total_kv=wl.total_kv, pool_slots=wl.pool_slots,
                              sm_scale=wl.sm_scale)
    d = wdev.to_device(inp, anc)
    vargs = attn.make_args(*wdev.positional(d), lse=d["lse"], visible_count=d["visible_count"])
    stream = torch.cuda.Stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    # Warm the kernels eagerly once, then capture the call's three kernels
    # (KV gather, split, reduce) as three graphs, so that each one's time is
    # taken with events between them.
    with torch.cuda.stream(stream):
        attn.run(vargs, stream.cuda_stream)
        attn.reduce(vargs, stream.cuda_stream)
    stream.synchronize()
    # The call as a serving loop replays it: one graph with the three kernels.
    g_call = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_call, stream=stream):
        attn.run(vargs, stream.cuda_stream)
        attn.reduce(vargs, stream.cuda_stream)
    g_gat, g_spl, g_red = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_gat, stream=stream):
        attn.gather(vargs, stream.cuda_stream)
    with torch.cuda.graph(g_spl, stream=stream):
        attn.split(vargs, stream.cuda_stream)
    with torch.cuda.graph(g_red, stream=stream):
        attn.reduce(vargs, stream.cuda_stream)
    code, bits = attn.status(stream.cuda_stream)
    if code != 0:
        raise RuntimeError(f"device status {code} ({bits:#x}) after warm-up")

    def step(ev):
        """One timed call: the whole-call graph between two events."""
        with torch.cuda.stream(stream):
            flush.zero_()
            if ev is not None:
                ev[0].record(stream)
            g_call.replay()
            if ev is not None:
                ev[1].record(stream)

    def step_parts(ev):
        """The same call as three graphs with events between the kernels."""
        with torch.cuda.stream(stream):
            flush.zero_()
            ev[0].record(stream)
            g_gat.replay()
            ev[1].record(stream)
            g_spl.replay()
            ev[2].record(stream)
            g_red.replay()
            ev[3].record(stream)

    for _ in range(args.warmup):
        step(None)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    part_events = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    visible = os.environ.get("CUDA_VISIBLE_DEVICES")
    gpu_index = int(visible.split(",")[local_rank]) if visible and visible.split(",")[0].isdigit() else local_rank
    with ClockSampler(gpu_index) as clocks:
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        for i in range(args.steps):
            step(events[i])
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
    clock_info = clocks.summary()
    # Per-kernel times (the roofline's split kernel alone), a second pass of
    # the same length after the timed one.
    for i in range(args.steps):
        step_parts(part_events[i])
    torch.cuda.synchronize()
    code, bits = attn.status(stream.cuda_stream)
    if code != 0:
        raise RuntimeError(f"device status {code} ({bits:#x}) after timing")
    call_ms = [e[0].elapsed_time(e[1]) for e in events]
    gather_ms = [e[0].elapsed_time(e[1]) for e in part_events]
    split_ms = [e[1].elapsed_time(e[2]) for e in part_events]
    reduce_ms = [e[2].elapsed_time(e[3]) for e in part_events]
    t_call = statistics.mean(call_ms) * 1e-3
    t_gather = statistics.mean(gather_ms) * 1e-3
    t_split = statistics.mean(split_ms) * 1e-3
    t_reduce = statistics.mean(reduce_ms) * 1e-3

    # End to end through the public call with host buffers: per step, copy
    # this call's inputs (queries, slot list, indptrs, tree masks) from pinned
    # host memory, run, and read the output and LSE back. The latent KV pool
    # is the device-resident KV cache and is not copied.
    host = {k: d[k].cpu().pin_memory() for k in ("q_latent", "q_rope", "kv_indices", "kv_indptr", "qo_indptr",
                                                   "tree_anc")}
    out_h = torch.empty_like(d["out"], device="cpu").pin_memory()
    lse_h = torch.empty_like(d["lse"], device="cpu").pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h.numel() * out_h.element_size() + lse_h.numel() * lse_h.element_size()
    e2e_steps = max(1, min(args.steps, 200))

    def e2e_step():
        with torch.cuda.stream(stream):
            for k, t in host.items():
                d[k].copy_(t, non_blocking=True)
            attn(*wdev.positional(d), lse=d["lse"], visible_count=d["visible_count"], stream=stream.cuda_stream)
            out_h.copy_(d["out"], non_blocking=True)
            lse_h.copy_(d["lse"], non_blocking=True)

    for _ in range(3):
        e2e_step()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    t_e2e = e0.elapsed_time(e1) * 1e-3 / e2e_steps

    t_call, t_gather, t_split, t_reduce, t_e2e = max_over_ranks([t_call, t_gather, t_split, t_reduce, t_e2e], dist,
                                                                "cuda")

    kv = wl.total_kv
    tflops_split = flops / t_split / 1e12
    t_roof = max(nbytes / (peaks["hbm_gbs"] * 1e9), flops / (peaks["bf16_tflops"] * 1e12))
    traffic = split_traffic()

    result = {
        "metric": METRIC, "value": kv * world / t_call, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_call * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(wl, {"parallelism": f"{world} independent replicas" if world > 1 else "1 GPU",
                                       "graph": "the call (gather, split, reduce) replayed from one CUDA graph"}),
        "detail": {
            "us_per_call": t_call * 1e6, "gather_us": t_gather * 1e6, "split_us": t_split * 1e6,
            "reduce_us": t_reduce * 1e6,
            "timing": "value from one graph per call (gather, split, reduce); per-kernel times from a second pass "
                      "of three graphs with events between them",
            "kv_tok_per_s_per_gpu": kv / t_call,
            "hbm_gbs_algorithmic": nbytes / t_call / 1e9,
            "tflops_split": tflops_split,
            "roofline_us": t_roof * 1e6, "roofline_frac_call": t_roof / t_call,
            "split_frac_of_sustained_bf16": tflops_split / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]),
            "algorithmic_flops": flops, "algorithmic_bytes": nbytes,
            "peaks": {k: v for k, v in peaks.items()}, "peaks_kind": peak_kind,
        },
        "roofline": {"bound": "tensor", "achieved": tflops_split, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": tflops_split / peaks["bf16_tflops"], "traffic": traffic,
                     "kernel": "verify_split_kernel",
                     "peak_kind": f"{peak_kind} burst bf16 (cuBLAS), kernel timed alone"},
        "clocks": clock_info,
        "e2e": {"value": kv * world / t_e2e, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": 3 * args.steps,   # gather + split + reduce per call
    }
    if rank == 0 and not args.no_cpu_baseline:
        import oracle

        result["cpu_baseline"] = cpu_baseline(inp, oracle.ancestor_masks(inp.parents, inp.qo_indptr))
    if dist is not None:
        dist.barrier()
        del g_call, g_gat, g_spl, g_red
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


DEFRAG_METRIC = "KV relocation (Tier 1 defragmentation) GB/s at 65k ctx"
DEFRAG_SOURCES = ("verify_defrag.cu", "verify_defrag.h", "verify_attn_internal.h")
DEFRAG_TRAFFIC_FILE = os.path.join(ROOT, "profiles", "defrag_kernel_long_traffic.txt")


def run_defrag(args):
    """``--op defrag``: time the KV relocation kernel on the long workload's
    slot list. Every step moves all 65,600 positions of the request between
    two free runs appended to the pool (ping-pong, so each step copies every
    row); the algorithmic bytes are one read and one write of each 1152-byte
    latent row plus 8 bytes of index traffic per position."""
    import torch

    import mla_speculative_verify_absorb_b200 as va

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    wl = WORKLOADS[WORKLOAD]
    inp = generate(wl)
    P, N, B = wl.pool_slots, wl.total_kv, wl.batch
    pool = torch.empty((P + 2 * N, 576), dtype=torch.bfloat16, device="cuda")
    pool[:P].copy_(torch.from_numpy(inp.kv_pool.view(np.int16)).view(torch.bfloat16))
    idx = torch.from_numpy(inp.kv_indices.astype(np.int32)).cuda()
    indptr = torch.from_numpy(inp.kv_indptr.astype(np.int32)).cuda()
    lens = np.diff(inp.kv_indptr)
    runs = [torch.from_numpy((base + np.concatenate([[0], np.cumsum(lens)[:-1]])).astype(np.int32)).cuda()
            for base in (P, P + N)]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()
    nbytes = N * 576 * 2 * 2 + N * 8 + (B + 1) * 4 + B * 4
    budget = int(lens.max())

    for i in range(args.warmup):
        with torch.cuda.stream(stream):
            va.defrag(pool, idx, indptr, runs[i & 1], budget, status=status, stream=stream.cuda_stream)
    stream.synchronize()
    # One graph per direction, so the timed region holds device work only.
    graphs = [torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()]
    for k in range(2):
        with torch.cuda.graph(graphs[k], stream=stream):
            va.defrag(pool, idx, indptr, runs[k], budget, status=status, stream=stream.cuda_stream)

    def step(i, ev):
        with torch.cuda.stream(stream):
            flush.zero_()
            ev[0].record(stream)
            graphs[i & 1].replay()
            ev[1].record(stream)

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    visible = os.environ.get("CUDA_VISIBLE_DEVICES")
    gpu_index = int(visible.split(",")[local_rank]) if visible and visible.split(",")[0].isdigit() else local_rank
    with ClockSampler(gpu_index) as clocks:
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        for i in range(args.steps):
            step(args.warmup + i, events[i])
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
    clock_info = clocks.summary()
    t = statistics.mean(e[0].elapsed_time(e[1]) for e in events) * 1e-3
    if int(status.item()) != 0:
        raise RuntimeError(f"relocation status {int(status.item()):#x}")
    # The last step left every position in one of the two runs, in order.
    last = runs[(args.warmup + args.steps - 1) & 1].item() if B == 1 else None
    if last is not None and not torch.equal(idx.cpu(), torch.arange(last, last + N, dtype=torch.int32)):
        raise RuntimeError("relocated indices are not the destination run")

    # End to end: the slot list comes from pinned host memory and the
    # rewritten one goes back; the pool is the device-resident KV cache.
    idx_h = idx.cpu().pin_memory()
    e2e_steps = max(1, min(args.steps, 200))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def e2e_step(i):
        with torch.cuda.stream(stream):
            idx.copy_(idx_h, non_blocking=True)
            va.defrag(pool, idx, indptr, runs[i & 1], budget, status=status, stream=stream.cuda_stream)
            idx_h.copy_(idx, non_blocking=True)

    base = args.warmup + args.steps
    for i in range(3):
        e2e_step(base + i)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(e2e_steps):
        e2e_step(base + 3 + i)
    e1.record(stream)
    torch.cuda.synchronize()
    t_e2e = e0.elapsed_time(e1) * 1e-3 / e2e_steps
    t, t_e2e = max_over_ranks([t, t_e2e], dist, "cuda")

    peaks, peak_kind = load_peaks()
    achieved = nbytes / t / 1e9
    result = {
        "metric": DEFRAG_METRIC, "value": nbytes * world / t / 1e9, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "op": "defrag",
        "config": workload_config(wl, {"moved_positions": N, "budget": budget,
                                       "step": "every position moves between two free runs appended to the pool",
                                       "graph": "the relocation launch replayed from a CUDA graph",
                                       "parallelism": f"{world} independent replicas" if world > 1 else "1 GPU"}),
        "detail": {"us_per_call": t * 1e6, "algorithmic_bytes": nbytes, "roofline_us": nbytes / (peaks["hbm_gbs"] * 1e9) * 1e6,
                   "peaks_kind": peak_kind},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"],
                     "traffic": source_traffic(DEFRAG_TRAFFIC_FILE, DEFRAG_SOURCES),
                     "kernel": "verify_defrag_kernel", "peak_kind": f"{peak_kind} HBM copy"},
        "clocks": clock_info,
        "e2e": {"value": nbytes * world / t_e2e / 1e9, "unit": "GB/s", "h2d_bytes_per_step": N * 4,
                "d2h_bytes_per_step": N * 4},
        "gpu_launches": args.steps,
    }
    if rank == 0 and not args.no_cpu_baseline:
        import oracle.defrag as odf

        host_pool = pool.view(torch.int16).cpu().numpy().view(np.uint16)
        host_idx = inp.kv_indices.astype(np.int32)
        dst = (P + np.concatenate([[0], np.cumsum(lens)[:-1]])).astype(np.int32)
        cores = 1
        t0 = time.perf_counter()
        odf.defrag(host_pool, host_idx, inp.kv_indptr, dst, budget)
        el = time.perf_counter() - t0
        result["cpu_baseline"] = {"value": nbytes / el / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
                                  "sample": f"the whole relocation of the {N} positions once ({el:.2f} s, "
                                            "numpy oracle, pool copies included)"}
    if dist is not None:
        dist.barrier()
        del graphs
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


SV_METRIC = METRIC + " — split-verify variant"


def run_split_verify(args):
    """``--op split-verify``: time the split-verify composition (tree block,
    dense pass, LSE merge) on the long workload, as one graph per call, and
    each of its kernels from a second pass of per-kernel graphs."""
    import torch

    import mla_speculative_verify_absorb_b200 as va
    from workloads import device as wdev

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    wl = WORKLOADS[WORKLOAD]
    inp = generate(wl)
    anc = np.concatenate([va.verify_attn_build_tree_mask(inp.parents[int(inp.qo_indptr[b]):int(inp.qo_indptr[b + 1])])
                          for b in range(wl.batch)])
    flops, nbytes = algorithmic_work(inp, anc)
    self_only = np.concatenate([np.uint64(1) << np.arange(int(t), dtype=np.uint64) for t in wl.tree_sizes])
    dense_flops, _ = algorithmic_work(inp, self_only)
    peaks, peak_kind = load_peaks()
    attn = va.VerifyAttention(max_batch=wl.batch, num_heads=wl.num_heads, max_tree=max(wl.tree_sizes),
                              max_kv_per_req=max(wl.kv_lens), max_total_kv=wl.total_kv, pool_slots=wl.pool_slots,
                              sm_scale=wl.sm_scale)
    d = wdev.to_device(inp, anc)
    stream = torch.cuda.Stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    pos = wdev.positional(d)
    with torch.cuda.stream(stream):
        a_d = attn.split_verify(*pos, lse=d["lse"], stream=stream.cuda_stream)   # allocates the scratch once
    stream.synchronize()
    sv = attn._sv
    tokens = inp.q_latent.shape[0]
    a_t = attn.make_args(*pos[:7], d["out"], lse=sv["lse_t"][:tokens])
    g_call, g_tb, g_den, g_spl = (torch.cuda.CUDAGraph() for _ in range(4))
    with torch.cuda.graph(g_call, stream=stream):
        attn.split_verify(*pos, lse=d["lse"], stream=stream.cuda_stream)
    with torch.cuda.graph(g_tb, stream=stream):
        attn.tree_block(a_t, True, sv["self_anc"].data_ptr(), stream.cuda_stream, out_f32_ptr=sv["o_t"].data_ptr())
    with torch.cuda.graph(g_den, stream=stream):
        attn.run(a_d, stream.cuda_stream)
        attn.reduce(a_d, stream.cuda_stream)
    with torch.cuda.graph(g_spl, stream=stream):
        attn.split(a_d, stream.cuda_stream)
    code, bits = attn.status(stream.cuda_stream)
    if code != 0:
        raise RuntimeError(f"device status {code} ({bits:#x}) after warm-up")

    def timed(graph, ev):
        with torch.cuda.stream(stream):
            flush.zero_()
            ev[0].record(stream)
            graph.replay()
            ev[1].record(stream)

    for _ in range(args.warmup):
        with torch.cuda.stream(stream):
            flush.zero_()
            g_call.replay()
    ev = {k: [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
          for k in ("call", "tb", "dense", "split")}
    visible = os.environ.get("CUDA_VISIBLE_DEVICES")
    gpu_index = int(visible.split(",")[local_rank]) if visible and visible.split(",")[0].isdigit() else local_rank
    with ClockSampler(gpu_index) as clocks:
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        for i in range(args.steps):
            timed(g_call, ev["call"][i])
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
    clock_info = clocks.summary()
    for i in range(args.steps):
        timed(g_tb, ev["tb"][i])
        timed(g_den, ev["dense"][i])
        timed(g_spl, ev["split"][i])
    with torch.cuda.stream(stream):
        g_call.replay()   # leave the call's own result in place
    torch.cuda.synchronize()
    code, bits = attn.status(stream.cuda_stream)
    if code != 0:
        raise RuntimeError(f"device status {code} ({bits:#x}) after timing")
    t = {k: statistics.mean(e[0].elapsed_time(e[1]) for e in v) * 1e-3 for k, v in ev.items()}

    # End to end: this call's inputs from pinned host memory, output and LSE back.
    host = {k: d[k].cpu().pin_memory() for k in ("q_latent", "q_rope", "kv_indices", "kv_indptr", "qo_indptr",
                                                   "tree_anc")}
    out_h = torch.empty_like(d["out"], device="cpu").pin_memory()
    lse_h = torch.empty_like(d["lse"], device="cpu").pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in host.values())
    d2h = out_h.numel() * out_h.element_size() + lse_h.numel() * lse_h.element_size()
    e2e_steps = max(1, min(args.steps, 200))

    def e2e_step():
        with torch.cuda.stream(stream):
            for k, x in host.items():
                d[k].copy_(x, non_blocking=True)
            attn.split_verify(*pos, lse=d["lse"], stream=stream.cuda_stream)
            out_h.copy_(d["out"], non_blocking=True)
            lse_h.copy_(d["lse"], non_blocking=True)

    for _ in range(3):
        e2e_step()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    t_e2e = e0.elapsed_time(e1) * 1e-3 / e2e_steps
    keys = ("call", "tb", "dense", "split")
    vals = max_over_ranks([t[k] for k in keys] + [t_e2e], dist, "cuda")
    t = dict(zip(keys, vals[:4]))
    t_e2e = vals[4]

    kv = wl.total_kv
    t_roof = max(nbytes / (peaks["hbm_gbs"] * 1e9), flops / (peaks["bf16_tflops"] * 1e12))
    tflops_split = dense_flops / t["split"] / 1e12
    result = {
        "metric": SV_METRIC, "value": kv * world / t["call"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t["call"] * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "op": "split-verify",
        "config": workload_config(wl, {"parallelism": f"{world} independent replicas" if world > 1 else "1 GPU",
                                       "graph": "the composition (tree block, gather, split, reduce, merge) "
                                                "replayed from one CUDA graph"}),
        "detail": {
            "us_per_call": t["call"] * 1e6, "tree_block_us": t["tb"] * 1e6,
            "dense_pass_us": t["dense"] * 1e6, "split_us": t["split"] * 1e6,
            "merge_us_by_difference": (t["call"] - t["tb"] - t["dense"]) * 1e6,
            "roofline_us": t_roof * 1e6, "roofline_frac_call": t_roof / t["call"],
            "algorithmic_flops": flops, "dense_pass_flops": dense_flops, "algorithmic_bytes": nbytes,
            "peaks_kind": peak_kind,
        },
        "roofline": {"bound": "tensor", "achieved": tflops_split, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": tflops_split / peaks["bf16_tflops"], "traffic": split_traffic(),
                     "kernel": "verify_split_kernel (dense pass: prefix + own key; same kernel and data "
                               "movement as the fused call, only the mask words differ)",
                     "peak_kind": f"{peak_kind} burst bf16 (cuBLAS), kernel timed alone"},
        "clocks": clock_info,
        "e2e": {"value": kv * world / t_e2e, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": 5 * args.steps,   # tree block, gather, split, reduce, merge per call
    }
    if dist is not None:
        dist.barrier()
        del g_call, g_tb, g_den, g_spl
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


SHARD_METRIC = METRIC + " — KV-sequence sharded"


def run_sequence_shard(args):
    """``--op sequence-shard``: the long call with its KV split over the N
    ranks (strong scaling: one request, fixed total work). Each rank attends
    its shard, the states are all-gathered over NCCL and every rank merges
    them; the time is the max over ranks of that whole sequence. With one
    GPU the same line also reports, for R = 2, 4, 8, each shard's pass and
    the stacked merge run one after another on this GPU (what a rank
    computes; the exchange is not part of those figures)."""
    import torch

    import mla_speculative_verify_absorb_b200 as va
    from mla_speculative_verify_absorb_b200.sequence_shard import ShardedVerify
    from workloads import device as wdev

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    wl = WORKLOADS[WORKLOAD]
    inp = generate(wl)
    anc = np.concatenate([va.verify_attn_build_tree_mask(inp.parents[int(inp.qo_indptr[b]):int(inp.qo_indptr[b + 1])])
                          for b in range(wl.batch)])
    flops, nbytes = algorithmic_work(inp, anc)
    peaks, peak_kind = load_peaks()
    d = wdev.to_device(inp, anc)
    T, L, H = int(wl.tree_sizes[0]), int(wl.prefixes[0]), wl.num_heads
    stream = torch.cuda.Stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    s = stream.cuda_stream

    def make(R):
        return ShardedVerify(world=R, num_heads=H, max_tree=T, max_prefix=L, pool_slots=wl.pool_slots,
                             sm_scale=wl.sm_scale)

    def local(sv, r, o, lse):
        return sv.local_state(r, d["q_latent"], d["q_rope"], d["kv_pool"], d["kv_indices"], d["tree_anc"], o, lse, s)

    def timed_graph(g, reps):
        ts = []
        for _ in range(reps):
            e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            with torch.cuda.stream(stream):
                flush.zero_()
                e[0].record(stream)
                g.replay()
                e[1].record(stream)
            ts.append(e)
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in ts) * 1e-3

    sv = make(world)
    if dist is not None:
        with torch.cuda.stream(stream):
            sv(d["q_latent"], d["q_rope"], d["kv_pool"], d["kv_indices"], d["tree_anc"], d["out"], d["lse"],
               stream=s)
    else:
        o_all, lse_all = sv.stacked(T)
        g_call = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            local(sv, 0, o_all[0], lse_all[0])
            sv.merge(o_all, lse_all, d["out"], d["lse"], s)
        stream.synchronize()
        with torch.cuda.graph(g_call, stream=stream):
            local(sv, 0, o_all[0], lse_all[0])
            sv.merge(o_all, lse_all, d["out"], d["lse"], s)

    def call():
        with torch.cuda.stream(stream):
            if dist is None:
                g_call.replay()
            else:
                sv(d["q_latent"], d["q_rope"], d["kv_pool"], d["kv_indices"], d["tree_anc"], d["out"], d["lse"],
                   stream=s)

    for _ in range(args.warmup):
        with torch.cuda.stream(stream):
            flush.zero_()
        call()
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    visible = os.environ.get("CUDA_VISIBLE_DEVICES")
    gpu_index = int(visible.split(",")[local_rank]) if visible and visible.split(",")[0].isdigit() else local_rank
    with ClockSampler(gpu_index) as clocks:
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        for i in range(args.steps):
            with torch.cuda.stream(stream):
                flush.zero_()
                events[i][0].record(stream)
            call()
            with torch.cuda.stream(stream):
                events[i][1].record(stream)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
    clock_info = clocks.summary()
    t_call = statistics.mean(a.elapsed_time(b) for a, b in events) * 1e-3
    code, bits = sv.attn.status(s)
    if code != 0:
        raise RuntimeError(f"device status {code} ({bits:#x})")

    emulated = {}
    if dist is None:
        reps = max(3, min(args.steps, 100))
        for R in (2, 4, 8):
            svR = make(R)
            o_all, lse_all = svR.stacked(T)
            shard_t = []
            for r in range(R):
                with torch.cuda.stream(stream):
                    ok = local(svR, r, o_all[r], lse_all[r])
                stream.synchronize()
                if not ok:
                    raise RuntimeError("every shard of the long call has keys")
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    local(svR, r, o_all[r], lse_all[r])
                shard_t.append(timed_graph(g, reps))
            gm = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                svR.merge(o_all, lse_all, d["out"], d["lse"], s)
            stream.synchronize()
            with torch.cuda.graph(gm, stream=stream):
                svR.merge(o_all, lse_all, d["out"], d["lse"], s)
            t_merge = timed_graph(gm, reps)
            code, bits = svR.attn.status(s)
            if code != 0:
                raise RuntimeError(f"device status {code} ({bits:#x}) at R={R}")
            emulated[str(R)] = {"max_shard_us": max(shard_t) * 1e6, "min_shard_us": min(shard_t) * 1e6,
                                "merge_us": t_merge * 1e6,
                                "exchange_bytes_per_rank_out": T * H * (512 * 2 + 4),
                                "exchange_bytes_per_rank_in": (R - 1) * T * H * (512 * 2 + 4)}
    (t_call,) = max_over_ranks([t_call], dist, "cuda")
    kv = wl.total_kv
    t_roof = max(nbytes / (peaks["hbm_gbs"] * 1e9), flops / (peaks["bf16_tflops"] * 1e12))
    achieved = flops / t_call / 1e12
    result = {
        "metric": SHARD_METRIC, "value": kv / t_call, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_call * 1e3, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "op": "sequence-shard",
        "config": workload_config(wl, {"parallelism": f"KV sequence split over {world} ranks, NCCL all-gather of "
                                                      "(o, lse), stacked LSE merge" if world > 1 else
                                                      "1 GPU (one shard, merge of one state)"}),
        "detail": {"us_per_call": t_call * 1e6, "roofline_us": t_roof * 1e6, "roofline_frac_call": t_roof / t_call,
                   "emulated_ranks_on_one_gpu": emulated, "algorithmic_flops": flops,
                   "algorithmic_bytes": nbytes, "peaks_kind": peak_kind},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops"], "traffic": None,
                     "kernel": "whole sharded call (gather, split, reduce, merge; all-gather when N > 1)",
                     "peak_kind": f"{peak_kind} burst bf16 (cuBLAS)"},
        "clocks": clock_info,
        "gpu_launches": 4 * args.steps,   # gather, split, reduce, merge per call (plus NCCL when N > 1)
    }
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def max_over_ranks(values, dist, device):
    """Element-wise max of a list of floats over all ranks (the job's time)."""
    import torch

    if dist is None:
        return [float(v) for v in values]
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


SPLIT_SOURCES = ("verify_split_sm100.cu", "sm100_ptx.cuh", "verify_attn_internal.h", "verify_split.h")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "split_kernel_long_traffic.txt")


def kernel_digest(sources=SPLIT_SOURCES) -> str:
    """Digest of the sources that define a kernel (default: the split kernel)."""
    import hashlib

    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mla_speculative_verify_absorb_b200", "csrc")
    for name in sources:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def split_traffic():
    """DRAM bytes per split-kernel launch from the committed ncu summary, or
    None when the kernel sources changed since that capture."""
    return source_traffic(TRAFFIC_FILE, SPLIT_SOURCES)


def source_traffic(path, sources):
    """DRAM bytes per launch recorded in `path`, or None when the sources
    changed since that capture."""
    if not os.path.exists(path):
        return None
    fields = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                fields[k.strip()] = v.strip()
    if fields.get("kernel_source_digest") != kernel_digest(sources):
        return None
    return int(fields["dram_bytes_per_launch"])


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--op", choices=["verify", "defrag", "split-verify", "sequence-shard"], default="verify",
                    help="verify: the attention call (default); defrag: the KV relocation kernel; "
                         "split-verify: the variant composed of tree block, dense pass and merge; "
                         "sequence-shard: the call with its KV split over the ranks")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.op != "verify" and args.impl == "reference":
        ap.error(f"--op {args.op} has no reference arm of its own (the oracle arm times --op verify)")
    if args.op == "defrag":
        run_defrag(args)
    elif args.op == "split-verify":
        run_split_verify(args)
    elif args.op == "sequence-shard":
        run_sequence_shard(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
