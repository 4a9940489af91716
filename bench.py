"""LCSA benchmark: ms per call and effective TFLOP/s (kept blocks only).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step is one whole LCSA call (prologue, block selection, block-sparse
attention) on one stream chunk of synthetic inputs already resident in HBM.
The default workload is the 768x1280 stream chunk: 2 query frames of 48x80
tokens, a 6-frame KV window, 12 heads, head_dim 128, 1x8x16 blocks,
local_range 11, sparse_ratio 2.0 (k = 60 blocks).

Timing: W untimed warm-up calls, then exactly K timed calls, each between
its own pair of CUDA events on the launching stream; a 256 MiB buffer is
written before every timed call so each call starts with a cold L2. The
timed region is bracketed by a barrier and a device synchronise; the
reported time is the maximum over ranks. Under torchrun every rank runs its
own independent chunk (weak scaling, no collective on the data path).

--impl reference times the fp64 CPU oracle (the independent checker) on the
host cores instead, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "LCSA ms/call and effective TFLOP/s (selected blocks) at 768×1280 stream chunk"
UNIT = "TFLOP/s"
FLUSH_BYTES = 256 << 20


def _args():
    from block_sparse_video_lcsa_b200 import synth
    ap = argparse.ArgumentParser(description="Time the LCSA call on synthetic inputs; prints one JSON line.")
    ap.add_argument("--gpus", type=int, default=1, help="ranks (one GPU each; N > 1 under torchrun)")
    ap.add_argument("--steps", type=int, default=50, help="timed calls")
    ap.add_argument("--warmup", type=int, default=5, help="untimed calls before them")
    ap.add_argument("--workload", default="stream_768x1280", choices=list(synth.WORKLOADS),
                    help="synthetic workload (default: the 768x1280 stream chunk)")
    ap.add_argument("--impl", default="lcsa", choices=["lcsa", "reference"],
                    help="lcsa: the CUDA library; reference: the fp64 CPU oracle on the host cores")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle sample of the CPU baseline")
    ap.add_argument("--e2e-steps", type=int, default=10,
                    help="calls timed end to end through host buffers (copies included)")
    ap.add_argument("--layers", type=int, default=0,
                    help="time N sequential calls (a DiT chunk's attention layers), eager and as one CUDA graph")
    ap.add_argument("--stream", action="store_true",
                    help="time a stream plan: each step brings the chunk's new frames into the KV ring")
    ap.add_argument("--reuse", action="store_true",
                    help="threshold reuse: calls after the first keep blocks by the recorded thresholds (no top-k)")
    ap.add_argument("--shard-heads", action="store_true",
                    help="one layer's heads split over the ranks: per-token sums of squares all-reduced (NCCL)")
    return ap.parse_args()


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def _code_only(text):
    """C/C++/CUDA source without its comments, whitespace runs collapsed: an
    edit that only touches comments or layout leaves it unchanged."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":  # string or character literal, kept verbatim
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            out.append(" ")
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def _kernel_source_hash(files):
    """sha256 prefix of the kernel's code (comments and layout excluded)."""
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "block_sparse_video_lcsa_b200", "csrc", f), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode("utf-8"))
    return h.hexdigest()[:16]


def _spread(values):
    """p10 / median / p90 of per-call times (linear interpolation between ranks)."""
    xs = sorted(float(x) for x in values)

    def q(f):
        i = f * (len(xs) - 1)
        lo = int(math.floor(i))
        hi = min(lo + 1, len(xs) - 1)
        return xs[lo] + (xs[hi] - xs[lo]) * (i - lo)
    return {"p10": q(0.1), "median": q(0.5), "p90": q(0.9)}


def _launches_per_call(wl):
    """Kernels of ours in one call: prologue, selection, attention; 64-token
    blocks add the pair-union kernel."""
    return 3 + (1 if wl.block_t * wl.block_h * wl.block_w == 64 else 0)


def _profiled_traffic(kernel_tag, files, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source (same hash) and on this workload; else None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    want = _kernel_source_hash(files)
    with open(path) as f:
        for line in f:
            m = re.match(r"\s*(\w+)\s+src=(\w+)\s+workload=(\S+)\s+dram_bytes_per_launch=([0-9.eE+]+)", line)
            if m and m.group(1) == kernel_tag and m.group(2) == want and m.group(3) == workload:
                return float(m.group(4))
    return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu = gpu_id
        self.proc = None
        self.lines = []
        self.thread = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            if self.thread is not None:
                self.thread.join(timeout=2)

    def summary(self):
        if not self.lines:
            return None
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def _max_over_ranks(value, device):
    """The largest `value` over the ranks of the default process group (the
    timing of a multi-GPU run is the slowest rank's)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def _oracle_sample(wl, inp, target_s=12.0):
    """Time the fp64 oracle on a bounded sample: pooled values and selection
    for the whole chunk, attention for a sample of rows; the full-call time is
    extrapolated by the row count."""
    import numpy as np
    import oracle

    og = oracle.Geometry.from_workload(wl)
    threads = oracle.hardware_threads()
    t0 = time.perf_counter()
    pq = oracle.pool(og, inp.q, inp.gamma_q, True)
    pk = oracle.pool(og, inp.k, inp.gamma_k, False)
    sel = oracle.select(og, pq, pk)
    t_pre = time.perf_counter() - t0
    rng = np.random.default_rng(0)
    n = min(og.rows, max(threads, 4))
    rows = np.sort(rng.choice(og.rows, size=n, replace=False)).astype(np.int64)
    t0 = time.perf_counter()
    oracle.attention(og, inp.q, inp.k, inp.v, inp.gamma_q, inp.gamma_k, sel, rows)
    t_probe = time.perf_counter() - t0
    # grow the sample to about target_s of attention work
    n2 = int(min(og.rows, max(n, n * max(1.0, (target_s - t_pre) / max(t_probe, 1e-3)))))
    if n2 > n:
        rows = np.sort(rng.choice(og.rows, size=n2, replace=False)).astype(np.int64)
        t0 = time.perf_counter()
        oracle.attention(og, inp.q, inp.k, inp.v, inp.gamma_q, inp.gamma_k, sel, rows)
        t_attn = time.perf_counter() - t0
    else:
        n2, t_attn = n, t_probe
    full_s = t_pre + t_attn * og.rows / n2
    flops = float(np.minimum(oracle.window_sizes(og), og.topk).sum()) * og.batch * og.heads * 4.0 * og.nb ** 2 * \
        og.head_dim
    return {"value": flops / full_s / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
            "ms_per_call": full_s * 1e3,
            "sample": "fp64 oracle: pooling + selection of the whole chunk (%.2f s), attention of %d of %d rows "
                      "(%.2f s), call time extrapolated by rows" % (t_pre, n2, og.rows, t_attn)}


def run_reference(args):
    world, rank, _ = _dist()
    if rank != 0:
        return 0
    from block_sparse_video_lcsa_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    inp = synth.make_inputs(wl)
    samples = []
    for i in range(args.warmup + args.steps):
        r = _oracle_sample(wl, inp, target_s=2.0)
        if i >= args.warmup:
            samples.append(r)
    ms = statistics.mean(s["ms_per_call"] for s in samples)
    value = statistics.mean(s["value"] for s in samples)
    import numpy as np
    import oracle
    og = oracle.Geometry.from_workload(wl)
    kept = int(np.minimum(oracle.window_sizes(og), og.topk).sum()) * og.batch * og.heads
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "q_tokens": wl.q_tokens, "kv_tokens": wl.kv_tokens,
                       "heads": wl.heads, "head_dim": wl.head_dim,
                       "block": "%dx%dx%d" % (wl.block_t, wl.block_h, wl.block_w), "local_range": wl.local_range,
                       "sparse_ratio": wl.sparse_ratio, "topk": og.topk, "kept_blocks": kept, "selection": "top-k",
                       "parallelism": "rank 0 of %d, host cores" % args.gpus},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": samples[-1]["cores"], "kind": "oracle",
                             "sample": samples[-1]["sample"]},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def run_lcsa(args):
    import torch
    import torch.distributed as dist

    import block_sparse_video_lcsa_b200 as lcsa
    from block_sparse_video_lcsa_b200 import synth

    world, rank, local = _dist()
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = synth.WORKLOADS[args.workload].replace(seed=rank)
    inp = synth.make_inputs(wl)

    def bf(a):
        return torch.from_numpy(a).view(torch.bfloat16).to(dev)

    q, k, v = bf(inp.q), bf(inp.k), bf(inp.v)
    gq, gk = torch.from_numpy(inp.gamma_q).to(dev), torch.from_numpy(inp.gamma_k).to(dev)
    out = torch.empty_like(q)
    plan = lcsa.lcsa_plan_create(lcsa.config_from_workload(wl, host_io=1), local)
    geo = plan.geometry
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    if args.reuse:
        plan.lcsa_plan_set_threshold_reuse(True)

    for _ in range(args.warmup):
        plan.lcsa_forward(q, k, v, gq, gk, out, stream)
    plan.lcsa_check_device_error(stream)

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    try:
        gpu_id = "GPU-%s" % torch.cuda.get_device_properties(dev).uuid
    except Exception:  # noqa: BLE001 - fall back to the index
        gpu_id = str(local)
    with ClockSampler(gpu_id) as clocks:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            starts[i].record(stream)
            plan.lcsa_forward(q, k, v, gq, gk, out, stream)
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
        # per-kernel times: the same calls again with events around each kernel
        # (an event between two kernels costs a few microseconds, so these
        # events stay out of the step timing above)
        plan.lcsa_plan_set_timing(args.steps)
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            plan.lcsa_forward(q, k, v, gq, gk, out, stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    plan.lcsa_check_device_error(stream)
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    kms, kcount = plan.lcsa_get_kernel_times()
    plan.lcsa_plan_set_timing(0)
    kept = plan.lcsa_selection_nnz()  # the blocks the timed calls kept (threshold reuse may differ from k)
    total_ms = _max_over_ranks(sum(step_ms), dev)
    # warm L2: the same calls without the flush between them (context for the
    # flushed figure, which is the reported one)
    warm_starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    warm_ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for i in range(args.steps):
        warm_starts[i].record(stream)
        plan.lcsa_forward(q, k, v, gq, gk, out, stream)
        warm_ends[i].record(stream)
    torch.cuda.synchronize(dev)
    plan.lcsa_check_device_error(stream)
    warm_ms = _max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(warm_starts, warm_ends)), dev) / args.steps

    # end to end: pinned host buffers through lcsa_forward_host (copies inside)
    hq = torch.from_numpy(inp.q).view(torch.bfloat16).pin_memory()
    hk = torch.from_numpy(inp.k).view(torch.bfloat16).pin_memory()
    hv = torch.from_numpy(inp.v).view(torch.bfloat16).pin_memory()
    hgq = torch.from_numpy(inp.gamma_q).pin_memory()
    hgk = torch.from_numpy(inp.gamma_k).pin_memory()
    hout = torch.empty(tuple(q.shape), dtype=torch.bfloat16).pin_memory()
    plan.lcsa_forward_host(hq, hk, hv, hgq, hgk, hout, stream)
    e2e_steps = max(1, args.e2e_steps)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        plan.lcsa_forward_host(hq, hk, hv, hgq, hgk, hout, stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = _max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev)
    if world > 1:
        dist.barrier()
    plan.destroy()

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return 0

    peaks = _peaks()
    flops = geo.selected_flops * kept / geo.nnz
    ms_per_step = total_ms / args.steps
    value = world * flops / (ms_per_step * 1e-3) / 1e12
    k3_tflops = flops / (kms[2] * 1e-3) / 1e12
    k1_gbs = geo.prologue_bytes / (kms[0] * 1e-3) / 1e9
    k3_src = "k3_attention_tc.cu"
    traffic = _profiled_traffic("k3", [k3_src, "lcsa_internal.h"], args.workload)
    roofline = {"bound": "tensor", "kernel": "attention (K3, %s)" % k3_src, "achieved": k3_tflops, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": k3_tflops / peaks["bf16_tflops"], "traffic": traffic,
                "peak_source": peaks["source"] + " burst bf16",
                "algorithmic_flops_per_launch": flops}
    h2d = (inp.q.nbytes + inp.k.nbytes + inp.v.nbytes + inp.gamma_q.nbytes + inp.gamma_k.nbytes)
    d2h = inp.q.nbytes
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "ms_per_step_spread": _spread(step_ms), "warm_l2_ms_per_step": warm_ms,
            "config": {"workload": wl.name, "q_tokens": geo.q_tokens, "kv_tokens": geo.kv_tokens,
                       "heads": wl.heads, "head_dim": wl.head_dim,
                       "block": "%dx%dx%d" % (wl.block_t, wl.block_h, wl.block_w), "local_range": wl.local_range,
                       "sparse_ratio": wl.sparse_ratio, "topk": geo.topk, "kept_blocks": kept,
                       "selection": "threshold reuse (recorded on the warm-up)" if args.reuse else "top-k",
                       "l2": "256 MiB buffer written before every timed call", "parallelism": "replicas%d" % world,
                       "kernel_times": "second pass of the same calls, CUDA events around each kernel"},
            "roofline": roofline,
            "kernels": {"prologue_ms": kms[0], "select_ms": kms[1], "attention_ms": kms[2], "timed_calls": kcount,
                        "prologue_gbs": k1_gbs, "prologue_hbm_frac": k1_gbs / peaks["hbm_gbs"],
                        "prologue_bytes": geo.prologue_bytes, "hbm_peak_gbs": peaks["hbm_gbs"]},
            "e2e": {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": _launches_per_call(wl) * args.steps,
            "clocks": clocks.summary()}
    if world == 1 and not args.no_cpu_baseline:
        cb = _oracle_sample(wl, inp)
        cb.pop("ms_per_call")
        line["cpu_baseline"] = cb
    print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_stream(args):
    """One step = one stream chunk (lcsa_forward_stream): the q_frames new
    frames of q, k and v enter the plan's KV ring; K1 works on the new frames
    only. Frames cycle through a 16-frame sequence resident in HBM (377 MB at
    768x1280, larger than L2), and L2 is flushed before every timed chunk."""
    import torch

    import block_sparse_video_lcsa_b200 as lcsa
    from block_sparse_video_lcsa_b200 import synth

    world, rank, local = _dist()
    if world > 1:
        print(json.dumps({"impl": "lcsa", "unavailable": "--stream times one GPU"}))
        return 0
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = synth.WORKLOADS[args.workload]
    nf = 16
    seq = synth.make_inputs(wl.replace(q_frames=nf, kv_frames=nf))
    plane = wl.grid_h * wl.grid_w

    def bf(a):
        return torch.from_numpy(a).view(torch.bfloat16).to(dev)

    q, k, v = bf(seq.q), bf(seq.k), bf(seq.v)
    gq, gk = torch.from_numpy(seq.gamma_q).to(dev), torch.from_numpy(seq.gamma_k).to(dev)
    plan = lcsa.lcsa_plan_create_stream(lcsa.config_from_workload(wl), local)
    geo = plan.geometry
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    out = torch.empty((wl.batch, wl.q_frames * plane, wl.channels), dtype=torch.bfloat16, device=dev)
    first = wl.kv_frames - wl.q_frames
    plan.lcsa_stream_push(k[:, :first * plane].contiguous(), v[:, :first * plane].contiguous(), gk, first, stream)
    starts_f = list(range(0, nf - wl.q_frames + 1, wl.q_frames))
    chunks = [tuple(t[:, f * plane:(f + wl.q_frames) * plane].contiguous() for t in (q, k, v)) for f in starts_f]

    def chunk(i):
        cq, ck, cv = chunks[i % len(chunks)]
        plan.lcsa_forward_stream(cq, ck, cv, gq, gk, out, stream)

    for i in range(args.warmup):
        chunk(i)
    plan.lcsa_check_device_error(stream)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    try:
        gpu_id = "GPU-%s" % torch.cuda.get_device_properties(dev).uuid
    except Exception:  # noqa: BLE001 - fall back to the index
        gpu_id = str(local)
    with ClockSampler(gpu_id) as clocks:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            starts[i].record(stream)
            chunk(args.warmup + i)
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
        # per-kernel times: the next chunks with events around each kernel
        plan.lcsa_plan_set_timing(args.steps)
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            chunk(args.warmup + args.steps + i)
        torch.cuda.synchronize(dev)
    plan.lcsa_check_device_error(stream)
    ms = sum(s_.elapsed_time(e_) for s_, e_ in zip(starts, ends)) / args.steps
    kms, _ = plan.lcsa_get_kernel_times()
    plan.destroy()
    flops = geo.selected_flops
    act = 2.0 * geo.channels
    k1_bytes = 2.0 * act * wl.batch * 2 * geo.q_tokens   # q and k of the new frames, read and written
    peaks = _peaks()
    line = {"metric": METRIC, "value": flops / (ms * 1e-3) / 1e12, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name + " (stream plan: KV ring, new frames per chunk)",
                       "q_tokens": geo.q_tokens, "kv_tokens": geo.kv_tokens, "topk": geo.topk,
                       "l2": "256 MiB buffer written before every timed chunk",
                       "kernel_times": "second pass of as many chunks, CUDA events around each kernel"},
            "kernels": {"prologue_ms": kms[0], "select_ms": kms[1], "attention_ms": kms[2],
                        "prologue_bytes": k1_bytes, "prologue_gbs": k1_bytes / (kms[0] * 1e-3) / 1e9,
                        "attention_tflops": flops / (kms[2] * 1e-3) / 1e12,
                        "hbm_peak_gbs": peaks["hbm_gbs"]},
            "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)
    return 0


def run_layers(args):
    """One step = the attention calls of one DiT chunk: args.layers sequential
    lcsa_forward calls of one geometry (three distinct input sets, cycled),
    timed eagerly and as one captured CUDA graph replayed per step."""
    import torch

    import block_sparse_video_lcsa_b200 as lcsa
    from block_sparse_video_lcsa_b200 import synth

    world, rank, local = _dist()
    if world > 1:
        print(json.dumps({"impl": "lcsa", "unavailable": "--layers times one GPU"}))
        return 0
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = synth.WORKLOADS[args.workload]

    def bf(a):
        return torch.from_numpy(a).view(torch.bfloat16).to(dev)

    sets = []
    for i in range(3):
        inp = synth.make_inputs(wl.replace(seed=i))
        sets.append((bf(inp.q), bf(inp.k), bf(inp.v), torch.from_numpy(inp.gamma_q).to(dev),
                     torch.from_numpy(inp.gamma_k).to(dev)))
    outs = [torch.empty_like(st[0]) for st in sets]
    plan = lcsa.lcsa_plan_create(lcsa.config_from_workload(wl), local)
    geo = plan.geometry
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))

    def chunk(stream):
        for layer in range(args.layers):
            q, k, v, gq, gk = sets[layer % 3]
            plan.lcsa_forward(q, k, v, gq, gk, outs[layer % 3], stream)

    with torch.cuda.stream(side):
        for _ in range(args.warmup):
            chunk(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            chunk(side)
        for _ in range(args.warmup):
            graph.replay()
    torch.cuda.synchronize(dev)
    plan.lcsa_check_device_error(side)

    def timed_pair():
        """Eager and graph steps alternate (so both see the same clocks under
        the power cap); returns the mean ms of each."""
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
        torch.cuda.synchronize(dev)
        for e in ev:
            e[0].record(side)
            chunk(side)
            e[1].record(side)
            e[2].record(side)
            graph.replay()
            e[3].record(side)
        torch.cuda.synchronize(dev)
        return (sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps,
                sum(e[2].elapsed_time(e[3]) for e in ev) / args.steps)

    try:
        gpu_id = "GPU-%s" % torch.cuda.get_device_properties(dev).uuid
    except Exception:  # noqa: BLE001 - fall back to the index
        gpu_id = str(local)
    with ClockSampler(gpu_id) as clocks:
        with torch.cuda.stream(side):
            eager_ms, graph_ms = timed_pair()
    plan.lcsa_check_device_error(side)
    del graph
    plan.destroy()
    flops = geo.selected_flops * args.layers
    line = {"metric": METRIC, "value": flops / (graph_ms * 1e-3) / 1e12, "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": graph_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "%s x %d layers (one CUDA graph per chunk)" % (wl.name, args.layers),
                       "l2": "three input sets (3 x %.0f MB) cycled over the layers" % (
                           (sets[0][0].numel() + 2 * sets[0][1].numel()) * 2 / 1e6)},
            "layers": {"count": args.layers, "eager_ms_per_layer": eager_ms / args.layers,
                       "graph_ms_per_layer": graph_ms / args.layers,
                       "eager_tflops": flops / (eager_ms * 1e-3) / 1e12},
            "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)
    return 0


def run_sharded(args):
    """One step = one layer's LCSA call with its heads split over the ranks
    (strong scaling: the layer is fixed, each rank computes its heads): the
    rank's per-token sums of squares, their all-reduce and the sharded call."""
    import torch
    import torch.distributed as dist

    import block_sparse_video_lcsa_b200 as lcsa
    from block_sparse_video_lcsa_b200 import synth
    from block_sparse_video_lcsa_b200.sharded import forward_heads_sharded, head_slices, sumsq_buffer

    world, rank, local = _dist()
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = synth.WORKLOADS[args.workload]
    inp = synth.make_inputs(wl)  # the same layer on every rank
    h0, h1 = head_slices(wl.heads, world)[rank]
    D = wl.head_dim
    sl = slice(h0 * D, h1 * D)

    def bf(a):
        return torch.from_numpy(a).view(torch.bfloat16)[..., sl].contiguous().to(dev)

    q, k, v = bf(inp.q), bf(inp.k), bf(inp.v)
    gq, gk = torch.from_numpy(inp.gamma_q[sl].copy()).to(dev), torch.from_numpy(inp.gamma_k[sl].copy()).to(dev)
    out = torch.empty_like(q)
    plan = lcsa.lcsa_plan_create(lcsa.config_from_workload(wl, heads=h1 - h0, heads_total=wl.heads), local)
    full_geo = lcsa.lcsa_config_resolve(lcsa.config_from_workload(wl))
    ssq = sumsq_buffer(plan, dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        forward_heads_sharded(plan, q, k, v, gq, gk, out, ssq=ssq)
    plan.lcsa_check_device_error(stream)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    s_starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    s_ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    try:
        gpu_id = "GPU-%s" % torch.cuda.get_device_properties(dev).uuid
    except Exception:  # noqa: BLE001 - fall back to the index
        gpu_id = str(local)
    with ClockSampler(gpu_id) as clocks:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            starts[i].record(stream)
            forward_heads_sharded(plan, q, k, v, gq, gk, out, ssq=ssq)
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
        # the sums-of-squares kernel alone
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            s_starts[i].record(stream)
            plan.lcsa_sumsq(q, k, ssq, stream)
            s_ends[i].record(stream)
        torch.cuda.synchronize(dev)
    plan.lcsa_check_device_error(stream)
    ms = _max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(starts, ends)) / args.steps, dev)
    ss_ms = _max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(s_starts, s_ends)) / args.steps, dev)
    ss_bytes = (q.numel() + k.numel()) * 2 + ssq.numel() * 4
    plan.destroy()
    if world > 1:
        dist.barrier()
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return 0
    peaks = _peaks()
    flops = full_geo.selected_flops
    line = {"metric": METRIC, "value": flops / (ms * 1e-3) / 1e12, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name + " (heads split over the ranks, sums of squares all-reduced)",
                       "heads_per_rank": [b - a for a, b in head_slices(wl.heads, world)],
                       "l2": "256 MiB buffer written before every timed call", "parallelism": "heads%d" % world},
            "sumsq": {"ms": ss_ms, "bytes": ss_bytes, "gbs": ss_bytes / (ss_ms * 1e-3) / 1e9,
                      "hbm_frac": ss_bytes / (ss_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]},
            "gpu_launches": (1 + _launches_per_call(wl)) * args.steps,
            "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    args = _args()
    if args.impl == "reference":
        return run_reference(args)
    if args.stream:
        return run_stream(args)
    if args.layers > 0:
        return run_layers(args)
    if args.shard_heads:
        return run_sharded(args)
    return run_lcsa(args)


if __name__ == "__main__":
    sys.exit(main())
