"""Benchmark of the paged MQA-logits hot path on B200.

One step = one pass of the whole path over one batch: the GPU split schedule
(mqa_logits_schedule) and the logits kernel (paged_mqa_logits_fp8 or _fp4),
both through the C ABI. Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config decode]
  python bench.py --impl reference ...   # the CPU oracle, timed the same way

Timing: inputs already in HBM; the K timed steps are CUDA-graph replays that
rotate over R copies of the inputs whose total exceeds L2, so no step reads
K from L2 that an earlier step brought in. CUDA events on the launching
stream time the whole region (max over ranks). The roofline's kernel figure
is the logits kernel's average launch duration in a separate region: graphs
of back-to-back logits launches (each input copy's schedule computed once and
reused, as a schedule is reused across layers), events around each replay,
the median over the replays; the median of event-bracketed single launches
is reported beside it. nvidia-smi samples SM clocks and throttle reasons
during a short soak of the same steps and the timed region. With N > 1 GPUs
every rank scores its own batch (weak scaling, no collective on the data
path). With one GPU the line also carries the kernel figures of the other
full-size workloads (per_config).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "paged MQA logits: K tokens scored/s, HBM GB/s and % of roofline (1×B200)"
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCES = ["paged_mqa_logits_b200/csrc/logits_fp8.cu", "paged_mqa_logits_b200/csrc/common.cuh",
                  "paged_mqa_logits_b200/csrc/epilogue.cuh", "paged_mqa_logits_b200/csrc/ptx.cuh"]
FP4_KERNEL_SOURCES = ["paged_mqa_logits_b200/csrc/logits_fp4.cu",
                      "paged_mqa_logits_b200/csrc/common.cuh",
                      "paged_mqa_logits_b200/csrc/epilogue.cuh", "paged_mqa_logits_b200/csrc/ptx.cuh"]
NVFP4_KERNEL_SOURCES = ["paged_mqa_logits_b200/csrc/logits_nvfp4.cu",
                        "paged_mqa_logits_b200/csrc/common.cuh",
                        "paged_mqa_logits_b200/csrc/epilogue.cuh", "paged_mqa_logits_b200/csrc/ptx.cuh"]
SOURCES_OF_KIND = {"fp8": KERNEL_SOURCES, "fp4": FP4_KERNEL_SOURCES, "nvfp4": NVFP4_KERNEL_SOURCES}

WORKLOAD_TEXT = {
    "tiny": "tiny: B=3, next_n=1, H=4, D=32, page_size=16, ctx {37,0,70}, L=72, fp8",
    "decode": "DeepSeek-V3.2-indexer decode: B=64, next_n=1, H=64, D=128, page_size=64, "
              "ctx U[1024,8192], L=8192, fp8-e4m3 q/k, shuffled pages",
    "stress": "large-batch scheduler stress: B=2048, next_n=1, H=64, D=128, page_size=64, "
              "ctx U[0,4096] (10% zero, 10% 256m+-1), L=4096, fp8",
    "mtp": "long-context MTP: B=32, next_n=2, H=64, D=128, page_size=64, ctx U[32768,131072], "
           "L=131072, fp8",
    "fp4": "FP4 path: B=128, next_n=1, H=32, D=128, page_size=64, ctx U[512,16384], L=16384, "
           "e2m1 K with e4m3 per-16 block scales, bf16 q",
    "nvfp4": "block-scaled FP4: the FP4 path's shapes with q in NVFP4 too (e2m1 codes, e4m3 "
             "per-16 scales), tcgen05 kind::mxf4nvf4",
}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS}, "fallback"


def product_source(text):
    """The source as compiled into the product library: every
    `#ifdef MQA_DEBUG` block (code of the -DMQA_DEBUG build only) removed,
    its `#else` branch kept."""
    out = []
    stack = []  # open conditionals: [is an MQA_DEBUG block, its lines are dropped]

    def dropping():
        return any(debug and drop for debug, drop in stack)

    for line in text.splitlines(keepends=True):
        d = line.strip()
        if d.startswith("#if"):
            if not dropping() and d == "#ifdef MQA_DEBUG":
                stack.append([True, True])
                continue
            keep = not dropping()
            stack.append([False, False])
            if keep:
                out.append(line)
        elif d.startswith(("#else", "#elif")) and stack:
            if stack[-1][0]:
                stack[-1][1] = False
            elif not dropping():
                out.append(line)
        elif d.startswith("#endif") and stack:
            debug, _ = stack.pop()
            if not debug and not dropping():
                out.append(line)
        elif not dropping():
            out.append(line)
    return "".join(out)


def source_hash(paths):
    """Hash of the kernel sources as compiled into the product (debug-only
    blocks removed), which ties a committed ncu summary to the kernel code."""
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), encoding="utf-8") as f:
            h.update(product_source(f.read()).encode("utf-8"))
    return h.hexdigest()[:16]


def profiled_traffic(config, kind):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", f"{kind}_logits_{config}.md")
    if not os.path.exists(path):
        return None
    vals = {}
    for line in open(path):
        if line.startswith("<!-- ") and "=" in line:
            k, v = line[5:].split("-->")[0].strip().split("=", 1)
            vals[k.strip()] = v.strip()
    if vals.get("source_hash") != source_hash(SOURCES_OF_KIND[kind]):
        return None
    try:
        return float(vals["dram_bytes_per_launch_full"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append(dict(sm=float(f[1]), smmax=float(f[2]), power=float(f[3]),
                                 hw=f[5], hwt=f[6], swt=f[7], swp=f[8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("swp", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": float(np.median([r["sm"] for r in rows])),
                "sm_max_mhz": max(r["smmax"] for r in rows),
                "power_w_max": max(r["power"] for r in rows),
                "samples": len(rows), "reasons": sorted(reasons)}


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def _oracle_rate(wl, threads, budget_s):
    """tokens/s of the oracle over whole passes of the workload (at least one,
    repeated until budget_s is used)."""
    import oracle
    tokens, t_total, passes = 0, 0.0, 0
    while passes == 0 or t_total < budget_s:
        t0 = time.perf_counter()
        oracle.logits(wl, with_absw=False, threads=threads)
        t_total += time.perf_counter() - t0
        tokens += wl.tokens()
        passes += 1
    return tokens / t_total, passes, t_total


def cpu_baseline(wl, budget_s=10.0):
    """The oracle as it stands, timed on the host cores: every core (row-
    parallel threads, the headline figure) and one core, on whole passes over
    the same workload."""
    import oracle
    cores = oracle.host_cores()
    v_all, p_all, t_all = _oracle_rate(wl, None, budget_s / 2)
    v_one, p_one, t_one = _oracle_rate(wl, 1, budget_s / 2)
    return {"value": v_all, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(), "single_core_value": v_one,
            "sample": f"the whole workload ({wl.tokens()} tokens a pass): {p_all} pass(es) on "
                      f"{cores} cores in {t_all:.1f} s (rows spread over threads), {p_one} "
                      f"pass(es) on one core in {t_one:.1f} s; fp64 C oracle"}


def run_reference(args):
    """--impl reference: the CPU oracle on every host core; each step is one
    whole pass over the workload (the same configuration as our arm)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    wl = workloads.make_config(args.config)
    cores = oracle.host_cores()

    def step():
        oracle.logits(wl, with_absw=False, threads=None)
        return wl.tokens()

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    tokens = sum(step() for _ in range(args.steps))
    dt = time.perf_counter() - t0
    v = tokens / dt
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / max(args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": WORKLOAD_TEXT[args.config],
                                        "sample": "the whole workload every step"},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "cpu_model": cpu_model(),
                         "sample": f"{args.steps} whole passes ({tokens} tokens) on {cores} "
                                   f"cores, rows spread over threads"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def device_sets(wl, dev, S):
    """R copies of the workload's inputs on the device (plus a schedule and an
    output each), R chosen so that the copies together exceed 3x L2."""
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    set_bytes = (wl.q.numel() * wl.q.element_size() + wl.kv_cache.numel()
                 + wl.block_table.numel() * 4 + wl.context_lens.numel() * 4
                 + wl.weights.numel() * 4 + wl.B * wl.next_n * wl.out_len * 4)
    R = min(64, max(2, -(-3 * l2 // set_bytes)))
    sets = []
    for _ in range(R):
        sets.append(dict(q=wl.q.to(dev), kv=wl.kv_cache.to(dev), bt=wl.block_table.to(dev),
                         ctx=wl.context_lens.to(dev), w=wl.weights.to(dev),
                         sched=torch.empty(S + 1, 2, dtype=torch.int32, device=dev),
                         out=torch.empty(wl.B, wl.next_n, wl.out_len, dtype=torch.float32,
                                         device=dev)))
    return sets, R, set_bytes, l2


def logits_fn(mq, wl):
    """The logits entry point for the workload's kind, as f(q, kv, bt, ctx, w, sched, out, ...)."""
    if wl.kind == "nvfp4":
        return lambda *args, **kw: mq.paged_mqa_logits_nvfp4(*args, num_heads=wl.H, **kw)
    return mq.paged_mqa_logits_fp8 if wl.kind == "fp8" else mq.paged_mqa_logits_fp4


def run_gather_only(args, mq, wl, sets, S, stream, dev):
    """Diagnostic: the FP8 kernel's data movement alone (mqa_diag_fp8_gather),
    timed like the logits kernel, against the logits kernel on the same
    copies. Bytes moved per launch: whole pages of K rows (page_size * D each)
    for every unit, plus q tiles and weights."""
    if wl.kind != "fp8":
        raise SystemExit("--gather-only covers the FP8 path")
    g = kernel_figures(mq, wl, sets, S, stream, dev, launches=max(200, args.steps),
                       soak_s=args.soak, fn=mq.mqa_diag_fp8_gather)
    k = kernel_figures(mq, wl, sets, S, stream, dev, launches=max(200, args.steps),
                       soak_s=args.soak)
    ctx = wl.context_lens.to(torch.int64)
    pages = int(((ctx + wl.page_size - 1) // wl.page_size).sum())
    moved = pages * wl.page_size * wl.D + wl.B * wl.next_n * wl.H * (wl.D + 4)
    peaks, peak_kind = measured_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    gbps = moved / (g["back_to_back_us"] * 1e-6) / 1e9
    print(json.dumps({"config": args.config, "gather_only_us": g["back_to_back_us"],
                      "gather_bytes_per_launch": moved, "gather_GBps": gbps,
                      "gather_frac": gbps / hbm, "peak_GBps": hbm, "peak_kind": peak_kind,
                      "logits_kernel_us": k["back_to_back_us"],
                      "timing": "back-to-back: median over 7 replays of a graph of >= 200 "
                                "launches over the rotating input copies"}), flush=True)


def soak(g, stream, seconds):
    t0 = time.perf_counter()
    with torch.cuda.stream(stream):
        while time.perf_counter() - t0 < seconds:
            for _ in range(10):
                g.replay()
            stream.synchronize()


def kernel_figures(mq, wl, sets, S, stream, dev, launches=200, reps=7, soak_s=0.3, fn=None):
    """The logits kernel's average launch duration (us): a graph of at least
    `launches` back-to-back launches over the R input copies (schedules computed
    once per copy and reused), timed by events around each of `reps` replays;
    the median replay / launches. Also the median of `launches` single
    launches, each bracketed by events (an event pair around a launch costs it
    the launch latency, and its programmatic overlap with the launch before)."""
    fn = fn or logits_fn(mq, wl)
    R = len(sets)
    with torch.cuda.stream(stream):
        for st in sets:
            mq.mqa_logits_schedule(st["ctx"], S, st["sched"])
    stream.synchronize()
    per_graph = -(-launches // R) * R

    def launch(st):
        fn(st["q"], st["kv"], st["bt"], st["ctx"], st["w"], st["sched"], st["out"],
           page_size=wl.page_size)

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(per_graph):
            launch(sets[i % R])
    with torch.cuda.stream(stream):
        g.replay()
    stream.synchronize()
    soak(g, stream, soak_s)
    times = []
    for _ in range(reps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record()
            g.replay()
            e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1) * 1e3 / per_graph)
    b2b = float(np.median(times))
    # single launches, each between an event pair, R per graph replay
    evs = [(torch.cuda.Event(enable_timing=True, external=True),
            torch.cuda.Event(enable_timing=True, external=True)) for _ in range(R)]
    gb = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gb, stream=stream):
        for i in range(R):
            evs[i][0].record()
            launch(sets[i])
            evs[i][1].record()
    single = []
    with torch.cuda.stream(stream):
        gb.replay()
    stream.synchronize()
    while len(single) < launches:
        with torch.cuda.stream(stream):
            gb.replay()
        stream.synchronize()
        single += [a.elapsed_time(b) * 1e3 for a, b in evs]
    del g, gb
    return {"back_to_back_us": b2b, "back_to_back_replays_us": times,
            "launches_per_replay": per_graph, "bracketed_median_us": float(np.median(single)),
            "bracketed_launches": len(single)}


def roofline_entry(wl, figs, hbm, peak_kind):
    algo = wl.algorithmic_bytes()
    us = figs["back_to_back_us"]
    achieved = algo / (us * 1e-6) / 1e9
    return {"kernel_us": us, "tokens_per_s": wl.tokens() / (us * 1e-6),
            "GBps": achieved, "frac": achieved / hbm,
            "frac_bracketed": algo / (figs["bracketed_median_us"] * 1e-6) / 1e9 / hbm,
            "bracketed_median_us": figs["bracketed_median_us"],
            "algorithmic_bytes_per_launch": algo, "peak_source": f"{peak_kind} hbm_gbs"}


def run_ours(args):
    import paged_mqa_logits_b200 as mq
    from paged_mqa_logits_b200.shard import reduce_max_sum

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", device_id=dev,
                                             timeout=datetime.timedelta(seconds=120))
    cfg_index = workloads.CONFIG_ORDER.index(args.config)
    wl = workloads.make_config(args.config, seed=1234 + cfg_index + 1000 * rank)
    kind = wl.kind
    fn = logits_fn(mq, wl)
    S = mq.mqa_logits_num_ctas(local)
    algo_bytes = wl.algorithmic_bytes()
    tokens = wl.tokens()
    sets, R, set_bytes, l2 = device_sets(wl, dev, S)

    def step(st):
        mq.mqa_logits_schedule(st["ctx"], S, st["sched"])
        fn(st["q"], st["kv"], st["bt"], st["ctx"], st["w"], st["sched"], st["out"],
           page_size=wl.page_size)

    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize(dev)
    # eager warm-up (loads the module, sets kernel attributes: before any capture)
    with torch.cuda.stream(stream):
        for i in range(2):
            step(sets[i % R])
    stream.synchronize()

    if args.kernel_only:
        figs = kernel_figures(mq, wl, sets, S, stream, dev, launches=max(200, args.steps),
                              soak_s=args.soak)
        peaks, peak_kind = measured_peaks()
        hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
        e = roofline_entry(wl, figs, hbm, peak_kind)
        print(json.dumps({"config": args.config, "kernel_only_us": e["kernel_us"],
                          "GBps": e["GBps"], "frac": e["frac"],
                          "bracketed_median_us": e["bracketed_median_us"]}), flush=True)
        return

    if args.gather_only:
        run_gather_only(args, mq, wl, sets, S, stream, dev)
        return

    if args.topk:
        run_topk(args, mq, wl, sets, step, stream, dev, R)
        return

    # the timed graph: R steps over the R input copies
    g_main = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_main, stream=stream):
        for i in range(R):
            step(sets[i])
    rem = args.steps % R
    g_rem = None
    if rem:
        g_rem = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_rem, stream=stream):
            for i in range(rem):
                step(sets[i])

    # warm-up: at least W steps, then a soak of about a second so the clocks settle
    with torch.cuda.stream(stream):
        for _ in range(max(1, -(-args.warmup // R))):
            g_main.replay()
    stream.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    soak(g_main, stream, args.soak)

    # timed region: exactly K steps
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record()
        for _ in range(args.steps // R):
            g_main.replay()
        if g_rem is not None:
            g_rem.replay()
        e1.record()
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if world > 1:
        torch.distributed.barrier()
    elapsed_ms, total_tokens = reduce_max_sum(e0.elapsed_time(e1), tokens, dev)
    value = total_tokens * args.steps / (elapsed_ms / 1e3)

    # ---- the roofline's kernel figure (outside the timed region)
    figs = kernel_figures(mq, wl, sets, S, stream, dev, soak_s=min(args.soak, 0.5))
    kern_us, _ = reduce_max_sum(figs["back_to_back_us"], 0.0, dev)
    figs["back_to_back_us"] = kern_us

    # ---- end to end through the public API with host buffers
    e2e = None
    if args.e2e_steps > 0:
        hq = wl.q.pin_memory()
        hkv = wl.kv_cache.pin_memory()
        hbt = wl.block_table.pin_memory()
        hctx = wl.context_lens.pin_memory()
        hw = wl.weights.pin_memory()
        hout = torch.empty(wl.B, wl.next_n, wl.out_len, dtype=torch.float32).pin_memory()
        st = sets[0]
        h2d = sum(x.numel() * x.element_size() for x in (hq, hkv, hbt, hctx, hw))
        d2h = hout.numel() * 4

        def e2e_step():
            st["q"].copy_(hq, non_blocking=True)
            st["kv"].copy_(hkv, non_blocking=True)
            st["bt"].copy_(hbt, non_blocking=True)
            st["ctx"].copy_(hctx, non_blocking=True)
            st["w"].copy_(hw, non_blocking=True)
            step(st)
            hout.copy_(st["out"], non_blocking=True)

        with torch.cuda.stream(stream):
            for _ in range(2):
                e2e_step()
        stream.synchronize()
        if world > 1:
            torch.distributed.barrier()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a0.record()
            for _ in range(args.e2e_steps):
                e2e_step()
            a1.record()
        torch.cuda.synchronize(dev)
        e_ms, _ = reduce_max_sum(a0.elapsed_time(a1), 0.0, dev)
        e2e = {"value": total_tokens * args.e2e_steps / (e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": args.e2e_steps}

    peaks, peak_kind = measured_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    entry = roofline_entry(wl, figs, hbm, peak_kind)
    traffic = profiled_traffic(args.config, kind)
    result = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": {"fp8": "e4m3", "fp4": "e2m1*e4m3->f16", "nvfp4": "nvfp4"}[kind],
        "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT[args.config],
                   "l2": f"inputs larger than L2: rotating {R} input copies, "
                         f"{R * set_bytes / 1e6:.0f} MB > {l2 / 1e6:.0f} MB L2",
                   "parallelism": f"weak: {world} rank(s), one batch each" if world > 1
                   else "single GPU"},
        "gpu_launches": 2 * args.steps,
        "roofline": {"bound": "hbm", "achieved": entry["GBps"], "peak": hbm, "unit": "GB/s",
                     "frac": entry["frac"], "traffic": traffic,
                     "peak_source": entry["peak_source"],
                     "kernel": f"paged_mqa_logits_{kind}", "kernel_us": kern_us,
                     "kernel_timing": (
                         f"back-to-back: median over {len(figs['back_to_back_replays_us'])} "
                         f"replays of a graph of {figs['launches_per_replay']} logits launches "
                         f"over {R} input copies (schedules reused), CUDA events around each "
                         f"replay; frac uses this figure"),
                     "kernel_us_bracketed_median": figs["bracketed_median_us"],
                     "frac_bracketed": entry["frac_bracketed"],
                     "bracketed_timing": f"median of {figs['bracketed_launches']} single "
                                         f"launches, each between its own event pair",
                     "algorithmic_bytes_per_launch": algo_bytes},
        "hbm_gbs_step": algo_bytes / (elapsed_ms / args.steps / 1e3) / 1e9,
        "tokens_per_step": tokens,
        "clocks": clocks,
    }
    if e2e is not None:
        result["e2e"] = e2e
    del g_main, g_rem
    if world == 1 and not args.no_per_config:
        per = {args.config: {k: entry[k] for k in ("kernel_us", "tokens_per_s", "GBps", "frac",
                                                  "bracketed_median_us")}}
        del sets
        torch.cuda.empty_cache()
        for name in ("decode", "stress", "mtp", "fp4", "nvfp4"):
            if name == args.config:
                continue
            w2 = workloads.make_config(name)
            s2, _, _, _ = device_sets(w2, dev, S)
            with torch.cuda.stream(stream):
                for st in s2[:2]:
                    mq.mqa_logits_schedule(st["ctx"], S, st["sched"])
                    logits_fn(mq, w2)(st["q"], st["kv"], st["bt"], st["ctx"], st["w"],
                                      st["sched"], st["out"], page_size=w2.page_size)
            stream.synchronize()
            f2 = kernel_figures(mq, w2, s2, S, stream, dev, soak_s=0.2)
            e = roofline_entry(w2, f2, hbm, peak_kind)
            per[name] = {k: e[k] for k in ("kernel_us", "tokens_per_s", "GBps", "frac",
                                           "bracketed_median_us")}
            per[name]["workload"] = WORKLOAD_TEXT[name]
            del s2
            torch.cuda.empty_cache()
        result["per_config"] = per
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wl, args.cpu_budget)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def run_topk(args, mq, wl, sets, step, stream, dev, R):
    """Top-k selection over this workload's logits (diagnostic line, not the
    step contract): the top-k kernel alone in both orders, back to back over
    the R input copies, and the step with and without it (schedule + logits
    [+ top-k by token]). Algorithmic bytes: the valid logits read once, the
    context lengths and the indices written."""
    k = args.topk
    with torch.cuda.stream(stream):
        for st in sets:
            st["idx"] = torch.empty(wl.B, wl.next_n, k, dtype=torch.int32, device=dev)
            step(st)
    stream.synchronize()

    def graph(body):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(R):
                body(sets[i % R])
        return g

    def topk(st, by_token):
        mq.mqa_logits_topk(st["out"], st["ctx"], k, st["idx"], by_token=by_token)

    g_value = graph(lambda st: topk(st, False))
    g_token = graph(lambda st: topk(st, True))
    g_with = graph(lambda st: (step(st), topk(st, True)))
    g_plain = graph(step)

    def timed(g):
        with torch.cuda.stream(stream):
            for _ in range(5):
                g.replay()
            t0 = time.perf_counter()
            while time.perf_counter() - t0 < args.soak / 4:
                for _ in range(20):
                    g.replay()
                stream.synchronize()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            reps = max(1, args.steps // R)
            a.record()
            for _ in range(reps):
                g.replay()
            b.record()
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) * 1e3 / (reps * R)

    order = args.topk_order
    value_us = timed(g_value) if order in ("both", "value") else None
    token_us = timed(g_token) if order in ("both", "token") else None
    with_us = timed(g_with) if order == "both" else None
    plain_us = timed(g_plain) if order == "both" else None
    ctx = wl.context_lens.to(torch.int64)
    n = torch.arange(wl.next_n, dtype=torch.int64)
    cbn = (ctx[:, None] - wl.next_n + 1 + n[None, :]).clamp(min=0)
    cbn = torch.minimum(cbn, ctx[:, None].clamp(max=wl.out_len))
    rows = wl.B * wl.next_n
    algo = 4 * int(cbn.sum()) + 4 * k * rows + 4 * wl.B
    hbm = float(measured_peaks()[0].get("hbm_gbs", FALLBACK_HBM_GBS))
    del g_value, g_token, g_with, g_plain
    print(json.dumps({"topk": k, "config": args.config, "rows": rows,
                      "topk_by_value_us": value_us, "topk_by_token_us": token_us,
                      "step_us_with_topk_by_token": with_us, "step_us_without_topk": plain_us,
                      "topk_algorithmic_bytes": algo,
                      "GBps_by_token": algo / token_us / 1e3 if token_us else None,
                      "frac_by_token": algo / token_us / 1e3 / hbm if token_us else None}),
          flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="decode", choices=list(WORKLOAD_TEXT))
    ap.add_argument("--soak", type=float, default=1.0, help="seconds of untimed steps for clocks")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the kernel figures of the other full-size workloads")
    ap.add_argument("--kernel-only", action="store_true",
                    help="time back-to-back logits launches only (diagnostic)")
    ap.add_argument("--gather-only", action="store_true",
                    help="time the FP8 kernel's page gather alone against the logits kernel "
                         "(diagnostic)")
    ap.add_argument("--topk", type=int, default=0,
                    help="time top-k selection (this k) over the workload's logits (diagnostic)")
    ap.add_argument("--topk-order", default="both", choices=["both", "value", "token"],
                    help="with --topk: which output order(s) to time")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
