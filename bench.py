"""Benchmark of the paged MQA-logits hot path on B200.

One step = one pass of the whole path over one batch: the GPU split schedule
(mqa_logits_schedule) and the logits kernel (paged_mqa_logits_fp8 or _fp4),
both through the C ABI. Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config decode]
  python bench.py --impl reference ...   # the CPU oracle, timed the same way

Timing: inputs already in HBM; the K timed steps are CUDA-graph replays that
rotate over R copies of the inputs whose total exceeds L2, so no step reads
K from L2 that an earlier step brought in. CUDA events on the launching
stream time the whole region (max over ranks) and, inside the graph, every
logits launch (the roofline figure). nvidia-smi samples SM clocks and
throttle reasons during a short soak of the same steps and the timed region.
With N > 1 GPUs every rank scores its own batch (weak scaling, no
collective on the data path).
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


def source_hash(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
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
    src = KERNEL_SOURCES if kind == "fp8" else FP4_KERNEL_SOURCES
    if vals.get("source_hash") != source_hash(src):
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


def cpu_baseline(wl, budget_s=10.0):
    """The oracle as it stands (single thread) on a bounded sample of rows."""
    import oracle
    t_total, tokens, rows = 0.0, 0, 0
    order = list(range(wl.B))
    for b in order:
        if wl.context_lens[b] <= 0:
            continue
        sub = workloads.Workload(**{**wl.__dict__, "B": 1, "q": wl.q[b:b + 1].contiguous(),
                                    "block_table": wl.block_table[b:b + 1].contiguous(),
                                    "context_lens": wl.context_lens[b:b + 1].contiguous(),
                                    "weights": wl.weights[b:b + 1].contiguous(),
                                    "out_len": int(wl.context_lens[b] + 3) // 4 * 4})
        t0 = time.perf_counter()
        oracle.logits(sub, with_absw=False)
        t_total += time.perf_counter() - t0
        tokens += int(wl.context_lens[b])
        rows += 1
        if t_total >= budget_s:
            break
    return {"value": tokens / t_total, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"first {rows} non-empty rows of the workload ({tokens} tokens), "
                      f"fp64 single-threaded C oracle, {t_total:.1f} s"}


def run_reference(args):
    """--impl reference: the CPU oracle, each step a bounded sample (one
    non-empty row, cycling) of the workload."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    wl = workloads.make_config(args.config)
    rows = [b for b in range(wl.B) if wl.context_lens[b] > 0]

    def step(i):
        b = rows[i % len(rows)]
        sub = workloads.Workload(**{**wl.__dict__, "B": 1, "q": wl.q[b:b + 1].contiguous(),
                                    "block_table": wl.block_table[b:b + 1].contiguous(),
                                    "context_lens": wl.context_lens[b:b + 1].contiguous(),
                                    "weights": wl.weights[b:b + 1].contiguous()})
        oracle.logits(sub, with_absw=False)
        return int(wl.context_lens[b])

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    tokens = sum(step(args.warmup + i) for i in range(args.steps))
    dt = time.perf_counter() - t0
    v = tokens / dt
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / max(args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": WORKLOAD_TEXT[args.config],
                                        "sample": "one non-empty row per step, cycling"},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": f"{args.steps} steps of one row each ({tokens} tokens)"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


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
    fn = mq.paged_mqa_logits_fp8 if kind == "fp8" else mq.paged_mqa_logits_fp4
    S = mq.mqa_logits_num_ctas(local)
    algo_bytes = wl.algorithmic_bytes()
    tokens = wl.tokens()

    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    set_bytes = (wl.q.numel() * wl.q.element_size() + wl.kv_cache.numel() + wl.block_table.numel() * 4
                 + wl.context_lens.numel() * 4 + wl.weights.numel() * 4
                 + wl.B * wl.next_n * wl.out_len * 4)
    R = max(2, -(-3 * l2 // set_bytes))
    R = min(R, 64)
    sets = []
    for _ in range(R):
        sets.append(dict(q=wl.q.to(dev), kv=wl.kv_cache.to(dev), bt=wl.block_table.to(dev),
                         ctx=wl.context_lens.to(dev), w=wl.weights.to(dev),
                         sched=torch.empty(S + 1, 2, dtype=torch.int32, device=dev),
                         out=torch.empty(wl.B, wl.next_n, wl.out_len, dtype=torch.float32,
                                         device=dev)))

    def step(st, ev=None):
        mq.mqa_logits_schedule(st["ctx"], S, st["sched"])
        if ev is not None:
            ev[0].record()
        fn(st["q"], st["kv"], st["bt"], st["ctx"], st["w"], st["sched"], st["out"],
           page_size=wl.page_size)
        if ev is not None:
            ev[1].record()

    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize(dev)
    # eager warm-up (compiles nothing; loads module, sets attributes)
    with torch.cuda.stream(stream):
        for i in range(2):
            step(sets[i % R])
    stream.synchronize()

    def capture(nsteps, timed_step):
        """A graph of nsteps steps; CUDA events bracket the logits launch of step
        `timed_step` only (None: no events), so every other launch keeps its
        programmatic overlap with the schedule kernel before it."""
        g = torch.cuda.CUDAGraph()
        ev = (torch.cuda.Event(enable_timing=True, external=True),
              torch.cuda.Event(enable_timing=True, external=True))
        with torch.cuda.graph(g, stream=stream):
            for i in range(nsteps):
                step(sets[i % R], ev if i == timed_step else None)
        return g, ([ev] if timed_step is not None else [])

    if args.kernel_only:
        # back-to-back logits launches only (schedules computed once): the
        # kernel's steady-state launch duration with PDL between launches
        for st in sets:
            mq.mqa_logits_schedule(st["ctx"], S, st["sched"])
        gk = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gk, stream=stream):
            for i in range(R):
                st = sets[i % R]
                fn(st["q"], st["kv"], st["bt"], st["ctx"], st["w"], st["sched"], st["out"],
                   page_size=wl.page_size)
        with torch.cuda.stream(stream):
            for _ in range(5):
                gk.replay()
        stream.synchronize()
        t_soak = time.perf_counter()  # let the clocks settle under load
        with torch.cuda.stream(stream):
            while time.perf_counter() - t_soak < args.soak:
                for _ in range(20):
                    gk.replay()
                stream.synchronize()
        k0 = torch.cuda.Event(enable_timing=True)
        k1 = torch.cuda.Event(enable_timing=True)
        reps = max(1, args.steps // R)
        with torch.cuda.stream(stream):
            k0.record()
            for _ in range(reps):
                gk.replay()
            k1.record()
        torch.cuda.synchronize(dev)
        kus = k0.elapsed_time(k1) * 1e3 / (reps * R)
        print(json.dumps({"kernel_only_us": kus, "GBps": algo_bytes / kus / 1e3,
                          "frac": algo_bytes / kus / 1e3 / measured_peaks()[0]["hbm_gbs"],
                          "config": args.config}), flush=True)
        return

    if args.topk:
        run_topk(args, mq, wl, sets, step, stream, dev, R)
        return

    # R graphs of the same R steps, graph j timing step j's logits launch; the
    # timed region replays them in turn, so each step's launch is timed once
    # per cycle and R - 1 of every R launches run with the overlap intact.
    graphs = [capture(R, j) for j in range(R)]
    g_main = graphs[0][0]
    rem = args.steps % R
    g_rem, ev_rem = capture(rem, 0) if rem else (None, [])

    # warm-up: W steps, plus a soak of about a second so the clocks settle
    with torch.cuda.stream(stream):
        for _ in range(max(1, -(-args.warmup // R))):
            g_main.replay()
    stream.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    t_soak = time.perf_counter()
    with torch.cuda.stream(stream):
        while time.perf_counter() - t_soak < args.soak:
            for _ in range(20):
                g_main.replay()
            stream.synchronize()

    # timed region: exactly K steps
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record()
        for i in range(args.steps // R):
            graphs[i % R][0].replay()
        if g_rem is not None:
            g_rem.replay()
        e1.record()
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if world > 1:
        torch.distributed.barrier()
    elapsed_ms = e0.elapsed_time(e1)
    timed = [g for g in graphs[:min(R, args.steps // R)]] if args.steps >= R else []
    kern_ms = [a.elapsed_time(b) for _, evs in timed for a, b in evs] + \
              [a.elapsed_time(b) for a, b in ev_rem]
    kern_avg_ms = float(np.mean(kern_ms)) if kern_ms else float("nan")

    elapsed_ms, total_tokens = reduce_max_sum(elapsed_ms, tokens, dev)
    kern_avg_ms, _ = reduce_max_sum(kern_avg_ms, 0.0, dev)

    value = total_tokens * args.steps / (elapsed_ms / 1e3)

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
    achieved = algo_bytes / (kern_avg_ms / 1e3) / 1e9
    traffic = profiled_traffic(args.config, kind)
    result = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3" if kind == "fp8" else "e2m1*e4m3->bf16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT[args.config],
                   "l2": f"rotating {R} input copies, {R * set_bytes / 1e6:.0f} MB > "
                         f"{l2 / 1e6:.0f} MB L2",
                   "parallelism": f"weak: {world} rank(s), one batch each" if world > 1
                   else "single GPU"},
        "gpu_launches": 2 * args.steps,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": traffic,
                     "peak_source": f"{peak_kind} hbm_gbs",
                     "kernel": f"paged_mqa_logits_{kind}", "kernel_us": kern_avg_ms * 1e3,
                     "kernel_timing": f"CUDA events around one logits launch per {R}-step "
                                      f"graph ({len(kern_ms)} launches sampled); the event "
                                      f"costs that launch its overlap with the schedule "
                                      f"kernel, so kernel_us is conservative",
                     "algorithmic_bytes_per_launch": algo_bytes},
        "hbm_gbs_step": algo_bytes / (elapsed_ms / args.steps / 1e3) / 1e9,
        "tokens_per_step": tokens,
        "clocks": clocks,
    }
    if e2e is not None:
        result["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wl, args.cpu_budget)
    if rank == 0:
        print(json.dumps(result), flush=True)
    del graphs, g_main, g_rem
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
    ap.add_argument("--kernel-only", action="store_true",
                    help="time back-to-back logits launches only (diagnostic)")
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
