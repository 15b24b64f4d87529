"""Benchmark of the NVFP4 KV-cache hot path on B200.

One step = one AR step of the 1.3B-like streaming workload (batch 1, 12 heads,
head_dim 128, 1560 tokens per frame, chunk 3 frames = 4680 query tokens,
sink 3 + window 18 frames = 32760 keys per query) in steady state:
kv_ring_evict + nvfp4_kv_append + chunk_attention_nvfp4kv.  Inputs are seeded
synthetic bf16 N(0,1) with 1% K outlier channels x8.  Four independent caches
(one per emulated layer) and four input sets are cycled, so each step reads
a cache and inputs that are not L2-resident (4 x ~100 MB > 126 MB L2).

Prints one JSON line (rank 0).  --impl reference times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4-KV chunk attention TFLOP/s & query tok/s; KV quant-append GB/s"
N_LAYERS = 4


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def _ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu capture of this kernel on
    this workload, or None when there is none or the kernel's sources changed
    since the counters were taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(kernel)
    if not d or not d["workload"].startswith(workload + " "):
        return None
    h = hashlib.sha256()
    for src in d["sources"]:
        with open(os.path.join(ROOT, src), "rb") as f:
            h.update(f.read())
    if h.hexdigest()[:16] != d["source_sha256_16"]:
        return None
    return d["dram_bytes_read"] + d["dram_bytes_write"]


def workload_numbers(wl):
    """Algorithmic work per step (see the per-kernel accounting in the docs)."""
    T, Lq = wl.T, wl.Lq
    n_keys = (wl.S + wl.W) * T
    flop = 4.0 * wl.B * wl.H * Lq * n_keys * 128
    # append: read bf16 K and V, write codes (64 B) + scales (8 B) per token-head
    append_bytes = wl.B * Lq * wl.H * (2 * 256 + 2 * 72)
    twin_append_bytes = wl.B * Lq * wl.H * (2 * 256 + 2 * 256)
    # attention HBM bytes: Q in, O out, every visible K/V row once
    attn_bytes = wl.B * wl.H * (2 * Lq * 256 + n_keys * 2 * 72)
    return dict(flop=flop, append_bytes=append_bytes, twin_append_bytes=twin_append_bytes,
                attn_bytes=attn_bytes, n_keys=n_keys)


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "samples": len(sm), "reasons": sorted(reasons)}


def _dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def bench_config(wl, kv, ws):
    """The workload a line is measured on (shared by both arms)."""
    n_keys = (wl.S + wl.W) * wl.T
    return {"workload": f"{wl.name}: B{wl.B} H{wl.H} D128 T{wl.T} ({wl.grid_h}x{wl.grid_w}) "
                        f"C{wl.C} S{wl.S} W{wl.W}, {wl.Lq} query tokens, {n_keys} keys",
            "kv_cache": kv, "layers_cycled": 1 if wl.name == "long600" else N_LAYERS,
            "l2": ("one stream's cache for every step; 4 input sets cycled (172 MB > L2)"
                   if wl.name == "long600" else
                   "inputs and caches larger than L2 (4 independent layers cycled)"),
            "parallelism": f"replicas x{ws}"}


# --------------------------------------------------------------- our arm

class StreamBench:
    """Steady-state AR steps of one workload on this GPU: evict + append +
    attention per step, over N_LAYERS independent caches and input sets
    cycled (one cache for the long run), inputs resident in HBM."""

    def __init__(self, nv, torch, wl, kvd, seed, stream):
        import kvsynth
        self.nv, self.torch, self.wl, self.stream = nv, torch, wl, stream
        self.n_layers = 1 if wl.name == "long600" else N_LAYERS
        self.sets = []
        for i in range(N_LAYERS):
            x = kvsynth.chunk_qkv(wl, 1000 + i, seed=seed)
            self.sets.append({k: v.cuda() for k, v in x.items()})
        self.caches = [nv.KVCache(wl.B, wl.H, wl.grid_h, wl.grid_w, wl.C, wl.S, wl.W, kvd)
                       for _ in range(self.n_layers)]
        self.outs = [torch.empty_like(self.sets[0]["q"]) for _ in range(self.n_layers)]
        # multi-shot streams: shot ids per AR step (per-shot sinks, masking)
        self.sched = kvsynth.shot_schedule(wl, seed) if wl.shots > 1 else None
        self.steps_done = [0] * self.n_layers
        # fill every ring to steady state (window full); multi-shot runs start
        # their shot schedule at the first step
        fill = 0 if self.sched is not None else (wl.S + wl.W) // wl.C
        for li in range(self.n_layers):
            for s_ in range(fill):
                x = self.sets[s_ % N_LAYERS]
                c = self.begin_step(li)
                c.append(x["k"], x["v"])
                c.attention(x["q"], out=self.outs[li])
        torch.cuda.synchronize()

    def shot_ids(self, li):
        if self.sched is None:
            return None
        # the schedule repeats; shot ids keep increasing across repeats
        n = len(self.sched[0])
        k, rep = self.steps_done[li] % n, self.steps_done[li] // n
        return [self.sched[b][k] + self.wl.shots * rep for b in range(self.wl.B)]

    def begin_step(self, li):
        c = self.caches[li]
        ids = self.shot_ids(li)
        if ids is not None:
            for b, sid in enumerate(ids):
                c.begin_shot(b, sid)
        self.steps_done[li] += 1
        need = self.wl.C - min(c.free_frames(b) for b in range(self.wl.B))
        if need > 0:
            c.evict(need)
        return c

    def run(self, steps, warmup, dist=None, clocks=None):
        """Device-timed steps: events around the whole loop and around each
        step's append and attention (all on one stream)."""
        torch, wl, stream = self.torch, self.wl, self.stream
        ev = lambda: torch.cuda.Event(enable_timing=True)
        visible = []

        def one_step(i, timing):
            li = i % self.n_layers
            x = self.sets[(i + 1) % N_LAYERS]
            e0 = e1 = e2 = None
            if timing:
                e0 = ev(); e0.record(stream)
            c = self.begin_step(li)
            c.append(x["k"], x["v"], stream=stream)
            if timing:
                e1 = ev(); e1.record(stream)
            c.attention(x["q"], out=self.outs[li], stream=stream)
            if timing:
                e2 = ev(); e2.record(stream)
                visible.append(sum(len(c.visible(b)[2]) for b in range(wl.B)) * wl.T)
            return e0, e1, e2

        for i in range(warmup):
            one_step(i, False)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        foot0 = [c.footprint_bytes() for c in self.caches]
        alloc0 = torch.cuda.memory_allocated()
        free0 = torch.cuda.mem_get_info()[0]
        if clocks is not None:
            clocks.start()
            time.sleep(0.3)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        t0, t1 = ev(), ev()
        t0.record(stream)
        marks = [one_step(warmup + i, True) for i in range(steps)]
        t1.record(stream)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        clk = clocks.stop() if clocks is not None else None
        for c in self.caches:
            assert c.device_status() == 0, "device-side pipeline error"
        app = [a.elapsed_time(b) for a, b, _ in marks]
        att = [b.elapsed_time(c) for _, b, c in marks]
        step = [a.elapsed_time(c) for a, _, c in marks]
        return {"total_ms": t0.elapsed_time(t1), "app_ms": app, "att_ms": att, "step_ms": step,
                "visible_keys": visible, "clocks": clk,
                "memory": {"cache_footprint_bytes": foot0[0],
                           "footprint_constant": [c.footprint_bytes() for c in self.caches] == foot0,
                           "allocated_delta_bytes": torch.cuda.memory_allocated() - alloc0,
                           "device_free_delta_bytes": torch.cuda.mem_get_info()[0] - free0}}


def _pct(xs, p):
    xs = sorted(xs)
    return xs[min(len(xs) - 1, int(p * len(xs)))]


def cold_append_us(nv, torch, wl, kvd, n=40, reps=5):
    """Isolated cold-L2 time of one steady-state append launch (s_g fixed),
    by difference: events around n x (256 MB L2 flush + append) and around
    n x flush, so launch gaps hide behind the flush writes; median of reps.
    The append runs as an in-place overwrite of the newest chunk, which
    launches the same kernel on the same slots without moving the ring."""
    import kvsynth
    x = {k: v.cuda() for k, v in kvsynth.chunk_qkv(wl, 1000, 0).items()}
    c = nv.KVCache(wl.B, wl.H, wl.grid_h, wl.grid_w, wl.C, wl.S, wl.W, kvd)
    for _ in range(2):
        c.append(x["k"], x["v"])
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def loop(with_append):
        a, b = ev(), ev()
        torch.cuda.synchronize()
        a.record()
        for i in range(n):
            flush.fill_(i & 255)
            if with_append:
                c.overwrite(x["k"], x["v"])
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) * 1e3 / n

    loop(True), loop(False)
    res = sorted(loop(True) - loop(False) for _ in range(reps))
    assert c.device_status() == 0, "device-side pipeline error"
    return res[len(res) // 2]


def workload_summary(nv, torch, wl, kvd, steps, warmup, stream, peaks, seed=0):
    """One short steady-state run of another workload: attention TFLOP/s over
    the visible keys, append GB/s (in the step and isolated cold), step
    latency percentiles."""
    num = workload_numbers(wl)
    fp4 = kvd == nv.NVKV_KV_NVFP4
    sb = StreamBench(nv, torch, wl, kvd, seed, stream)
    r = sb.run(steps, warmup)
    K = len(r["att_ms"])
    flop = 4.0 * wl.H * wl.Lq * 128 * (sum(r["visible_keys"]) / K)
    att = sum(r["att_ms"]) / K
    app = sum(r["app_ms"]) / K
    tfl = flop / (att / 1e3) / 1e12
    app_bytes = num["append_bytes"] if fp4 else num["twin_append_bytes"]
    out = {"workload": bench_config(wl, "nvfp4" if fp4 else "bf16", 1)["workload"],
           "steps": K, "attn_ms": att, "attn_tflops": tfl,
           "attn_frac": tfl / peaks["bf16_tflops"],
           "append_in_step_gbs": app_bytes / (app / 1e3) / 1e9,
           "step_ms_p50": _pct(r["step_ms"], 0.5), "step_ms_p99": _pct(r["step_ms"], 0.99)}
    if wl.shots > 1:
        # steps differ in work (a shot start sees 7 of 21 frames per stream):
        # the latency per visible key is the flat quantity
        per = [1e6 * t / v for t, v in zip(r["step_ms"], r["visible_keys"])]
        out["step_ns_per_visible_key_p50"] = _pct(per, 0.5)
        out["step_ns_per_visible_key_p99"] = _pct(per, 0.99)
        out["visible_keys_per_step_min_max"] = [min(r["visible_keys"]), max(r["visible_keys"])]
    if wl.name == "long600":
        out["memory"] = r["memory"]
    if wl.name != "long600":
        us = cold_append_us(nv, torch, wl, kvd)
        out["append_cold_us"] = us
        out["append_cold_gbs"] = app_bytes / (us / 1e6) / 1e9
        out["append_cold_frac"] = out["append_cold_gbs"] / peaks["hbm_gbs"]
    del sb
    torch.cuda.empty_cache()
    return out


# Other workloads reported beside the headline (one GPU only): the 5B-like
# stream, the bf16-KV twin on both streams, the multi-shot batch, and the
# 600-step stream's latency and allocation record.
EXTRA_RUNS = [("stream5b", "nvfp4", 60), ("stream1p3b", "bf16", 60), ("stream5b", "bf16", 60),
              ("multishot", "nvfp4", 96), ("long600", "nvfp4", 300)]


def run_ours(args):
    import torch
    import torch.distributed as dist

    import kvsynth
    import nvfp4_kv_cache_append_b200 as nv

    ws, rank, local = _dist_env()
    torch.cuda.set_device(local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    wl = kvsynth.WORKLOADS[args.workload]
    num = workload_numbers(wl)
    fp4 = args.kv == "nvfp4"
    kvd = nv.NVKV_KV_NVFP4 if fp4 else nv.NVKV_KV_BF16
    stream = torch.cuda.Stream()
    torch.cuda.set_stream(stream)

    sb = StreamBench(nv, torch, wl, kvd, rank, stream)
    clocks = ClockSampler(local)
    r = sb.run(args.steps, args.warmup, dist if ws > 1 else None, clocks)
    clk = r["clocks"]
    total_ms = r["total_ms"]
    if ws > 1:
        t = torch.tensor([total_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())

    # end to end through the public host pipeline: every step uploads its
    # q/k/v from pinned host memory, runs evict + append + attention and
    # downloads the output to pinned host memory, on three streams so that
    # step k's upload overlaps step k-1's compute and step k-2's download
    host = [{k: v.cpu().pin_memory() for k, v in s_.items()} for s_ in sb.sets]
    host_out = [torch.empty(sb.sets[0]["q"].shape, dtype=torch.bfloat16).pin_memory()
                for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host[0].values())
    d2h = host_out[0].numel() * host_out[0].element_size()
    # one set of streams for all emulated layers: their steps run in order,
    # as a model's layers would
    pstreams = tuple(torch.cuda.Stream() for _ in range(3))
    pipes = [nv.HostPipeline(c, streams=pstreams) for c in sb.caches]

    def e2e_step(i):
        li = i % sb.n_layers
        shot = sb.shot_ids(li)
        sb.steps_done[li] += 1
        x = host[(i + 1) % N_LAYERS]
        pipes[li].submit(x["q"], x["k"], x["v"], host_out[i & 1], shot=shot)

    for i in range(3):
        e2e_step(i)
    for p in pipes:
        p.synchronize()
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    ev = lambda: torch.cuda.Event(enable_timing=True)
    a, b = ev(), ev()
    a.record(pstreams[0])
    for i in range(args.steps):
        e2e_step(i)
    b.record(pstreams[2])
    torch.cuda.synchronize()
    e2e_ms = a.elapsed_time(b)
    if ws > 1:
        t = torch.tensor([e2e_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    for c in sb.caches:
        assert c.device_status() == 0, "device-side pipeline error"

    peaks = _peaks()
    K = args.steps
    ms_step = total_ms / K
    tok_per_step = wl.B * wl.Lq
    value = ws * tok_per_step * K / (total_ms / 1e3)
    att_avg = sum(r["att_ms"]) / K
    app_avg = sum(r["app_ms"]) / K
    # FLOP of the steps actually timed: visible keys only (multi-shot masks)
    flop_step = 4.0 * wl.H * wl.Lq * 128 * (sum(r["visible_keys"]) / K)
    attn_tflops = flop_step / (att_avg / 1e3) / 1e12
    app_bytes = num["append_bytes"] if fp4 else num["twin_append_bytes"]
    append_gbs = app_bytes / (app_avg / 1e3) / 1e9
    peak = peaks["bf16_tflops_sustained"] if K * ms_step > 2000 else peaks["bf16_tflops"]
    del pipes
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "query tok/s",
        "n_gpus": ws,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e2m1/e4m3 cache, f16 MMA, f32 accumulate" if fp4 else "bf16 MMA, f32 accumulate",
        "data": "synthetic (seeded bf16 N(0,1), 1% K outlier channels x8)",
        "config": bench_config(wl, args.kv, ws),
        "attn_tflops": attn_tflops,
        "attn_flop_per_step": flop_step,
        "step_ms": {"p50": _pct(r["step_ms"], 0.5), "p99": _pct(r["step_ms"], 0.99)},
        "memory": r["memory"],
        "attn_ms": att_avg,
        "append_gbs": append_gbs,
        "append_ms": app_avg,
        "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": peak,
                     "unit": "TFLOP/s", "frac": attn_tflops / peak,
                     "traffic": _ncu_traffic("k_chunk_attn<1, 0>", wl.name) if fp4 else None,
                     "kernel": "k_chunk_attn", "peak_source": peaks["source"] + " bf16 (f16 same nominal rate)"},
        "append_roofline_in_step": {"bound": "hbm", "achieved": append_gbs, "peak": peaks["hbm_gbs"],
                                    "unit": "GB/s", "frac": append_gbs / peaks["hbm_gbs"],
                                    "timing": "events around the append inside the timed steps"},
        "e2e": {"value": ws * tok_per_step * K / (e2e_ms / 1e3), "unit": "query tok/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": 2 * K,
        "clocks": clk,
    }
    del sb
    torch.cuda.empty_cache()
    if ws == 1 and wl.name != "long600":
        us = cold_append_us(nv, torch, wl, kvd)
        gbs = app_bytes / (us / 1e6) / 1e9
        line["append_roofline"] = {
            "bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": gbs / peaks["hbm_gbs"], "kernel": "k_nvfp4_append" if fp4 else "k_bf16_append",
            "us_per_launch": us,
            "traffic": _ncu_traffic("k_nvfp4_append", wl.name) if fp4 else None,
            "traffic_note": "ncu DRAM bytes of one cold launch; the codes and scales it writes "
                            "stay in L2, so only the bf16 reads show",
            "timing": "isolated, cold L2: 40 x (256 MB flush + append) minus 40 x flush, median of 5"}
    if ws == 1 and not args.no_extra:
        clocks2 = ClockSampler(local)
        clocks2.start()
        extra = {}
        for name, kv, steps in EXTRA_RUNS:
            if name == wl.name and kv == args.kv:
                continue
            kd = nv.NVKV_KV_NVFP4 if kv == "nvfp4" else nv.NVKV_KV_BF16
            extra[f"{name} {kv}"] = workload_summary(nv, torch, kvsynth.WORKLOADS[name], kd,
                                                     steps, args.warmup, stream, peaks)
        extra["clocks"] = clocks2.stop()
        line["other_workloads"] = extra
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, seconds=args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------------- sequence-parallel mode

def run_sp(args):
    """--sp: one cache split over the ranks (strong scaling).  Each rank holds
    1/N of every frame's tokens; one step is append + attention over the
    shard + one barrier + the merge of the rank's query slice, which reads
    every rank's partial result (peers' over NVLink)."""
    import datetime

    import torch
    import torch.distributed as dist

    import kvsynth
    import nvfp4_kv_cache_append_b200 as nv
    from nvfp4_kv_cache_append_b200.sp import SequenceParallelKV

    ws, rank, local = _dist_env()
    torch.cuda.set_device(local)
    if "MASTER_ADDR" not in os.environ:          # one process without torchrun
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(29500 + os.getpid() % 1000),
                          RANK="0", WORLD_SIZE="1")
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                            device_id=torch.device("cuda", local))
    wl = kvsynth.WORKLOADS[args.workload]
    kvd = nv.NVKV_KV_NVFP4 if args.kv == "nvfp4" else nv.NVKV_KV_BF16
    stream = torch.cuda.Stream()
    torch.cuda.set_stream(stream)
    n_layers = 1 if wl.name == "long600" else N_LAYERS
    sets = [{k: v.cuda() for k, v in kvsynth.chunk_qkv(wl, 1000 + i, seed=0).items()}
            for i in range(N_LAYERS)]
    sps = [SequenceParallelKV(wl.B, wl.H, wl.grid_h, wl.grid_w, wl.C, wl.S, wl.W, kvd)
           for _ in range(n_layers)]
    q0, q1 = sps[0].plan.queries
    outs = [torch.empty(wl.B, q1 - q0, wl.H, 128, dtype=torch.bfloat16, device="cuda")
            for _ in range(n_layers)]
    for li in range(n_layers):
        for s_ in range((wl.S + wl.W) // wl.C):
            x = sets[s_ % N_LAYERS]
            sps[li].step(x["q"], x["k"], x["v"], out=outs[li])
    torch.cuda.synchronize()
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def one_step(i):
        x = sets[(i + 1) % N_LAYERS]
        sps[i % n_layers].step(x["q"], x["k"], x["v"], out=outs[i % n_layers])

    for i in range(args.warmup):
        one_step(i)
    torch.cuda.synchronize()
    dist.barrier()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    dist.barrier()
    a, b = ev(), ev()
    a.record(stream)
    for i in range(args.steps):
        one_step(args.warmup + i)
    b.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    clk = clocks.stop()
    t = torch.tensor([a.elapsed_time(b)], device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_ms = float(t.item())
    for sp in sps:
        assert sp.cache.device_status() == 0, "device-side pipeline error"
    K = args.steps
    line = {
        "metric": METRIC, "value": wl.B * wl.Lq * K / (total_ms / 1e3), "unit": "query tok/s",
        "n_gpus": ws, "steps": K, "warmup": args.warmup, "ms_per_step": total_ms / K,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": "e2m1/e4m3 cache, f16 MMA, f32 accumulate" if kvd == nv.NVKV_KV_NVFP4
                 else "bf16 MMA, f32 accumulate",
        "data": "synthetic (seeded bf16 N(0,1), 1% K outlier channels x8)",
        "config": dict(bench_config(wl, args.kv, ws),
                       parallelism=f"sequence-parallel KV split x{ws}",
                       kv_tokens_per_rank=f"{wl.T // ws} of {wl.T} per frame"),
        "gpu_launches": 3 * K,
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del sps
    dist.barrier()
    dist.destroy_process_group()


# ------------------------------------------ one-GPU shard emulation mode

def run_sp_emulate(args):
    """--sp-emulate: the per-rank kernel times of the sequence-parallel split
    for N = 1, 2, 3, 4, 6, 8 shards (those that divide T), all run on this one GPU: one shard's
    attention over its 1/N of every frame's tokens, and the merge of one
    rank's query slice from the N shards' partial results (local here; over
    NVLink on N GPUs).  L2 is flushed (256 MB written) before every timed
    launch.  Prints one JSON line."""
    import torch

    import kvsynth
    import nvfp4_kv_cache_append_b200 as nv

    torch.cuda.set_device(0)
    wl = kvsynth.WORKLOADS[args.workload]
    x = {k: v.cuda() for k, v in kvsynth.chunk_qkv(wl, 1000, 0).items()}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def timed(fn, n):
        ms = []
        for i in range(n + 3):
            flush.fill_(i & 0xFF)
            a, b = ev(), ev()
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            if i >= 3:
                ms.append(a.elapsed_time(b))
        return statistics.median(ms)

    rows = []
    for n in (1, 2, 3, 4, 6, 8):
        if wl.T % n:
            continue
        shards = [nv.KVCache(wl.B, wl.H, wl.grid_h, wl.grid_w, wl.C, wl.S, wl.W, nv.NVKV_KV_NVFP4,
                             shard_rank=r, shard_count=n) for r in range(n)]
        outs = [torch.empty_like(x["q"]) for _ in range(n)]
        lses = [torch.empty(wl.B, wl.H, wl.Lq, device="cuda") for _ in range(n)]
        for _ in range((wl.S + wl.W) // wl.C):
            for r, c in enumerate(shards):
                c.step(x["q"], x["k"], x["v"], out=outs[r], lse=lses[r])
        torch.cuda.synchronize()
        c = shards[-1]
        att = timed(lambda: c.attention(x["q"], out=outs[-1], lse=lses[-1]), args.steps)
        q1 = wl.Lq // n
        mo = torch.empty(wl.B, q1, wl.H, 128, dtype=torch.bfloat16, device="cuda")
        mrg = timed(lambda: nv.lse_merge(outs, lses, 0, q1, out=mo), args.steps)
        assert all(s_.device_status() == 0 for s_ in shards)
        rows.append({"shards": n, "shard_attention_ms": att, "merge_ms": mrg,
                     "cache_bytes_per_rank": shards[0].footprint_bytes()})
        del shards, outs, lses
    base = rows[0]["shard_attention_ms"] + rows[0]["merge_ms"]
    for r in rows:
        r["attention_plus_merge_speedup"] = base / (r["shard_attention_ms"] + r["merge_ms"])
    print(json.dumps({"metric": "sequence-parallel split, per-rank kernel times emulated on one GPU",
                      "workload": bench_config(wl, "nvfp4", 1)["workload"],
                      "l2": "256 MB written before every timed launch", "steps": args.steps,
                      "rows": rows}), flush=True)


# ------------------------------------------- projection + append mode

def run_project(args):
    """--project: the K/V projection of the step's chunk (hidden = H * 128,
    synthetic N(0, 1/hidden) weights) with the NVFP4 append fused into its
    epilogue, against the same work as two launches (projection to bf16 K/V,
    then the append).  Steady state (s_g fixed), 4 caches cycled."""
    import torch

    import kvsynth
    import nvfp4_kv_cache_append_b200 as nv

    ws, rank, local = _dist_env()
    torch.cuda.set_device(local)
    wl = kvsynth.WORKLOADS[args.workload]
    hidden = wl.H * 128
    g = torch.Generator().manual_seed(3)
    xs = [torch.randn(wl.B, wl.Lq, hidden, generator=g).to(torch.bfloat16).cuda()
          for _ in range(N_LAYERS)]
    ws_k = [(torch.randn(wl.H * 128, hidden, generator=g) / hidden ** 0.5).to(torch.bfloat16).cuda()
            for _ in range(N_LAYERS)]
    ws_v = [(torch.randn(wl.H * 128, hidden, generator=g) / hidden ** 0.5).to(torch.bfloat16).cuda()
            for _ in range(N_LAYERS)]
    caches = [nv.KVCache(wl.B, wl.H, wl.grid_h, wl.grid_w, wl.C, wl.S, wl.W, nv.NVKV_KV_NVFP4)
              for _ in range(N_LAYERS)]
    k_tmp = torch.empty(wl.B, wl.Lq, wl.H, 128, dtype=torch.bfloat16, device="cuda")
    v_tmp = torch.empty_like(k_tmp)
    stream = torch.cuda.Stream()
    torch.cuda.set_stream(stream)

    def room(c):
        need = wl.C - min(c.free_frames(b) for b in range(wl.B))
        if need > 0:
            c.evict(need)

    def fused(i):
        li = i % N_LAYERS
        room(caches[li])
        caches[li].project_append(xs[li], ws_k[li], ws_v[li], stream=stream)

    def two(i):
        li = i % N_LAYERS
        c = caches[li]
        room(c)
        c.project(xs[li], ws_k[li], ws_v[li], k_out=k_tmp, v_out=v_tmp, stream=stream)
        c.append(k_tmp, v_tmp, stream=stream)

    for i in range(N_LAYERS * ((wl.S + wl.W) // wl.C)):      # rings full, s_g fixed
        fused(i)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    res = {}
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    for name, fn in (("fused", fused), ("two_launch", two), ("fused_again", fused)):
        for i in range(args.warmup):
            fn(i)
        torch.cuda.synchronize()
        a, b = ev(), ev()
        a.record(stream)
        for i in range(args.steps):
            fn(i)
        b.record(stream)
        torch.cuda.synchronize()
        res[name] = a.elapsed_time(b) / args.steps
    clk = clocks.stop()
    for c in caches:
        assert c.device_status() == 0, "device-side pipeline error"
    fused_ms = min(res["fused"], res["fused_again"])
    flop = 2.0 * wl.B * wl.Lq * hidden * 2 * wl.H * 128
    peaks = _peaks()
    tflops = flop / (fused_ms / 1e3) / 1e12
    line = {
        "metric": "fused K/V projection + NVFP4 append, ms per step", "value": fused_ms,
        "unit": "ms", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": fused_ms, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 MMA, f32 accumulate, e2m1/e4m3 out",
        "data": "synthetic (seeded N(0,1) hidden states, N(0, 1/hidden) weights)",
        "config": {"workload": bench_config(wl, "nvfp4", 1)["workload"], "hidden": hidden,
                   "gemm": f"M={wl.B * wl.Lq} N={2 * wl.H * 128} K={hidden}",
                   "l2": "4 input/weight sets and caches cycled"},
        "two_launch_ms": res["two_launch"],
        "fused_gain": res["two_launch"] / fused_ms,
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": tflops / peaks["bf16_tflops"], "traffic": None,
                     "kernel": "k_kv_project", "peak_source": peaks["source"] + " bf16"},
        "gpu_launches": args.steps,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ oracle arm

class OracleSample:
    """Inputs of one steady-state step for timing the CPU oracle, drawn once
    (outside every timed region); `run` times the oracle on a bounded sample
    of the step: the quantize of `n_tok` of the chunk's tokens (K and V, every
    head) and the attention of `n_rows` query tokens (every head) over all
    the step's keys.  Returns query tok/s = 1 / (quantize s per token +
    attention s per query token)."""

    def __init__(self, wl, seed=0):
        import numpy as np

        import kvsynth
        self.wl = wl
        x = kvsynth.chunk_qkv(wl, 1, seed)
        self.kf = np.ascontiguousarray(x["k"].float().numpy()[0].transpose(1, 0, 2))   # [H][Lq][D]
        self.vf = np.ascontiguousarray(x["v"].float().numpy()[0].transpose(1, 0, 2))
        self.q = np.ascontiguousarray(x["q"].float().numpy()[0].transpose(1, 0, 2))
        n_keys = (wl.S + wl.W) * wl.T
        rng = np.random.default_rng(seed)
        self.k = rng.standard_normal((n_keys, 128))
        self.v = rng.standard_normal((n_keys, 128))
        self.fpos = np.repeat(np.arange(wl.S + wl.W, dtype=np.int32), wl.T)
        self.tok = np.tile(np.arange(wl.T, dtype=np.int32), wl.S + wl.W)
        l = np.arange(wl.Lq)
        self.qpos = (wl.S + wl.W - wl.C + l // wl.T).astype(np.int32)
        self.qtok = (l % wl.T).astype(np.int32)
        self.rng = rng

    def run(self, n_tok, n_rows):
        import numpy as np

        import oracle
        wl = self.wl
        t0 = time.perf_counter()
        for arr in (self.kf, self.vf):
            for h in range(wl.H):
                rows = arr[h, :n_tok]
                oracle.quantize_rows(rows, oracle.global_scale(oracle.amax(rows)))
        t_app = time.perf_counter() - t0
        rows = self.rng.choice(wl.Lq, n_rows, replace=False)
        t0 = time.perf_counter()
        for h in range(wl.H):
            oracle.attention_rows(self.q[h], self.k, self.v, self.fpos, self.tok, self.qpos,
                                  self.qtok, rows, wl.grid_w)
        t_att = time.perf_counter() - t0
        return 1.0 / (t_app / n_tok + t_att / n_rows), t_app, t_att


def _oracle_cores():
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def cpu_baseline(wl, seconds=20.0):
    import oracle
    oracle.build()
    sample = OracleSample(wl)
    # a pilot of 32 rows (after 8 that warm the thread pool) sizes the
    # sample to about `seconds` of oracle work
    sample.run(64, 8)
    _, t_app, t_att = sample.run(wl.Lq, 32)
    per_row = max(t_att / 32, 1e-6)
    n_rows = int(max(8, min(wl.Lq, (seconds - t_app) / per_row)))
    value, t_app, t_att = sample.run(wl.Lq, n_rows)
    return {"value": value, "unit": "query tok/s", "cores": _oracle_cores(), "kind": "oracle",
            "sample": f"one {wl.name} step: full-chunk quantize ({wl.Lq} tokens x {wl.H} heads, "
                      f"K and V) + attention of {n_rows} query tokens x {wl.H} heads over "
                      f"{(wl.S + wl.W) * wl.T} keys; tok/s = 1 / (quantize s/token + attention "
                      f"s/token)",
            "append_s": t_app, "attention_s": t_att}


def run_reference(args):
    """The reference arm: the CPU oracle as it stands, on this arm's workload,
    metric and config.  Each step is a bounded sample of the step (quantize
    of a slice of the chunk, attention of a few query rows), sized so that the
    whole run stays within about two minutes."""
    import kvsynth
    ws, rank, _ = _dist_env()
    if rank != 0:
        return
    wl = kvsynth.WORKLOADS[args.workload]
    import oracle
    oracle.build()
    sample = OracleSample(wl)
    # about 1.5 s of oracle work per step at 8 rows and the full chunk (8
    # host cores); shrink the sample when many steps are asked for
    budget_s = 120.0
    frac = min(1.0, budget_s / (1.5 * max(1, args.steps + args.warmup)))
    n_tok = max(wl.T // 8, int(wl.Lq * frac))
    n_rows = max(1, int(8 * frac))
    for _ in range(args.warmup):
        sample.run(n_tok, n_rows)
    vals = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        vals.append(sample.run(n_tok, n_rows)[0])
    wall = time.perf_counter() - t0
    value = len(vals) / sum(1.0 / v for v in vals)
    desc = (f"per step: quantize of {n_tok} of the chunk's {wl.Lq} tokens x {wl.H} heads (K and V) "
            f"+ attention of {n_rows} query tokens x {wl.H} heads over {(wl.S + wl.W) * wl.T} keys; "
            f"tok/s = 1 / (quantize s/token + attention s/token)")
    line = {"metric": METRIC, "value": value, "unit": "query tok/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * wall / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded bf16 N(0,1), 1% K outlier channels x8)",
            "config": bench_config(wl, args.kv, ws),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "query tok/s", "cores": _oracle_cores(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "query tok/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="stream1p3b")
    ap.add_argument("--kv", default="nvfp4", choices=["nvfp4", "bf16"])
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other workloads reported beside the headline")
    ap.add_argument("--sp-emulate", action="store_true",
                    help="per-rank kernel times of the sequence-parallel split, emulated on one GPU")
    ap.add_argument("--project", action="store_true",
                    help="time the fused K/V projection + append against two launches")
    ap.add_argument("--sp", action="store_true",
                    help="sequence-parallel KV split over the ranks instead of replicas")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.sp:
        run_sp(args)
    elif args.project:
        run_project(args)
    elif args.sp_emulate:
        run_sp_emulate(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
