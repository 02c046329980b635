"""Benchmark: streamed frames/s of 24-block paged attention (and attention
TFLOP/s against the B200 bf16 tensor peak).

Workload (synthetic, shapes of a ViT-L/14 on 518 px frames): 24 transformer
blocks, each with its own page-pool region; H=16, D=64, 1369 patches +
6 special tokens per frame (page_size 1369), scale_frames 8, sliding window
64, 2-D RoPE (37x37 grid, theta 100) on patch Q/K, bf16.  One step = one
frame of the stream: for every block, append the frame's K/V (block 0 also
evicts, builds the visible page table and plans), then run paged attention
for the frame's 1375 queries.  The stream is pre-filled (appends only,
untimed), then W warm-up frames, then K timed frames.  The timed frames sit
in the middle of the 1000-frame stream, so that a short run costs what the
stream costs on average (the special tokens grow by 6 per frame, so later
frames attend over more keys); the defaults (W=3, K=925) stream frames
0..999 and time 75..999.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints one JSON line.  With N>1 (torchrun) every rank streams its own
replica (no data exchange; weak scaling) and rank 0 prints.
"""
from __future__ import annotations

import argparse
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

METRIC = "streamed frames/s (24-block paged attn) and attn TFLOP/s as % of bf16 peak"
WORKLOAD = "vitl_stream24"
# frames appended (no attention) before the warm-up steps, at least
PREFILL = {"vitl_stream24": 72, "vitl_step": 200}
STREAM_FRAMES = 1000      # length of the 24-block stream


def prefill_frames(workload, warmup, steps):
    """Untimed frames before the warm-up: the K timed frames are centred in the
    part of the stream after the minimum pre-fill and warm-up."""
    base = PREFILL[workload]
    if workload != "vitl_stream24":
        return base
    room = STREAM_FRAMES - base - warmup
    return base + max(0, (room - steps) // 2)
# further workloads measured by run_secondary (one JSON line each), with the
# workload whose shapes they use
SECONDARY = {"tiny_stream": "tiny_stream", "ragged4": "ragged4", "rollback10k": "rollback10k",
             "first_pass8": "vitl_stream24", "skip_append": "vitl_step",
             "nocross_step": "vitl_step"}


# DRAM traffic of one attention launch, from an ncu capture of the single
# ViT-L step (one 1375-row frame over 99,792 visible keys, 5 KV splits):
# dram__bytes_read.sum 454.0 MB + dram__bytes_write.sum 23.4 MB.  Traffic
# grows with the visible keys, so the bench scales it to the mean key count of
# its timed frames.  Set to None when the attention kernel changes until a new
# capture is taken.
ATTN_TRAFFIC_BYTES, ATTN_TRAFFIC_KEYS = 477.37e6, 99792


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["bf16_tflops"], p["bf16_tflops_sustained"], p["hbm_gbs"], "measured"
    except Exception:
        return 1590.0, 1400.0, 6650.0, "fallback"


L2_BYTES = 126 * 2**20


def _l2_note(w):
    """Visible K/V bytes per block at the last frame, against the L2 size."""
    ages = w.ages or (w.frames,)
    elem = 4 if w.dtype == "fp32" else 2
    tokens = sum(min(a, w.S + w.W) * w.P + w.ns * a for a in ages)
    kv = tokens * w.H * w.D * 2 * elem
    if kv > L2_BYTES:
        return f"inputs larger than L2 ({kv / 1e6:.0f} MB of visible K/V per block)"
    return f"visible K/V ({kv / 1e3:.0f} KB per block) fits in L2: timings are L2-resident"


def _config(w, extra=None):
    desc = (f"{w.name}: {w.blocks} block(s), H={w.H}, D={w.D}, P=page={w.P}, {w.ns} special/frame, "
            f"S={w.S}, W={w.W}, " + (f"2-D RoPE {w.rope_grid}x{w.rope_grid} theta={w.rope_theta:g}, "
                                     if w.rope_grid else "no RoPE, ") + w.dtype)
    cfg = {"workload": desc,
           "blocks": w.blocks, "heads": w.H, "head_dim": w.D, "page_size": w.P,
           "num_special": w.ns, "scale_frames": w.S, "sliding_window": w.W,
           "parallelism": "replicas", "l2": _l2_note(w)}
    if extra:
        cfg.update(extra)
    return cfg


def max_over_ranks(values, world, device):
    """Element-wise max of per-rank timings (all ranks take part)."""
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_rate(world, units_per_rank, elapsed_ms):
    """Units all ranks processed per second, timed by the slowest rank."""
    return world * units_per_rank / (elapsed_ms / 1e3)


def _visible(t, w):
    """Visible tokens once t frames are in the stream (append + evict)."""
    return min(t, w.S) * w.P + min(max(t - w.S, 0), w.W) * w.P + w.ns * t


class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons sampled during the
    timed region: read through NVML every 20 ms on the device the run uses
    (found by its UUID), else with nvidia-smi every 200 ms.  Read-only: no
    setting of the GPU is touched."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40}
    INTERVAL_S = 0.02

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None
        self.path = None
        self.thread = None
        self.rows = []
        self.max_mhz = None
        self.limit_w = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        uuid = str(torch.cuda.get_device_properties(self.idx).uuid)
        if not uuid.startswith("GPU-"):
            uuid = "GPU-" + uuid
        return pynvml, pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())

    def _poll(self, nv, h):
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop.is_set():
            try:
                self.rows.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                  nv.nvmlDeviceGetPowerUsage(h) / 1000.0, int(get_reasons(h))))
            except Exception:
                pass
            self.stop.wait(self.INTERVAL_S)

    def __enter__(self):
        try:
            import threading
            nv, h = self._nvml_handle()
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            try:
                self.limit_w = nv.nvmlDeviceGetEnforcedPowerLimit(h) / 1000.0
            except Exception:
                self.limit_w = None
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._poll, args=(nv, h), daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.thread = None
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.idx)], stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.out.close()

    def summary(self):
        if self.thread is not None:
            if not self.rows:
                return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples"],
                        "source": "nvml"}
            reasons = sorted({n for _, _, bits in self.rows
                              for n, b in self.REASON_BITS.items() if bits & b})
            return {"sm_mhz": statistics.median(r[0] for r in self.rows),
                    "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.rows),
                    "power_w_max": max(r[1] for r in self.rows),
                    "power_limit_w": self.limit_w,
                    "source": f"nvml every {int(self.INTERVAL_S * 1000)} ms"}
        if self.proc is None or not self.path:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows),
                "power_w_max": max((float(r[3]) for r in rows
                                    if r[3].replace(".", "").isdigit()), default=None),
                "source": "nvidia-smi every 200 ms"}


# ------------------------------------------------------------------ GPU arm
def run_gpu(args, rank, world, local_rank):
    import numpy as np
    import torch
    from dataclasses import replace

    from streaming_video_transformer_b200.cache import PagedKVCache
    from streaming_video_transformer_b200.inputs import WORKLOADS, frame_qkv

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = replace(WORKLOADS[args.workload], R=4)
    L = w.blocks
    prefill = prefill_frames(args.workload, args.warmup, args.steps)
    # The end-to-end leg's first copy in and last copy out cannot overlap
    # compute; as many frames as the device-resident leg (8 to 64) keep
    # that fill and drain from dominating a short run.
    e2e_steps = min(max(args.steps, 8), 64)
    total_frames = prefill + args.warmup + args.steps + e2e_steps
    max_pages = (w.S + w.W + 1) + math.ceil(total_frames * w.ns / w.P) + 2
    cache = PagedKVCache(max_pages, w.P, w.H, w.D, w.W, w.S, num_blocks=L, num_special=w.ns,
                         dtype=w.dtype, rope_grid=w.rope_grid, rope_theta=w.rope_theta,
                         device=dev)
    # R distinct frames per block: pinned host copies (end-to-end leg) and device copies.
    host = [[[x.pin_memory() for x in frame_qkv(w, b, rank, i)] for i in range(w.R)]
            for b in range(L)]
    devin = [[[x.to(dev) for x in host[b][i]] for i in range(w.R)] for b in range(L)]
    out = torch.empty((w.Nq, w.H, w.D), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    t_frame = 0

    def append_only(t):
        for b in range(L):
            q, k, v = devin[b][t % w.R]
            cache.append_frame(b, k, v)
        cache.evict_frames()

    def step(t, inputs, ev=None, outs=None):
        """One frame: append (+ evict/build/plan at block 0) and attention per block."""
        for b in range(L):
            q, k, v = inputs(b, t)
            cache.append_frame(b, k, v)
            if b == 0:
                cache.evict_frames()
                cache.build_visible_page_table()
                cache.plan([w.Nq])
            if ev is not None:
                ev[0].record(stream)
            cache.run(b, q, out=outs[b] if outs is not None else out)
            if ev is not None:
                ev[1].record(stream)
                ev = None

    dev_inputs = lambda b, t: devin[b][t % w.R]
    for t in range(prefill):
        append_only(t)
    t_frame = prefill
    for _ in range(args.warmup):
        step(t_frame, dev_inputs)
        t_frame += 1
    info = cache.plan_info()
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    # --- device-resident timed region ---------------------------------------
    run_events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    first_timed = t_frame
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        start.record(stream)
        for i in range(args.steps):
            step(t_frame, dev_inputs, ev=run_events[i])
            t_frame += 1
        end.record(stream)
        torch.cuda.synchronize()
    barrier()
    elapsed_ms = start.elapsed_time(end)
    run_ms = [a.elapsed_time(b) for a, b in run_events]        # block-0 run of each frame
    cache.device_error()
    clocks = clk.summary()
    timed_frames = list(range(first_timed, t_frame))
    flops_per_block = [4.0 * w.Nq * _visible(t + 1, w) * w.H * w.D for t in timed_frames]
    total_flops = L * sum(flops_per_block)

    # --- end-to-end: every frame's Q/K/V of all blocks copied in from pinned
    # host memory, and every block's output copied back to pinned host memory.
    # Copies in and out run on their own streams, double-buffered by frame
    # parity, so they overlap the attention of the neighbouring frames.
    h2d_stream = torch.cuda.Stream(device=dev)
    d2h_stream = torch.cuda.Stream(device=dev)
    stage = [[[torch.empty_like(x) for x in devin[b][0]] for b in range(L)] for _ in range(2)]
    outs = [[torch.empty((w.Nq, w.H, w.D), dtype=torch.bfloat16, device=dev) for _ in range(L)]
            for _ in range(2)]
    res_host = [[torch.empty((w.Nq, w.H, w.D), dtype=torch.bfloat16).pin_memory()
                 for _ in range(L)] for _ in range(2)]
    copied = [torch.cuda.Event() for _ in range(2)]       # inputs of a parity landed
    consumed = [torch.cuda.Event() for _ in range(2)]     # inputs of a parity used
    computed = [torch.cuda.Event() for _ in range(2)]     # outputs of a parity written
    drained = [torch.cuda.Event() for _ in range(2)]      # outputs of a parity copied out
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h2d = d2h = 0

    def enqueue_copy_in(i, t):
        nonlocal h2d
        with torch.cuda.stream(h2d_stream):
            h2d_stream.wait_event(consumed[i % 2])
            for b in range(L):
                for dst, src in zip(stage[i % 2][b], host[b][t % w.R]):
                    dst.copy_(src, non_blocking=True)
                    h2d += src.numel() * src.element_size()
            copied[i % 2].record(h2d_stream)

    def enqueue_copy_out(i):
        nonlocal d2h
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(computed[i % 2])
            for b in range(L):
                res_host[i % 2][b].copy_(outs[i % 2][b], non_blocking=True)
                d2h += outs[i % 2][b].numel() * outs[i % 2][b].element_size()
            drained[i % 2].record(d2h_stream)

    for ev in consumed + drained:
        ev.record(stream)
    barrier()
    torch.cuda.synchronize()
    t0 = t_frame
    e_start.record(stream)
    enqueue_copy_in(0, t0)
    for i in range(e2e_steps):
        if i + 1 < e2e_steps:
            enqueue_copy_in(i + 1, t0 + i + 1)
        stream.wait_event(copied[i % 2])
        stream.wait_event(drained[i % 2])
        buf = stage[i % 2]
        if args.e2e_path == "graph":   # one svt_frame_step call, replayed as a CUDA graph
            cache.frame_step([buf[b][1] for b in range(L)], [buf[b][2] for b in range(L)],
                             [buf[b][0] for b in range(L)], outs[i % 2], use_graph=True)
        else:
            step(t0 + i, lambda b, t: buf[b], outs=outs[i % 2])
        consumed[i % 2].record(stream)
        computed[i % 2].record(stream)
        enqueue_copy_out(i)
    for ev in drained:
        stream.wait_event(ev)
    e_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e_start.elapsed_time(e_end)
    h2d_per_step = h2d // e2e_steps
    d2h_per_step = d2h // e2e_steps
    e2e_flops = L * sum(4.0 * w.Nq * _visible(t0 + i + 1, w) * w.H * w.D for i in range(e2e_steps))

    elapsed_ms, e2e_ms = max_over_ranks([elapsed_ms, e2e_ms], world, dev)

    # per block: append, [RoPE on Q], attention, [merge]; plus one table build per frame
    kernels_per_step = L * (2 + (1 if w.rope_grid else 0)
                            + (1 if max(info["splits"]) > 1 else 0)) + 1
    return dict(elapsed_ms=elapsed_ms, run_ms=run_ms, flops_per_block=flops_per_block,
                total_flops=total_flops, clocks=clocks, info=info, w=w,
                e2e_ms=e2e_ms, e2e_steps=e2e_steps, e2e_flops=e2e_flops,
                h2d_per_step=h2d_per_step, d2h_per_step=d2h_per_step,
                kernels_per_step=kernels_per_step, first_timed=first_timed, last_timed=t_frame)


# ----------------------------------------------------- secondary workloads
def run_secondary(args):
    """The other workloads of the scheme, each timed with CUDA events:
    tiny_stream -- the whole 12-frame stream (append, evict, build, plan, run
                   per frame), repeated; ragged4 -- one batched run over four
                   streams aged 10/70/300/2000 (fp16, D=128); rollback10k --
                   10,000 offered frames, every 3rd deferred and rejected with
                   p=0.3, in bf16, and a sample of late frames with an fp32 pool;
    first_pass8 -- the first pass over the 8 scale frames of the RoPE stream
                   (one block): all 8 x 1375 queries attend over all 8
                   frames at once, no mask among them;
    skip_append -- a non-keyframe of the single ViT-L step attending to the
                   cache plus its own K/V: as a dense segment (nothing
                   stored), and through defer, append, attend and roll back;
    nocross_step -- the single ViT-L step on a pool without cross-frame
                   special retention (a frame's specials leave with it)."""
    import torch
    from dataclasses import replace

    from streaming_video_transformer_b200.cache import PagedKVCache
    from streaming_video_transformer_b200.inputs import WORKLOADS, frame_qkv, keyframe_decisions

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = WORKLOADS[SECONDARY[args.workload]]
    if args.workload == "first_pass8":
        w = replace(w, blocks=1)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    line = {"impl": "svt", "workload": args.workload, "n_gpus": 1, "data": "synthetic",
            "dtype": w.dtype, "config": _config(w)}
    flops_of = lambda nq, nk, H, D: 4.0 * nq * nk * H * D

    def make(wl, frames, streams=1):
        mp = streams * (wl.S + wl.W + 1) + sum(math.ceil(f * wl.ns / wl.P) for f in frames) + 2 * streams
        return PagedKVCache(mp, wl.P, wl.H, wl.D, wl.W, wl.S, num_special=wl.ns, num_streams=streams,
                            dtype=wl.dtype, max_qo_len=streams * wl.Nq, device=dev)

    if args.workload == "tiny_stream":
        c = make(w, [w.frames])
        fr = [[x.to(dev) for x in frame_qkv(w, 0, 0, t)] for t in range(w.frames)]
        out = torch.empty_like(fr[0][0])

        def separate_calls():
            c.reset()
            for t in range(w.frames):
                q, k, v = fr[t]
                c.append_frame(0, k, v)
                c.evict_frames()
                c.build_visible_page_table()
                c.plan([w.Nq])
                c.run(0, q, out=out)

        def one_call(use_graph):
            def f():
                c.reset()
                for t in range(w.frames):
                    q, k, v = fr[t]
                    c.frame_step([k], [v], [q], [out], use_graph=use_graph)
            return f

        variants = {"separate_calls": separate_calls, "frame_step": one_call(False),
                    "frame_step_graph": one_call(True)}
        us = {}
        for name, fn in variants.items():
            for _ in range(args.warmup):
                fn()
            torch.cuda.synchronize()
            a, b = ev(), ev()
            a.record()
            for _ in range(args.steps):
                fn()
            b.record()
            torch.cuda.synchronize()
            us[name] = 1e3 * a.elapsed_time(b) / (args.steps * w.frames)
        builds, replays = c.graph_counts()
        line.update(metric="frames/s (12-frame stream, full frame step)",
                    value=1e6 / us["frame_step_graph"], unit="frames/s",
                    us_per_frame=us, steps=args.steps,
                    note="value: svt_frame_step with CUDA-graph replay (one call and one graph "
                         "launch per frame); us_per_frame also gives the five separate calls "
                         "and svt_frame_step without a graph",
                    graphs={"built": builds, "replays": replays})
    elif args.workload == "ragged4":
        ages = list(w.ages)
        c = make(w, ages, streams=4)
        for s_, age in enumerate(ages):
            fr = [[x.to(dev) for x in frame_qkv(w, 0, s_, i)] for i in range(min(w.R, age))]
            for t in range(age):
                c.append_frame(0, fr[t % len(fr)][1], fr[t % len(fr)][2], stream=s_)
                c.evict_frames(s_)
        c.build_visible_page_table()
        c.plan([w.Nq] * 4)
        info = c.plan_info()
        q = torch.cat([frame_qkv(w, 0, s_, 0)[0] for s_ in range(4)]).to(dev)
        out = torch.empty_like(q)
        for _ in range(args.warmup):
            c.run(0, q, out=out)
        torch.cuda.synchronize()
        times = []
        for _ in range(args.steps):
            a, b = ev(), ev()
            a.record()
            c.run(0, q, out=out)
            b.record()
            times.append((a, b))
        torch.cuda.synchronize()
        ms = statistics.median(x.elapsed_time(y) for x, y in times)
        flops = sum(flops_of(w.Nq, nk, w.H, w.D) for nk in info["kv_tokens"])
        line.update(metric="batched run over 4 ragged streams", value=flops / (ms / 1e3) / 1e12,
                    unit="TFLOP/s", ms_per_run=ms, kv_tokens=info["kv_tokens"],
                    splits=info["splits"], steps=args.steps)
    elif args.workload == "first_pass8":
        F = w.S
        c = PagedKVCache(F + w.W + 4, w.P, w.H, w.D, w.W, w.S, num_special=w.ns, dtype=w.dtype,
                         max_qo_len=F * w.Nq, rope_grid=w.rope_grid, rope_theta=w.rope_theta,
                         device=dev)
        fr = [[x.to(dev) for x in frame_qkv(w, 0, 0, t)] for t in range(F)]
        q = torch.cat([fr[t][0] for t in range(F)])
        out = torch.empty_like(q)
        # the 8 frames' K/V (90 MB) fit in L2: flush it before every timed pass
        flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)

        def first_pass():
            c.reset()
            for t in range(F):
                c.append_frame(0, fr[t][1], fr[t][2])
                c.evict_frames()
            c.build_visible_page_table()
            c.plan([F * w.Nq])
            c.run(0, q, out=out)

        for _ in range(args.warmup):
            first_pass()
        torch.cuda.synchronize()
        whole, runs = [], []
        for _ in range(args.steps):
            flush.zero_()
            a, b = ev(), ev()
            a.record()
            first_pass()
            b.record()
            flush.zero_()
            x, y = ev(), ev()
            x.record()
            c.run(0, q, out=out)
            y.record()
            whole.append((a, b))
            runs.append((x, y))
        torch.cuda.synchronize()
        nk = c.plan_info()["kv_tokens"][0]
        flops = flops_of(F * w.Nq, nk, w.H, w.D)
        ms_whole = statistics.median(x.elapsed_time(y) for x, y in whole)
        ms_run = statistics.median(x.elapsed_time(y) for x, y in runs)
        line["config"]["l2"] = "8 frames' K/V (90 MB) fit in L2; L2 flushed before each timed pass"
        line.update(metric="attention TFLOP/s of the multi-frame first pass (8 scale frames)",
                    value=flops / (ms_run / 1e3) / 1e12, unit="TFLOP/s", ms_run=ms_run,
                    ms_first_pass=ms_whole, query_rows=F * w.Nq, kv_tokens=nk,
                    splits=c.plan_info()["splits"], steps=args.steps,
                    note="value: svt_run over all 8 frames' queries; ms_first_pass adds the 8 "
                         "appends (with the K rotation), the table build and the plan")
    elif args.workload in ("skip_append", "nocross_step"):
        cross = args.workload == "skip_append"
        pre = PREFILL["vitl_step"]
        c = PagedKVCache(w.S + w.W + 2 + math.ceil(pre * w.ns / w.P) + 2, w.P, w.H, w.D, w.W, w.S,
                         num_special=w.ns, dtype=w.dtype, max_qo_len=w.Nq,
                         cross_frame_special=cross, device=dev)
        fr = [[x.to(dev) for x in frame_qkv(w, 0, 0, i)] for i in range(w.R)]
        for t in range(pre):
            c.append_frame(0, fr[t % w.R][1], fr[t % w.R][2])
            c.evict_frames()
        c.build_visible_page_table()
        q, k, v = fr[pre % w.R]
        out = torch.empty_like(q)

        def timed(fn):
            for _ in range(args.warmup):
                fn()
            torch.cuda.synchronize()
            marks = []
            for _ in range(args.steps):
                a, b = ev(), ev()
                a.record()
                fn()
                b.record()
                marks.append((a, b))
            torch.cuda.synchronize()
            return statistics.median(x.elapsed_time(y) for x, y in marks)

        if cross:
            def segment():
                c.plan([w.Nq], extra_len=[w.Nq])
                c.run(0, q, out=out, k_extra=k, v_extra=v)

            def via_pool():
                c.set_defer_eviction(True)
                c.append_frame(0, k, v)
                c.evict_frames()
                c.build_visible_page_table()
                c.plan([w.Nq])
                c.run(0, q, out=out)
                c.rollback_last_frame()
                c.set_defer_eviction(False)
                c.build_visible_page_table()

            ms_seg = timed(segment)
            c.plan([w.Nq], extra_len=[w.Nq])
            nk = c.plan_info()["kv_tokens"][0]
            ms_pool = timed(via_pool)
            line.update(metric="non-keyframe step: attention over the cache plus its own K/V",
                        value=flops_of(w.Nq, nk, w.H, w.D) / (ms_seg / 1e3) / 1e12,
                        unit="TFLOP/s", ms_dense_segment=ms_seg, ms_defer_append_rollback=ms_pool,
                        kv_tokens=nk, steps=args.steps,
                        note="value: svt_plan_extra + svt_run_extra with the frame's K/V as a "
                             "dense segment (nothing written to the pool); "
                             "ms_defer_append_rollback: the frame appended, attended and rolled "
                             "back (the table rebuilt afterwards)")
        else:
            c.plan([w.Nq])
            nk = c.plan_info()["kv_tokens"][0]
            ms = timed(lambda: c.run(0, q, out=out))
            line.update(metric="single ViT-L step without cross-frame special retention",
                        value=flops_of(w.Nq, nk, w.H, w.D) / (ms / 1e3) / 1e12, unit="TFLOP/s",
                        ms_run=ms, kv_tokens=nk, splits=c.plan_info()["splits"],
                        steps=args.steps)
        line["config"]["cross_frame_special"] = cross
    else:   # rollback10k
        dec = keyframe_decisions(w, w.frames)
        n_acc = sum(1 for d, r in dec if not r)
        res = {}
        for mode in ("bf16", "fp32"):
            wm = w if mode == "bf16" else replace(w, dtype="fp32")
            c = make(wm, [n_acc + 1])
            fr = [[x.to(dev) for x in frame_qkv(wm, 0, 0, i)] for i in range(4)]
            out = torch.empty((w.Nq, w.H, w.D), dtype=torch.float32 if mode == "fp32" else torch.bfloat16,
                              device=dev)
            timed = range(w.frames) if mode == "bf16" else range(w.frames - 20, w.frames)
            flops = 0.0
            a, b = ev(), ev()
            for t, (deferred, rejected) in enumerate(dec):
                q, k, v = fr[t % 4]
                c.set_defer_eviction(deferred)
                c.append_frame(0, k, v)
                c.evict_frames()
                if t == timed[0]:
                    torch.cuda.synchronize()
                    a.record()
                if t in timed:
                    c.build_visible_page_table()
                    c.plan([w.Nq])
                    c.run(0, q, out=out, force_fp32=(mode == "fp32"))
                    flops += flops_of(w.Nq, c.plan_info()["kv_tokens"][0], w.H, w.D)
                if deferred:
                    (c.rollback_last_frame if rejected else c.execute_deferred_eviction)()
            b.record()
            torch.cuda.synchronize()
            ms = a.elapsed_time(b)
            res[mode] = {"frames": len(timed), "frames_per_s": len(timed) / (ms / 1e3),
                         "tflops": flops / (ms / 1e3) / 1e12}
        line.update(metric="frames/s over the 10,000-frame stream with rollbacks",
                    value=res["bf16"]["frames_per_s"], unit="frames/s", modes=res,
                    accepted_frames=n_acc)
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------- CPU oracle
def oracle_block_frame_seconds(w, t_frames, rows=None, heads=None):
    """Times the oracle on one block at a cache holding t_frames frames."""
    import numpy as np
    import torch

    from oracle import FrameStream, attend, rope2d
    from streaming_video_transformer_b200.inputs import frame_qkv

    st = FrameStream(w.P, w.ns, w.S, w.W)
    data = []
    for i in range(w.R):
        q, k, v = frame_qkv(w, 0, 0, i)
        qr = torch.from_numpy(rope2d(q, w.ns, w.rope_grid, w.rope_theta)).to(q.dtype)
        kr = torch.from_numpy(rope2d(k, w.ns, w.rope_grid, w.rope_theta)).to(k.dtype)
        data.append(tuple(x.double().numpy() for x in (qr, kr, v)))
    for t in range(t_frames):
        st.append_frame(data[t % w.R][1], data[t % w.R][2])
    q = data[(t_frames - 1) % w.R][0]
    if rows is not None:
        q = q[rows]
    t0 = time.perf_counter()
    k, v = st.visible_kv()
    if heads is not None:
        k, v, q = k[:, heads], v[:, heads], q[:, heads]
    attend(q, k, v)
    return time.perf_counter() - t0


def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def oracle_vitl_step_one_thread_seconds():
    """The oracle on the single ViT-L step (cache pre-filled with 200 frames,
    one 1375-row frame attends over 99,768 tokens) with its BLAS limited to
    one thread.  One head of the sixteen is timed (gather of that head's
    visible K/V and its attention); the step time is 16 x that."""
    import torch
    from threadpoolctl import threadpool_limits

    from oracle import FrameStream, attend
    from streaming_video_transformer_b200.inputs import WORKLOADS, frame_qkv

    w = WORKLOADS["vitl_step"]
    data = [tuple(x.double().numpy() for x in frame_qkv(w, 0, 0, i)) for i in range(w.R)]
    st = FrameStream(w.P, w.ns, w.S, w.W)
    for t in range(w.frames):
        st.append_frame(data[t % w.R][1], data[t % w.R][2])
    q = data[(w.frames - 1) % w.R][0]
    with threadpool_limits(limits=1), torch.autograd.no_grad():
        torch_threads = torch.get_num_threads()
        torch.set_num_threads(1)
        try:
            t0 = time.perf_counter()
            k, v = st.visible_kv(heads=slice(0, 1))
            attend(q[:, 0:1], k, v)
            secs = time.perf_counter() - t0
        finally:
            torch.set_num_threads(torch_threads)
    return w.H * secs, st.num_visible_tokens()


def run_reference(args):
    """The CPU oracle as it stands, on the same workload: each step streams
    one frame into the oracle's cache and computes attention for a sample of
    the frame's query rows of one head of one block."""
    import numpy as np
    import torch
    from dataclasses import replace

    from oracle import FrameStream, attend, rope2d
    from streaming_video_transformer_b200.inputs import WORKLOADS, frame_qkv

    w = replace(WORKLOADS[WORKLOAD], R=4)
    data = []
    for i in range(w.R):
        q, k, v = frame_qkv(w, 0, 0, i)
        qr = torch.from_numpy(rope2d(q, w.ns, w.rope_grid, w.rope_theta)).to(q.dtype)
        kr = torch.from_numpy(rope2d(k, w.ns, w.rope_grid, w.rope_theta)).to(k.dtype)
        data.append(tuple(x.double().numpy() for x in (qr, kr, v)))
    st = FrameStream(w.P, w.ns, w.S, w.W)
    prefill = prefill_frames(WORKLOAD, args.warmup, args.steps)   # the GPU arm's frames
    for t in range(prefill):
        st.append_frame(data[t % w.R][1], data[t % w.R][2])
    budget_s = 150.0          # whole run, so that the default K/W end within a few minutes
    n_steps = args.warmup + args.steps
    rows_n = 64
    rng = np.random.default_rng(0)
    per_frame = []
    t_frame = prefill
    for i in range(n_steps):
        t_frame += 1
        q, k, v = data[(t_frame - 1) % w.R]
        st.append_frame(k, v)
        h = i % w.H
        t0 = time.perf_counter()
        kh, vh = st.visible_kv(heads=slice(h, h + 1))
        t1 = time.perf_counter()
        rows = np.sort(rng.choice(w.Nq, size=rows_n, replace=False))
        attend(q[rows][:, h:h + 1], kh, vh)
        t2 = time.perf_counter()
        # one frame = 24 blocks x 16 heads x (gather of one head + attention of all rows)
        frame_s = w.blocks * w.H * ((t1 - t0) + (t2 - t1) * (w.Nq / rows_n))
        if i >= args.warmup:
            per_frame.append(frame_s)
        if i == 0:   # size the row sample so the whole run stays within the budget
            per_step = max(1e-3, budget_s / max(1, n_steps))
            rows_n = int(max(1, min(w.Nq, rows_n * max(0.02, (per_step - (t1 - t0)) /
                                                       max(t2 - t1, 1e-4)))))
    mean_frame = sum(per_frame) / max(1, len(per_frame))
    fps = 1.0 / mean_frame
    flops = w.blocks * 4.0 * w.Nq * _visible(t_frame, w) * w.H * w.D
    return {
        "impl": "reference", "metric": METRIC, "value": fps, "unit": "frames/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * mean_frame, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config(w, {"frames": f"pre-filled 0..{prefill - 1}, warm-up to "
                                        f"{prefill + args.warmup - 1}, timed "
                                        f"{prefill + args.warmup}..{t_frame - 1}"}),
        "tflops": flops / mean_frame / 1e12,
        "cpu_baseline": {"value": fps, "unit": "frames/s", "cores": cpu_threads(),
                         "kind": "oracle",
                         "sample": f"per step: stream one frame into the oracle, gather one "
                                   f"head's visible K/V, attention for {rows_n} sampled query rows "
                                   f"of that head; frame time = 24 blocks x 16 heads x (gather + "
                                   f"1375/{rows_n} x sampled attention)"},
        "e2e": {"value": fps, "unit": "frames/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=925)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="svt", choices=["svt", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-path", default="graph", choices=["graph", "calls"],
                    help="end-to-end leg: svt_frame_step with CUDA-graph replay, or the separate "
                         "calls of the device-resident leg")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(PREFILL) + list(SECONDARY),
                    help="vitl_step (1 block, no RoPE) is the small case used for profiling; "
                         "tiny_stream, ragged4, rollback10k, first_pass8, skip_append and "
                         "nocross_step print their own metric")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if args.workload in SECONDARY:
        from streaming_video_transformer_b200.build import build
        build()
        run_secondary(args)
        return

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    from streaming_video_transformer_b200.build import build
    if rank == 0:
        build()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    r = run_gpu(args, rank, world, local_rank)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return
    w = r["w"]
    burst, sustained, hbm, peak_kind = _peaks()
    fps = whole_job_rate(world, args.steps, r["elapsed_ms"])
    tflops = r["total_flops"] / (r["elapsed_ms"] / 1e3) / 1e12
    run_avg_ms = sum(r["run_ms"]) / len(r["run_ms"])
    run_flops = sum(r["flops_per_block"]) / len(r["flops_per_block"])
    achieved = run_flops / (run_avg_ms / 1e3) / 1e12
    traffic = None
    if ATTN_TRAFFIC_BYTES:
        keys = [_visible(t + 1, w) for t in range(r["first_timed"], r["last_timed"])]
        traffic = ATTN_TRAFFIC_BYTES * (sum(keys) / len(keys)) / ATTN_TRAFFIC_KEYS
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        try:
            secs = oracle_block_frame_seconds(w, r["last_timed"])
            cpu = {"value": 1.0 / (w.blocks * secs), "unit": "frames/s", "cores": cpu_threads(),
                   "kind": "oracle", "cpu_model": cpu_model(),
                   "sample": f"one of 24 blocks at frame t={r['last_timed']} (all 1375 query rows, "
                             f"16 heads, {_visible(r['last_timed'], w)} visible tokens); "
                             f"{secs:.1f} s x 24 blocks per frame"}
            s1, nk = oracle_vitl_step_one_thread_seconds()
            cpu["one_thread_vitl_step"] = {
                "seconds_per_step": s1, "cores": 1,
                "tflops": 4.0 * 1375 * nk * 16 * 64 / s1 / 1e12,
                "sample": f"single ViT-L step (1375 query rows over {nk} visible tokens), BLAS "
                          f"limited to one thread; one head of 16 timed, x16"}
        except Exception as exc:  # the CPU leg never blocks the GPU number
            cpu = {"value": None, "unit": "frames/s", "cores": cpu_threads(), "kind": "oracle",
                   "sample": f"failed: {exc!r}"}
    e2e_fps = whole_job_rate(world, r["e2e_steps"], r["e2e_ms"])
    line = {
        "metric": METRIC, "value": fps, "unit": "frames/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["elapsed_ms"] / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": _config(w, {"frames": f"pre-filled 0..{r['first_timed'] - args.warmup - 1}, "
                                        f"warm-up to {r['first_timed'] - 1}, timed "
                                        f"{r['first_timed']}..{r['last_timed'] - 1}",
                              "splits": r["info"]["splits"][0],
                              "work_items": r["info"]["num_items"]}),
        "tflops": tflops,
        "tflops_frac_of_peak": {"burst": tflops / burst, "sustained": tflops / sustained,
                                "peak_kind": peak_kind},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": burst,
                     "unit": "TFLOP/s", "frac": achieved / burst, "traffic": traffic,
                     "kernel": "svt_run (RoPE on Q + tcgen05 attention + split merge), block 0 "
                               "of every timed frame, CUDA events on the launch stream",
                     "peak_kind": f"dense bf16 burst ({peak_kind}): each launch is timed on its "
                                  f"own at the running clock",
                     "frac_of_sustained": achieved / sustained},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_fps, "unit": "frames/s", "h2d_bytes_per_step": r["h2d_per_step"],
                "d2h_bytes_per_step": r["d2h_per_step"], "steps": r["e2e_steps"],
                "path": args.e2e_path,
                "note": f"Q/K/V of all {w.blocks} blocks copied from pinned host memory and the "
                        f"outputs of all {w.blocks} blocks copied back to pinned host memory every "
                        "frame, on two copy streams (double-buffered by frame parity); frame step "
                        + ("through svt_frame_step with CUDA-graph replay" if args.e2e_path == "graph"
                           else "through the separate calls")},
        "gpu_launches": r["kernels_per_step"] * args.steps,
        "clocks": r["clocks"],
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
