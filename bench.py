"""Throughput of the KDA + modality-aware short-conv forward pass on B200.

One step = one `kda_fwd` call through the C ABI (short conv on q, k, v, then the
chunked KDA scan) over one batch of the synthetic workload, inputs resident in
HBM.  Default workload: the 30-second 480x832 video (512 text tokens + a
121x30x52 latent grid = 189,272 tokens, H=16, d=128, bf16), whose inputs
(4.66 GB) are far larger than the 126 MB L2, so no flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Prints one JSON line (rank 0).  Under torchrun every rank runs its own copy of
the workload (weak scaling, no collective on the data path); the value is the
tokens of all ranks divided by the slowest rank's device time.

  python bench.py --shard seq [--seq-ranks R]        (torchrun for N > 1)

times the sequence-sharded pass instead: the workload's frames split over the
ranks (conv halo exchange, per-rank state maps composed across ranks), total
work fixed (strong scaling).  On one GPU, --seq-ranks R runs R ranks as threads.
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

import kda_synth  # noqa: E402

METRIC = "KDA+shortconv fwd tokens/sec on 1 B200 (30 s video); % of roofline"
DEFAULT_WORKLOAD = "video_30s_480x832"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


def workload_by_name(name):
    for i, w in enumerate(kda_synth.WORKLOADS):
        if w.name == name:
            return i, w
    raise SystemExit(f"unknown workload {name}; choose from {[w.name for w in kda_synth.WORKLOADS]}")


def algorithmic_bytes(w):
    """Bytes the fused path must move once: q, k, v, beta and o in the storage
    dtype, log alpha in fp32 (weights and states are negligible)."""
    e = 2 if w.dtype == "bf16" else 4
    per_tok = 3 * w.H * w.d * e + w.H * w.d * 4 + w.H * e + w.H * w.d * e
    return per_tok * w.tokens


def conv_bytes(w):
    e = 2 if w.dtype == "bf16" else 4
    return 2 * 3 * w.H * w.d * e * w.tokens


def tensor_flops(w):
    """Algorithmic tensor-core flops of the chunked scan: H*(6 d^2 + 5 C d) per token."""
    return w.H * (6 * w.d * w.d + 5 * w.chunk * w.d) * w.tokens


# ---------------------------------------------------------------------------
# clock sampling during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.gpu_index)], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
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
        rows = []
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        finally:
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        hi = max(sm) if sm else 0
        loaded = [s for s in sm if s >= 0.5 * hi] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# CPU oracle baseline (a bounded sample of the same workload)
# ---------------------------------------------------------------------------
def oracle_sample_workload(w, frames):
    """The workload cut to its first `frames` frames (same shapes otherwise)."""
    import dataclasses
    T, Hg, Wg = w.grid
    return dataclasses.replace(w, grid=(min(frames, T), Hg, Wg), B=1)


def run_oracle_sample(w, idx, frames, heads, causal_t=False):
    import oracle
    ws = oracle_sample_workload(w, frames)
    inp = kda_synth.generate(ws, kda_synth.seed_for(idx))
    oracle.build()
    t0 = time.perf_counter()
    oracle.forward(inp, ws.text_len, ws.grid, heads=list(range(heads)), vis_causal_t=causal_t)
    dt = time.perf_counter() - t0
    # throughput in full-width tokens: the sample covers `heads` of H heads
    tokens_equiv = ws.N * heads / w.H
    sample = (f"oracle (fp64 conv + token recurrence) on 1 batch item, heads 0..{heads - 1} of {w.H}, "
              f"first {ws.grid[0]} of {w.grid[0]} frames ({ws.N} tokens)")
    return tokens_equiv / dt, dt, sample


def sample_frames(w):
    """All frames of the workload (the sample is bounded by the head count)."""
    return w.grid[0]


def run_config(args, w, world):
    """The `config` object of both arms' JSON lines (same keys, so the two lines compare)."""
    return {"workload": w.name, "B": w.B, "N": w.N, "H": w.H, "d": w.d, "text_len": w.text_len,
            "vis_conv_t": "causal" if args.causal_t else "centred", "grid": list(w.grid), "chunk": w.chunk,
            "parallelism": f"replicas{world}", "l2": "inputs larger than L2 (no flush)"}


def reference_arm(args, w, idx, rank, world):
    """The CPU oracle as it stands, on the same head sample as the GPU arm's cpu_baseline."""
    cores = os.cpu_count()
    if rank != 0:
        return
    frames = sample_frames(w) if w.grid[0] > 1 else 1
    vals, secs = [], []
    for i in range(args.warmup + args.steps):
        v, dt, sample = run_oracle_sample(w, idx, frames, args.cpu_heads, args.causal_t)
        if i >= args.warmup:
            vals.append(v)
            secs.append(dt)
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        # measured wall time of one sampled step; the whole workload would take extrapolated_ms_per_step
        "ms_per_step": 1e3 * statistics.mean(secs), "extrapolated_ms_per_step": 1e3 * w.tokens / value,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": run_config(args, w, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def time_calls(fn, steps, stream):
    import torch
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(steps):
        fn()
    ev1.record(stream)
    torch.cuda.synchronize()
    return ev0.elapsed_time(ev1) / steps


def reduce_max(value: float, device, world: int) -> float:
    """The largest of the ranks' values (every rank gets it); the identity on one rank."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def seq_arm(args, w, idx, rank, world, local_rank):
    """Sequence-sharded pass: rank r owns an even share of the frames (rank 0 the text too)."""
    import torch
    import linear_attention_video_b200 as kda
    from linear_attention_video_b200 import seqshard
    from tests._util import to_device

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream(dev)
    ranks = world if world > 1 else max(1, args.seq_ranks)
    segs = seqshard.partition(w.text_len, w.grid, ranks, args.causal_t)
    mine = [rank] if world > 1 else list(range(ranks))
    inp = kda_synth.generate(w, kda_synth.seed_for(idx))
    B, N, H, d = inp["shape"]
    full = to_device(inp, "cpu")
    host = {}
    for r in mine:
        sg = segs[r]
        host[r] = {n: full[n][:, sg.t0:sg.t1].contiguous().pin_memory() for n in ("q", "k", "v", "log_alpha", "beta")}
    weights = {n: full[n].to(dev) for n in ("w_text", "w_vis")}
    dev_in = {r: {n: x.to(dev) for n, x in host[r].items()} for r in mine}
    backends = {r: seqshard.GpuBackend(B, H, d, w.chunk, args.causal_t) for r in mine}
    outs = {}

    def rank_step(comm, src):
        r = comm.rank
        x = src[r]
        outs[r] = seqshard.seqshard_fwd(backends[r], comm, (x["q"], x["k"], x["v"]), x["log_alpha"], x["beta"],
                                        weights["w_text"], weights["w_vis"], w.text_len, w.grid)

    if world > 1:
        comm = seqshard.DistComm()
        step = lambda src=dev_in: rank_step(comm, src)   # noqa: E731
    else:
        group = seqshard.LocalGroup(ranks)
        step = lambda src=dev_in: group.run(lambda c: rank_step(c, src))   # noqa: E731

    with ClockSampler(local_rank) as clk:
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()
        ms = time_calls(step, args.steps, stream)
    clocks = clk.summary()
    ms = reduce_max(ms, dev, world)
    value = w.tokens / (ms * 1e-3)

    # end to end: this rank's inputs from pinned host memory, the pass, its outputs back
    e2e = None
    if not args.no_e2e:
        o_host = {r: torch.empty((B, segs[r].t1 - segs[r].t0, H, d), dtype=dev_in[r]["q"].dtype).pin_memory()
                  for r in mine}
        h2d = sum(x.numel() * x.element_size() for r in mine for x in host[r].values())
        d2h = sum(x.numel() * x.element_size() for x in o_host.values())

        def e2e_step():
            for r in mine:
                for n in host[r]:
                    dev_in[r][n].copy_(host[r][n], non_blocking=True)
            step()
            for r in mine:
                o_host[r].copy_(outs[r][0], non_blocking=True)
        e2e_step()
        ms_e2e = reduce_max(time_calls(e2e_step, max(3, min(args.steps, 10)), stream), dev, world)
        e2e = {"value": w.tokens / (ms_e2e * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h}
    # launches per step on this process: conv (text + visual) and three scans per rank
    # kernels one step launches on this process (every rank's backend counts its own)
    for be in backends.values():
        be.launches = 0
    step()
    torch.cuda.synchronize()
    launches = sum(be.launches for be in backends.values())
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "f16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "N": w.N, "H": w.H, "d": w.d, "text_len": w.text_len,
                       "vis_conv_t": "causal" if args.causal_t else "centred", "grid": list(w.grid),
                       "chunk": w.chunk, "parallelism": f"sequence{ranks}" + ("" if world > 1 else " (threads on 1 GPU)"),
                       "l2": "inputs larger than L2 (no flush)"},
            "e2e": e2e, "gpu_launches": launches * args.steps, "clocks": clocks,
        }
        print(json.dumps(line), flush=True)


def bwd_bytes(w):
    """Bytes the backward pass must move once: q, k, v, beta, d_o read and dq, dk, dv, dbeta written in
    the storage dtype, log alpha read and its gradient written in fp32."""
    e = 2 if w.dtype == "bf16" else 4
    per_tok = w.H * w.d * (7 * e + 8) + 2 * w.H * e
    return w.B * w.N * per_tok


def bwd_arm(args, w, idx, rank, world, local_rank):
    """One step = one kda_bwd call (gradients of the whole forward) over the workload."""
    import torch
    import linear_attention_video_b200 as kda
    from tests._util import to_device

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream(dev)
    peaks = load_peaks()
    inp = kda_synth.generate(w, kda_synth.seed_for(idx))
    B, N, H, d = inp["shape"]
    t = to_device(inp, dev)
    dt = t["q"].dtype
    p = kda.problem(B, H, d, w.text_len, w.grid, chunk=w.chunk, vis_causal_t=args.causal_t)
    gen = torch.Generator(device=dev).manual_seed(kda_synth.seed_for(idx))
    d_o = torch.randn(B, N, H, d, device=dev, generator=gen).to(dt)
    g = [torch.empty(B, N, H, d, dtype=dt, device=dev) for _ in range(3)]
    dla = torch.empty(B, N, H, d, dtype=torch.float32, device=dev)
    dbeta = torch.empty(B, N, H, dtype=dt, device=dev)
    dwt = torch.empty(3, H * d, w.text_k, device=dev)
    dwv = torch.empty(3, H * d, 27, device=dev)
    ws = kda.alloc_bwd_workspace(p, dt, dev)

    def step():
        kda.kda_bwd(p, t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], t["w_text"], t["w_vis"], d_o, *g, dla,
                    dbeta, dwt, dwv, ws, stream=stream)
    with ClockSampler(local_rank) as clk:
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        launches = kda.kda_last_launch_count()
        ms = time_calls(step, args.steps, stream)
    ms = reduce_max(ms, dev, world)
    hbm = float(peaks["hbm_gbs"])
    achieved = bwd_bytes(w) / (ms * 1e-3) / 1e9
    if rank == 0:
        print(json.dumps({
            "metric": "KDA+shortconv bwd tokens/sec on 1 B200", "value": w.tokens * world / (ms * 1e-3),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "tf32 per-chunk products, fp16 chain operands, f32 accumulation, bf16 storage"
            if w.dtype == "bf16" else "f32 (split-tf32 tensor products)", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "N": w.N, "H": w.H, "d": w.d, "text_len": w.text_len,
                       "grid": list(w.grid), "pass": "backward", "parallelism": f"replicas{world}",
                       "l2": "inputs larger than L2 (no flush)"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                         "traffic": None, "kernel": "kda_bwd (all its kernels)",
                         "peak_source": peaks["source"] + " hbm_gbs"},
            "e2e": None, "gpu_launches": launches * args.steps, "clocks": clk.summary(),
        }), flush=True)


def ours_arm(args, w, idx, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import linear_attention_video_b200 as kda
    from tests._util import to_device

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream(dev)
    peaks = load_peaks()

    inp = kda_synth.generate(w, kda_synth.seed_for(idx))
    B, N, H, d = inp["shape"]
    t = to_device(inp, dev)
    dt = t["q"].dtype
    p = kda.problem(B, H, d, w.text_len, w.grid, chunk=w.chunk, vis_causal_t=args.causal_t)
    o = torch.empty(B, N, H, d, dtype=dt, device=dev)
    ws = kda.alloc_workspace(p, dt, dev)

    def step():
        kda.kda_fwd(p, t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], t["w_text"], t["w_vis"], o, ws,
                    stream=stream)

    # the clock sampler runs from the warm-up through the timed region (its period is 200 ms)
    with ClockSampler(local_rank) as clk:
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        st = kda.kda_read_status(ws, stream)
        if st != kda.KDA_OK:
            raise SystemExit(f"device status after warm-up: {kda.kda_status_str(st)}")
        launches_per_step = kda.kda_last_launch_count()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        ms = time_calls(step, args.steps, stream)
    clocks = clk.summary()
    ms = reduce_max(ms, dev, world)
    tokens_all = w.tokens * world
    value = tokens_all / (ms * 1e-3)

    # per-kernel timings: the step's own kernels, launched through the single-op entry points (for
    # bf16 problems the step passes fp16 activations from the conv to the scan: KDA_FLAG_QKV_F16)
    f16 = dt == torch.bfloat16
    p1 = kda.problem(B, H, d, w.text_len, w.grid, chunk=w.chunk, vis_causal_t=args.causal_t, qkv_f16=f16)
    conv_out = [torch.empty(t["q"].shape, dtype=torch.float16 if f16 else dt, device=dev) for _ in range(3)]

    def conv_step():
        kda.kda_shortconv_fwd(p1, t["q"], t["k"], t["v"], t["w_text"], t["w_vis"], *conv_out, stream=stream)

    def scan_step():
        kda.kda_chunk_fwd(p1, conv_out[0], conv_out[1], conv_out[2], t["log_alpha"], t["beta"], o, ws,
                          stream=stream)
    # each entry point gets its own warm-up, so neither timing includes module loading
    for _ in range(max(3, args.warmup)):
        conv_step()
        scan_step()
    ms_conv = time_calls(conv_step, args.steps, stream)
    ms_scan = time_calls(scan_step, args.steps, stream)
    del conv_out

    scan_bytes = algorithmic_bytes(w)
    scan_gbs = scan_bytes / (ms_scan * 1e-3) / 1e9
    conv_gbs = conv_bytes(w) / (ms_conv * 1e-3) / 1e9
    hbm = float(peaks["hbm_gbs"])
    # the scan entry point (one launch: record and state-pass CTAs) is the dominant launch; its
    # algorithmic bytes are those of the fused step: q', k', v', log alpha, beta read once, o written once
    dominant = "kda_chunk" if ms_scan >= ms_conv else "shortconv"
    achieved = scan_gbs if dominant == "kda_chunk" else conv_gbs
    traffic = None
    prof = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(prof):
        try:
            traffic = json.load(open(prof)).get(dominant, {}).get(w.name)
        except (ValueError, OSError):
            traffic = None
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "traffic": traffic, "kernel": dominant + (" (kda_chunk_fwd: kda_tc_prep, record and state-pass CTAs)"
                                                          if dominant == "kda_chunk" else ""),
                "peak_source": peaks["source"] + " hbm_gbs"}
    step_roof_ms = max(algorithmic_bytes(w) / (hbm * 1e9), tensor_flops(w) / (float(peaks["bf16_tflops"]) * 1e12)) * 1e3

    # end to end through the public API for host-resident data: kda_fwd_host copies the pinned host
    # inputs in and o out segment by segment, overlapped with the kernels (the conv weights are
    # model parameters, resident on the device)
    e2e = None
    if not args.no_e2e:
        host = {k2: v.cpu().pin_memory() for k2, v in t.items() if k2 not in ("w_text", "w_vis")}
        o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = o_host.numel() * o_host.element_size()
        ws_host = kda.alloc_fwd_host_workspace(p, o.dtype, args.seg_frames, dev)
        cin, cout = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def e2e_step():
            kda.kda_fwd_host(p, host["q"], host["k"], host["v"], host["log_alpha"], host["beta"], t["w_text"],
                             t["w_vis"], o_host, ws_host, args.seg_frames, stream=stream, copy_in_stream=cin,
                             copy_out_stream=cout)
        e2e_step()
        e2e_steps = max(3, min(args.steps, 10))
        ms_e2e = time_calls(e2e_step, e2e_steps, stream)
        ms_e2e = reduce_max(ms_e2e, dev, world)
        e2e = {"value": tokens_all / (ms_e2e * 1e-3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "api": "kda_fwd_host",
               "seg_frames": args.seg_frames}
        del host, ws_host

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        frames = sample_frames(w)
        v, secs, sample = run_oracle_sample(w, idx, frames, args.cpu_heads, args.causal_t)
        cpu = {"value": v, "unit": "tokens/s", "cores": os.cpu_count(), "kind": "oracle", "sample": sample,
               "seconds": secs}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": run_config(args, w, world),
            "roofline": roofline,
            "roofline_step": {"time_ms": step_roof_ms, "frac": step_roof_ms / ms,
                              "bytes": algorithmic_bytes(w), "tensor_flops": tensor_flops(w)},
            "kernels_ms": {"shortconv": ms_conv, "kda_chunk": ms_scan},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)


def mixer_arm(args, rank, world, local_rank):
    """KDA/MLA 3:1 against MHA/MLA 3:1 token-mixer stacks as N grows (synthetic weights, one GPU
    per rank, every rank the same sweep): forward latency and peak memory per stack."""
    import torch
    from linear_attention_video_b200 import mixer
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    H, d, text_len, Hg, Wg = 16, 128, 512, 30, 52   # the 480x832 video layout, 16 heads of 128
    frames = [int(f) for f in args.mixer_frames.split(",")]
    stream = torch.cuda.current_stream(dev)
    rows = []
    with ClockSampler(local_rank) as clk:
        for T in frames:
            N = text_len + T * Hg * Wg
            row = {"frames": T, "tokens": N}
            for kind in ("kda", "mha"):
                torch.cuda.empty_cache()
                torch.cuda.reset_peak_memory_stats(dev)
                try:
                    layers = mixer.stack(kind, 1, H, d, text_len, (T, Hg, Wg), dev)
                    x = torch.randn(1, N, H * d, generator=torch.Generator().manual_seed(T)).to(dev, torch.bfloat16)

                    def step():
                        mixer.run_stack(layers, x)
                    for _ in range(args.warmup):
                        step()
                    ms = time_calls(step, args.steps, stream)
                    row[kind + "_ms"] = reduce_max(ms, dev, world)
                    row[kind + "_peak_gb"] = torch.cuda.max_memory_allocated(dev) / 1e9
                    del layers, x
                except torch.cuda.OutOfMemoryError:
                    row[kind + "_ms"] = None
                    row[kind + "_peak_gb"] = "oom"
            if row.get("kda_ms") and row.get("mha_ms"):
                row["speedup"] = row["mha_ms"] / row["kda_ms"]
            rows.append(row)
    clocks = clk.summary()
    if rank == 0:
        last = rows[-1]
        line = {"metric": "KDA/MLA 3:1 vs MHA/MLA 3:1 token-mixer stack forward latency, 1 B200",
                "value": last.get("speedup"), "unit": "x (MHA/MLA time / KDA/MLA time at the largest N)",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": "mixer_sweep_480x832", "B": 1, "H": H, "d": d, "text_len": text_len,
                           "grid_hw": [Hg, Wg], "layers": "4 per stack (3 KDA or MHA, 1 MLA), residual",
                           "mla": {"d_latent": mixer.D_LATENT, "d_nope": mixer.D_NOPE, "d_direct": mixer.D_DIRECT},
                           "parallelism": f"replicas{world}"},
                "sweep": rows, "clocks": clocks}
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--seg-frames", type=int, default=8, help="frames per segment of the e2e (host-buffer) call")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-heads", type=int, default=2,
                    help="heads in the CPU-oracle sample (the cpu_baseline and the reference arm)")
    ap.add_argument("--pass", dest="which", default="fwd", choices=["fwd", "bwd"],
                    help="bwd: time the backward pass (kda_bwd) instead of the forward")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "seq"],
                    help="replicas: every rank runs the whole workload; seq: the frames are split over the ranks")
    ap.add_argument("--seq-ranks", type=int, default=2, help="--shard seq on one GPU: ranks run as threads")
    ap.add_argument("--causal-t", action="store_true",
                    help="temporal taps of the 3D conv cover frames t-2..t instead of t-1..t+1")
    ap.add_argument("--mixer", action="store_true",
                    help="time KDA/MLA 3:1 against MHA/MLA 3:1 token-mixer stacks as N grows")
    ap.add_argument("--mixer-frames", default="20,40,80,121,163",
                    help="visual frames of the --mixer sweep (N = 512 + frames x 30 x 52)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    idx, w = workload_by_name(args.workload)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        reference_arm(args, w, idx, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        if args.mixer:
            mixer_arm(args, rank, world, local_rank)
            return
        arm = bwd_arm if args.which == "bwd" else (seq_arm if args.shard == "seq" else ours_arm)
        arm(args, w, idx, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
