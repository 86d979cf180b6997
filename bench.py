#!/usr/bin/env python3
"""Benchmark of one denoising step of block discrete-diffusion decoding.

A step = canvas attention over [prefix KV || canvas KV] (tcgen05 kernel +
split merge) followed by the vocabulary-wide sampler and re-noise (chunk
pass + row merge): every step of the hot path, through the C ABI
(dd_canvas_attn, dd_sample_renoise).  Default workload (`ragged_b8`, the
largest single-GPU configuration): a ragged batch of 8 canvases, 16 query /
8 kv heads, head_dim 128, prefix lengths drawn from [512, 16384], canvas
256, vocabulary 262144 (2048 x 262144 bf16 logits per step), bf16.  The
batch-1 step is `--workload b1_L4096`.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
  python bench.py --workload block12_L8192   # + the 12-step block loop: eager,
                                             #   replayed graph, E4M3 inputs
  python bench.py --policy       # the pages' adaptive block, eager and on-device loop
  python bench.py --attn-e4m3 [--workload W]  # attention on 8-bit inputs beside bf16
  python bench.py --soft-embed   # the self-conditioning soft embedding

Prints ONE JSON line (rank 0).  `value` is canvas-steps/s over all ranks
(each rank runs its own independent canvases: no collective on the data
path), from CUDA events on the launch stream, max over ranks.  Inputs are
rotated among 3 sets, each larger than the 126 MB L2 (1.35 GB for
ragged_b8, 152 MB for b1_L4096), so no step reads the previous step's
inputs from L2.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "denoise steps/s per 256-token canvas"
UNIT = "canvas-steps/s"
# Nominal denominators, reported beside the measured ones: the benchmark spec's
# ~8 TB/s of HBM3e and the 2.25 PFLOP/s dense bf16 datasheet figure.
NOMINAL_HBM_GBS = 8000.0
NOMINAL_BF16_TFLOPS = 2250.0
N_SETS = 3


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), \
            "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi samples every 100 ms in a background thread."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.samples = []
        self.proc = None
        self.gpu = gpu_index
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [x.strip() for x in line.split(",")]))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        sel = [s for t, s in self.samples if t0 <= t <= t1] or [s for _, s in self.samples[-3:]]
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(s[0]) for s in sel if s[0].replace(".", "").isdigit()]
        mx = [float(s[1]) for s in sel if s[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for s in sel for n, v in zip(names, s[4:8]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(sel)}


def _dist():
    """One process per GPU (NCCL; gloo when no GPU is visible, which the CPU
    tests of the multi-rank plumbing use).  Replicas only: the process group
    carries the barrier and the max-over-ranks timing, no data."""
    n = int(os.environ.get("WORLD_SIZE", "1"))
    if n > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        return dist, dist.get_rank(), n, int(os.environ.get("LOCAL_RANK", "0"))
    return None, 0, 1, 0


def _max_over_ranks(dist, x: float) -> float:
    if dist is None:
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(dist):
    if dist is not None:
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def make_inputs(w, rank: int, dev):
    """N_SETS independent input sets on the device (seeded per rank and set)."""
    sets = []
    for s in range(N_SETS):
        ws = workloads.scaled(w, seed=w.seed + 1000 * rank + s)
        q, kc, vc = workloads.canvas_qkv(ws, 0, device=dev)
        kp, vp, cu = workloads.prefix_kv(ws, device=dev)
        lg = workloads.logits(ws, 0, device=dev)
        sets.append({"q": q, "kc": kc, "vc": vc, "kp": kp, "vp": vp, "cu": cu.to(dev),
                     "cu_host": cu.numpy(), "logits": lg})
    return sets


def run_ours(args, w, dist, rank, world, local_rank):
    import block_discrete_diffusion_dd_b200 as dd

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    sets = make_inputs(w, rank, dev)
    R, V = w.rows, w.vocab
    desc = dd.attn_desc(sets[0]["q"], sets[0]["kc"], w.scale)
    ws_attn = dd.new_workspace(dd.canvas_attn_workspace_bytes(desc, sets[0]["cu_host"]), dev)
    ws_samp = dd.new_workspace(dd.sample_workspace_bytes(R, V, w.torch_dtype), dev)
    attn_out = torch.empty_like(sets[0]["q"])
    outs = {"tokens": torch.empty(R, dtype=torch.int32, device=dev),
            "pred": None, "entropy": torch.empty(R, dtype=torch.float32, device=dev),
            "conf": torch.empty(R, dtype=torch.float32, device=dev),
            "renoised": torch.empty(R, dtype=torch.uint8, device=dev)}
    rate, tau = w.rates[0], w.temperatures[0]

    def attn(i):
        s = sets[i % N_SETS]
        dd.canvas_attn(s["q"], s["kc"], s["vc"], s["kp"], s["vp"], s["cu"], s["cu_host"],
                       scale=w.scale, out=attn_out, workspace=ws_attn)

    def samp(i):
        s = sets[i % N_SETS]
        dd.sample_renoise(s["logits"], tau, rate, w.seed + rank, i, row_offset=0, outputs=outs,
                          workspace=ws_samp)

    def step(i):
        attn(i)
        samp(i)

    # eager warm-up (first calls set kernel attributes), then CUDA graphs
    # per input set: the whole step, and the whole step with timing events
    # between the attention and the sampler calls
    for i in range(N_SETS):
        step(i)
    dd.query_device_error(ws_attn)
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(stream)
    graphs, timed = [], []
    with torch.cuda.stream(side):
        for i in range(N_SETS):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                step(i)
            graphs.append(g)
            ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)]
            g2 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g2, stream=side):
                ev[0].record()
                attn(i)
                ev[1].record()
                samp(i)
                ev[2].record()
            timed.append((g2, ev))
    launches_per_step = _launches_per_step(dd, step)
    stream.wait_stream(side)
    for i in range(args.warmup):
        graphs[i % N_SETS].replay()
    torch.cuda.synchronize()

    clocks = ClockSampler(local_rank if world > 1 else torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    # the whole-job number: K steps between one event pair
    _barrier(dist)
    t_wall0 = time.time()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        graphs[i % N_SETS].replay()
    e1.record(stream)
    _barrier(dist)
    t_wall1 = time.time()
    launches = launches_per_step * args.steps
    ms_total = _max_over_ranks(dist, e0.elapsed_time(e1))
    # per-kernel durations inside whole steps (events between the calls)
    n2 = max(N_SETS, min(args.steps, 300))
    ta, ts = [], []
    for i in range(n2):
        g2, ev = timed[i % N_SETS]
        g2.replay()
        torch.cuda.synchronize()
        ta.append(ev[0].elapsed_time(ev[1]))
        ts.append(ev[1].elapsed_time(ev[2]))
    per = {"attn": _max_over_ranks(dist, statistics.mean(ta) / 1e3),
           "samp": _max_over_ranks(dist, statistics.mean(ts) / 1e3)}
    # warm: the same input set replayed back to back (what stays in L2 from
    # one call to the next is reused)
    wa, wsm = [], []
    for i in range(min(n2, 100)):
        g2, ev = timed[0]
        g2.replay()
        torch.cuda.synchronize()
        wa.append(ev[0].elapsed_time(ev[1]))
        wsm.append(ev[1].elapsed_time(ev[2]))
    warm = {"attn": _max_over_ranks(dist, statistics.mean(wa) / 1e3),
            "samp": _max_over_ranks(dist, statistics.mean(wsm) / 1e3)}
    time.sleep(0.2)
    clocks.stop()
    dd.query_device_error(ws_attn)
    t_attn, t_samp = per["attn"], per["samp"]
    del graphs, timed

    # end to end: host buffers, copies inside the timed region
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, w, sets[0], dd, dev, stream, desc, dist)

    ms_per_step = ms_total / args.steps
    value = world * w.batch * args.steps / (ms_total / 1e3)
    hbm, tf_burst, tf_sus, src = _peaks()
    samp_bytes = w.logit_bytes() + R * (4 + 4 + 4 + 1)
    samp_gbs = samp_bytes / t_samp / 1e9
    attn_tf = w.attn_flops() / t_attn / 1e12
    traffic = _profile_traffic()
    clk = clocks.summary(t_wall0, t_wall1)
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "batch_per_gpu": w.batch, "canvas": w.canvas,
                   "heads_q": w.heads_q, "heads_kv": w.heads_kv, "head_dim": w.head_dim,
                   "prefix": list(w.prefix_lens), "vocab": w.vocab, "renoise_rate": w.rates[0],
                   "temperature": w.temperatures[0],
                   "l2": f"{N_SETS} rotating input sets of "
                         f"{(w.logit_bytes() + 2 * sets[0]['kp'].numel() * 2) / 1e6:.0f} MB "
                         "(> 126 MB L2)",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "kernel": "sampler (scan pass + row merge)",
                     "achieved": samp_gbs, "peak": hbm, "unit": "GB/s", "frac": samp_gbs / hbm,
                     "traffic": traffic.get(f"sampler@{w.name}"), "peak_source": src,
                     "algorithmic_bytes": samp_bytes, "ms": t_samp * 1e3,
                     "ms_warm": warm["samp"] * 1e3,
                     "nominal_peak": NOMINAL_HBM_GBS, "frac_of_nominal": samp_gbs / NOMINAL_HBM_GBS,
                     "alu_ceiling": _sampler_alu_ceiling(samp_gbs, clk.get("sm_mhz"))},
        "roofline_attn": {"bound": "tensor", "kernel": "canvas attention (tcgen05 + merge)",
                          "achieved": attn_tf, "peak": tf_burst, "unit": "TFLOP/s",
                          "frac": attn_tf / tf_burst, "frac_of_sustained": attn_tf / tf_sus,
                          "nominal_peak": NOMINAL_BF16_TFLOPS,
                          "frac_of_nominal": attn_tf / NOMINAL_BF16_TFLOPS,
                          "flops": w.attn_flops(), "ms": t_attn * 1e3,
                          "ms_warm": warm["attn"] * 1e3,
                          # the step time less the sampler's: the event records
                          # between the two calls in `ms` stop the attention
                          # launch from overlapping the previous kernel's tail
                          "ms_marginal": (ms_per_step / 1e3 - t_samp) * 1e3,
                          "frac_marginal": (w.attn_flops() / (ms_per_step / 1e3 - t_samp) / 1e12
                                            / tf_burst) if ms_per_step / 1e3 > t_samp else None,
                          "traffic": traffic.get(f"attention@{w.name}"), "peak_source": src},
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clk,
    }
    if w.steps > 1:
        res["block"] = run_block(w, dd, dev, dist)
    if rank == 0 and world == 1 and not args.no_cpu:
        res["cpu_baseline"] = cpu_baseline(w, sets[0])
    return res


def run_block(w, dd, dev, dist, reps: int = 20):
    """The whole block loop (dd_denoise_block over the workload's steps, with
    its rate schedule) on pre-generated per-step inputs: mean device time of
    one block, max over ranks."""
    q, kc, vc, lg = workloads.all_steps(w, device=dev)
    kp, vp, cu = workloads.prefix_kv(w, device=dev)
    cud = cu.to(dev)
    desc = dd.attn_desc(q[0], kc[0], w.scale)
    ws = dd.new_workspace(dd.denoise_block_workspace_bytes(desc, cu.numpy(), w.vocab), dev)
    attn_out = torch.empty_like(q)
    canvas = torch.empty(w.rows, dtype=torch.int32, device=dev)

    def block():
        dd.denoise_block(q, kc, vc, kp, vp, cud, lg, w.rates, w.temperatures, w.seed,
                         cu_prefix_host=cu.numpy(), scale=w.scale, attn_out=attn_out,
                         canvas=canvas, keep_history=False, workspace=ws)

    for _ in range(3):
        block()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        block()
    e1.record()
    torch.cuda.synchronize()
    ms = _max_over_ranks(dist, e0.elapsed_time(e1) / reps)
    dd.query_device_error(ws)
    # the same loop captured once (dd_denoise_block_graph) and replayed
    g = dd.denoise_block_graph(q, kc, vc, kp, vp, cud, lg, w.rates, w.temperatures, w.seed,
                               cu_prefix_host=cu.numpy(), scale=w.scale, attn_out=attn_out,
                               canvas=canvas, keep_history=False, workspace=ws)
    for _ in range(3):
        g.launch()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(reps):
        g.launch()
    e1.record()
    torch.cuda.synchronize()
    ms_g = _max_over_ranks(dist, e0.elapsed_time(e1) / reps)
    g.destroy()
    dd.query_device_error(ws)
    res = {"steps": w.steps, "ms_per_block": ms, "blocks_per_s": 1e3 / ms,
           "ms_per_block_graph": ms_g, "blocks_per_s_graph": 1e3 / ms_g,
           "timing": f"mean of {reps} eager dd_denoise_block calls, and of {reps} replays of "
                     "the same loop captured once (dd_denoise_block_graph), CUDA events"}
    if w.dtype == "bf16" and w.head_dim == 128:
        # the same block with 8-bit attention inputs (dd_denoise_block_fp8)
        q8, kc8, vc8, kp8, vp8, _, f8 = workloads.e4m3_block_inputs(w, device=dev)

        def block8():
            dd.denoise_block_fp8(q8, kc8, vc8, kp8, vp8, cud, f8, lg, w.rates, w.temperatures,
                                 w.seed, cu_prefix_host=cu.numpy(), scale=w.scale,
                                 attn_out=attn_out, canvas=canvas, keep_history=False,
                                 workspace=ws)

        for _ in range(3):
            block8()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(reps):
            block8()
        e1.record()
        torch.cuda.synchronize()
        ms8 = _max_over_ranks(dist, e0.elapsed_time(e1) / reps)
        dd.query_device_error(ws)
        res.update({"ms_per_block_e4m3": ms8, "blocks_per_s_e4m3": 1e3 / ms8,
                    "timing_e4m3": f"mean of {reps} eager dd_denoise_block_fp8 calls on the "
                                   "same block, E4M3 attention inputs, bf16 logits"})
    return res


def run_attn_e4m3(w, reps: int = 50):
    """Canvas attention on E4M3 inputs (dd_canvas_attn_fp8) beside the bf16
    kernel on the same workload: device time of one call (attention + split
    combine), CUDA events around the call only, L2 flushed before every
    call (a 256 MB write), median of `reps`."""
    import block_discrete_diffusion_dd_b200 as dd
    dev = torch.device("cuda", torch.cuda.current_device())
    q8, kc8, vc8, kp8, vp8, cu, f = workloads.e4m3_attn_inputs(w, 0, device=dev)
    q, kc, vc = workloads.canvas_qkv(w, 0, device=dev)
    kp, vp, _ = workloads.prefix_kv(w, device=dev)
    cud = cu.to(dev)
    d8, d16 = dd.attn_desc(q8, kc8, w.scale), dd.attn_desc(q, kc, w.scale)
    ws8 = dd.new_workspace(dd.canvas_attn_workspace_bytes(d8, cu), dev)
    ws16 = dd.new_workspace(dd.canvas_attn_workspace_bytes(d16, cu), dev)
    o8 = torch.empty(q8.shape, dtype=torch.bfloat16, device=dev)
    o16 = torch.empty_like(q)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    calls = {
        "e4m3": lambda: dd.canvas_attn_fp8(q8, kc8, vc8, kp8, vp8, cud, f, cu, scale=w.scale,
                                           out=o8, workspace=ws8),
        "bf16": lambda: dd.canvas_attn(q, kc, vc, kp, vp, cud, cu, scale=w.scale, out=o16,
                                       workspace=ws16),
    }
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    t_wall0 = time.time()
    ms = {}
    for name, fn in calls.items():
        for _ in range(5):
            fn()
        ts = []
        for _ in range(reps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        ms[name] = statistics.median(ts)
    t_wall1 = time.time()
    time.sleep(0.2)
    clocks.stop()
    dd.query_device_error(ws8)
    dd.query_device_error(ws16)
    hbm, tf_burst, tf_sus, src = _peaks()
    flops = w.attn_flops()
    tf8, tf16 = flops / ms["e4m3"] / 1e9, flops / ms["bf16"] / 1e9
    return {
        "metric": "canvas attention throughput, E4M3 inputs", "value": tf8, "unit": "TFLOP/s",
        "higher_is_better": True, "dtype": "e4m3", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "canvas": w.canvas,
                   "heads_q": w.heads_q, "heads_kv": w.heads_kv, "head_dim": w.head_dim,
                   "prefix": list(w.prefix_lens), "factors": list(f),
                   "l2": "flushed (256 MB write) before every call"},
        "ms": ms["e4m3"],
        "roofline": {"bound": "tensor", "achieved": tf8, "peak": 2 * tf_burst, "unit": "TFLOP/s",
                     "frac": tf8 / (2 * tf_burst), "flops": flops,
                     "nominal_peak": 2 * NOMINAL_BF16_TFLOPS,
                     "frac_of_nominal": tf8 / (2 * NOMINAL_BF16_TFLOPS),
                     "traffic": _profile_traffic().get(f"attention_e4m3@{w.name}"),
                     "peak_source": f"{src} bf16 burst x 2 (nominal E4M3 / bf16 ratio)"},
        "bf16_same_workload": {"ms": ms["bf16"], "TFLOP/s": tf16, "frac": tf16 / tf_burst,
                               "frac_of_nominal": tf16 / NOMINAL_BF16_TFLOPS},
        "timing": f"median of {reps} calls, CUDA events around each call",
        "clocks": clocks.summary(t_wall0, t_wall1),
    }


def run_soft_embed(w, reps: int = 30):
    """The self-conditioning soft embedding softmax(logits / tau) E on the
    workload's logits and a synthetic E [V, Hq * D] (dd_soft_embed: row
    log-sum-exp, split-K tensor-core product, fixed-order split reduction):
    device time of one call, CUDA events around the call only, L2 flushed
    before every call, median of `reps`."""
    import block_discrete_diffusion_dd_b200 as dd
    dev = torch.device("cuda", torch.cuda.current_device())
    lg = workloads.logits(w, 0, device=dev)
    E = workloads.embedding(w, device=dev)
    d = E.shape[1]
    ws = dd.new_workspace(dd.soft_embed_workspace_bytes(w.rows, w.vocab, d), dev)
    out = torch.empty((w.rows, d), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    t_wall0 = time.time()
    for _ in range(3):
        dd.soft_embed(lg, w.temperatures[0], E, out=out, workspace=ws)
    ts = []
    for _ in range(reps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        dd.soft_embed(lg, w.temperatures[0], E, out=out, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    # the MLP alone (dd_ffw) and the whole signal (dd_self_condition)
    w1, b1, w2, b2 = workloads.ffw_weights(w, d, device=dev)
    u = out.clone()
    z = torch.empty_like(u)
    hidden = w1.shape[1]
    ws_f = dd.new_workspace(int(dd.load().dd_ffw_workspace(w.rows, d, hidden)), dev)
    ws_c = dd.new_workspace(int(dd.load().dd_self_condition_workspace(w.rows, w.vocab, d,
                                                                       hidden)), dev)

    def timed(fn):
        for _ in range(3):
            fn()
        tt = []
        for _ in range(reps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            tt.append(e0.elapsed_time(e1))
        return statistics.median(tt)

    ms_ffw = timed(lambda: dd.ffw(u, w1, b1, w2, b2, out=z, workspace=ws_f))
    ms_sc = timed(lambda: dd.self_condition(lg, w.temperatures[0], E, w1, b1, w2, b2, out=z,
                                            workspace=ws_c))
    t_wall1 = time.time()
    time.sleep(0.2)
    clocks.stop()
    dd.query_device_error(ws)
    dd.query_device_error(ws_f)
    dd.query_device_error(ws_c)
    ms = statistics.median(ts)
    hbm, tf_burst, tf_sus, src = _peaks()
    ffw_flops = 4 * w.rows * d * hidden
    ffw_bytes = 2 * (2 * d * hidden + hidden + d + 2 * w.rows * d + 2 * w.rows * hidden)
    flops = 2 * w.rows * w.vocab * d
    nbytes = (w.vocab * d + w.rows * w.vocab + w.rows * d) * 2
    gbs, tfs = nbytes / ms / 1e6, flops / ms / 1e9
    return {
        "metric": "self-conditioning soft embedding softmax(logits / tau) E", "value": ms * 1e3,
        "unit": "us per call", "higher_is_better": False, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "rows": w.rows, "vocab": w.vocab, "d": d,
                   "temperature": w.temperatures[0],
                   "l2": "flushed (256 MB write) before every call"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                     "frac": gbs / hbm, "bytes": nbytes, "peak_source": src},
        "tensor": {"achieved": tfs, "peak": tf_burst, "unit": "TFLOP/s", "frac": tfs / tf_burst,
                   "flops": flops},
        "timing": f"median of {reps} calls, CUDA events around each call",
        "ffw": {"what": "the self-conditioning MLP GELU(u W1 + b1) W2 + b2 (dd_ffw), "
                        f"d {d}, hidden {hidden}, synthetic weights",
                "ms": ms_ffw, "flops": ffw_flops, "bytes": ffw_bytes,
                "TFLOP/s": ffw_flops / ms_ffw / 1e9, "frac_tensor": ffw_flops / ms_ffw / 1e9 / tf_burst,
                "GB/s": ffw_bytes / ms_ffw / 1e6, "frac_hbm": ffw_bytes / ms_ffw / 1e6 / hbm},
        "self_condition": {"what": "dd_self_condition: soft embedding, then the MLP",
                           "ms": ms_sc},
        "clocks": clocks.summary(t_wall0, t_wall1),
    }


# The sampler's arithmetic ceiling: per warp-item of 256 logits the scan
# issues 2 Philox4x32-10 blocks x 18 IMAD.WIDE (two of the 20 products per
# block are row-invariant and hoisted) plus 16 packed fp32 ops, all on the
# FMA-heavy pipe of an SM sub-partition; the ncu counters of the scan kernel
# (heavy-pipe cycles per IMAD) put an IMAD.WIDE at 4 cycles of that pipe and
# a packed fp32 op at 2.  B200: 148 SMs x 4 sub-partitions.
SAMPLER_HEAVY_CYCLES_PER_ITEM = 36 * 4 + 16 * 2
B200_SUBPARTITIONS = 148 * 4


def _sampler_alu_ceiling(achieved_gbs, sm_mhz):
    if not sm_mhz:
        return None
    items_per_s = B200_SUBPARTITIONS * sm_mhz * 1e6 / SAMPLER_HEAVY_CYCLES_PER_ITEM
    ceiling = items_per_s * 256 * 2 / 1e9  # GB/s of bf16 logits
    return {"bound": "alu", "unit": "GB/s", "peak": ceiling, "frac": achieved_gbs / ceiling,
            "sm_mhz": sm_mhz, "heavy_cycles_per_256_logits": SAMPLER_HEAVY_CYCLES_PER_ITEM}


def _launches_per_step(dd, step) -> int:
    """Kernels one step launches (counted by the library on this thread)."""
    dd.reset_launch_count()
    step(0)
    torch.cuda.synchronize()
    return dd.launch_count()


def run_e2e(args, w, s, dd, dev, stream, desc, dist):
    """Same step through the C ABI with inputs in pinned host memory: every
    step copies its inputs host->device and reads tokens + confidences back."""
    names = ["q", "kc", "vc", "kp", "vp", "logits"]
    host = {k: s[k].cpu().pin_memory() for k in names}
    host["cu"] = s["cu"].cpu().pin_memory()
    devb = {k: torch.empty_like(s[k]) for k in names}
    devb["cu"] = torch.empty_like(s["cu"])
    ws_attn = dd.new_workspace(dd.canvas_attn_workspace_bytes(desc, s["cu_host"]), dev)
    ws_samp = dd.new_workspace(dd.sample_workspace_bytes(w.rows, w.vocab, w.torch_dtype), dev)
    attn_out = torch.empty_like(s["q"])
    outs = {"tokens": torch.empty(w.rows, dtype=torch.int32, device=dev), "pred": None,
            "entropy": None, "conf": torch.empty(w.rows, dtype=torch.float32, device=dev),
            "renoised": None}
    tok_h = torch.empty(w.rows, dtype=torch.int32).pin_memory()
    conf_h = torch.empty(w.rows, dtype=torch.float32).pin_memory()
    h2d = sum(host[k].numel() * host[k].element_size() for k in host)
    d2h = tok_h.numel() * 4 + conf_h.numel() * 4

    def step(i):
        for k in host:
            devb[k].copy_(host[k], non_blocking=True)
        dd.canvas_attn(devb["q"], devb["kc"], devb["vc"], devb["kp"], devb["vp"], devb["cu"],
                       s["cu_host"], scale=w.scale, out=attn_out, workspace=ws_attn,
                       stream=stream)
        dd.sample_renoise(devb["logits"], w.temperatures[0], w.rates[0], w.seed, i,
                          outputs=outs, workspace=ws_samp, stream=stream)
        tok_h.copy_(outs["tokens"], non_blocking=True)
        conf_h.copy_(outs["conf"], non_blocking=True)

    n = max(3, min(args.steps, args.e2e_steps))
    for i in range(3):
        step(i)
    _barrier(dist)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(n):
        step(i)
    b.record(stream)
    _barrier(dist)
    ms = _max_over_ranks(dist, a.elapsed_time(b))
    world = dist.get_world_size() if dist is not None else 1
    return {"value": world * w.batch * n / (ms / 1e3), "unit": UNIT, "steps": n,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": ms / n}


def _source_sha(name: str) -> str:
    import hashlib
    path = os.path.join(ROOT, "block_discrete_diffusion_dd_b200", "csrc", name)
    try:
        with open(path, "rb") as f:
            return hashlib.sha256(f.read()).hexdigest()[:16]
    except OSError:
        return ""


def _profile_traffic() -> dict:
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum)
    from the committed ncu summary profiles/traffic.txt.  A line reads
    `<kernel group>@<workload> <bytes per launch> <source file> <sha256/16 of
    that source>`; a figure taken on another version of the kernel source
    reads as None."""
    out = {}
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.txt")) as f:
            for line in f:
                parts = line.split()
                if len(parts) == 4 and not line.startswith("#"):
                    kernel, nbytes, src, sha = parts
                    out[kernel] = float(nbytes) if _source_sha(src) == sha else None
    except OSError:
        pass
    return out


def _cpu_model() -> str:
    """The host CPU's model name (lscpu), for the baseline's record."""
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for line in out.splitlines():
            if line.startswith("Model name:"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    import platform
    return platform.processor() or "unknown"


def _host_cores() -> int:
    if "OMP_NUM_THREADS" in os.environ:
        return int(os.environ["OMP_NUM_THREADS"])
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_sample_plan(w, cores: int):
    """The bounded sample of one step that both CPU legs (the `cpu_baseline`
    of our line and the `--impl reference` arm) time: `npos` canvas positions
    of every batch row and head for the attention, and `nrows` sampler rows,
    at least two units of work per core (and 16 rows) so every core is busy.
    The step time is extrapolated from it: attention x C / npos, sampler x
    R / nrows."""
    npos = min(w.canvas, max(8, -(-2 * cores // (w.batch * w.heads_q))))
    nrows = min(w.rows, max(16, 2 * cores))
    return npos, nrows


def _oracle_sample(w, s, lg, npos, nrows, rep, threads=0):
    """One timed sample of the oracle step: (attention s, sampler s), over
    positions and rows spread evenly and rotated by `rep`."""
    import oracle
    off = (rep * 37) % w.canvas
    pos = ((np.arange(npos) * (w.canvas // npos) + off) % w.canvas).astype(np.int32)
    sel = ((np.arange(nrows) * (w.rows // nrows) + off) % w.rows).astype(np.int64)
    t0 = time.perf_counter()
    oracle.canvas_attn(s["q"], s["kc"], s["vc"], s["kp"], s["vp"], s["cu_host"], w.scale,
                       positions=pos, threads=threads)
    t1 = time.perf_counter()
    oracle.sample_renoise(lg, w.temperatures[0], w.rates[0], w.seed, rep, rows=sel,
                          threads=threads)
    t2 = time.perf_counter()
    return t1 - t0, t2 - t1


def _extrapolate(w, t_attn, t_samp, npos, nrows):
    return t_attn * (w.canvas / npos) + t_samp * (w.rows / nrows)


def cpu_baseline(w, s, budget_s: float = 10.0):
    """The oracle, as it stands, on this host's cores, on the bounded sample
    of oracle_sample_plan, repeated for about `budget_s` seconds and
    extrapolated to whole steps; plus one sample on a single thread."""
    import oracle
    oracle.build()
    cores = _host_cores()
    npos, nrows = oracle_sample_plan(w, cores)
    q, kc, vc, kp, vp = (s[k].cpu() for k in ("q", "kc", "vc", "kp", "vp"))
    host = {"q": q, "kc": kc, "vc": vc, "kp": kp, "vp": vp, "cu_host": s["cu_host"]}
    lg = s["logits"].cpu()
    ta = ts = 0.0
    reps = 0
    t_start = time.perf_counter()
    while reps == 0 or time.perf_counter() - t_start < budget_s:
        a, b = _oracle_sample(w, host, lg, npos, nrows, reps)
        ta, ts, reps = ta + a, ts + b, reps + 1
    step_s = _extrapolate(w, ta / reps, ts / reps, npos, nrows)
    a1, b1 = _oracle_sample(w, host, lg, npos, nrows, reps, threads=1)
    step1_s = _extrapolate(w, a1, b1, npos, nrows)
    return {"value": w.batch / step_s, "unit": UNIT, "cores": cores, "kind": "oracle",
            "extrapolated": True,
            "sample": f"{reps} x ({npos}/{w.canvas} canvas positions of every batch row and "
                      f"head for attention + {nrows}/{w.rows} sampler rows), float64, "
                      f"{ta + ts:.1f} s on {cores} host cores; extrapolated to whole steps",
            "per_step_s": {"attention": ta / reps * (w.canvas / npos),
                           "sampler": ts / reps * (w.rows / nrows)},
            "one_thread": {"value": w.batch / step1_s, "unit": UNIT,
                           "per_step_s": {"attention": a1 * (w.canvas / npos),
                                          "sampler": b1 * (w.rows / nrows)}},
            "cpu_model": _cpu_model(), "seconds": ta + ts}


def run_reference(args, w, dist, rank, world):
    """The reference arm: the oracle timed on host cores, each step the
    bounded sample of oracle_sample_plan (the same sample as our line's
    cpu_baseline), extrapolated to a whole step."""
    if rank != 0:
        return None
    import oracle
    oracle.build()
    cores = _host_cores()
    npos, nrows = oracle_sample_plan(w, cores)
    ws0 = workloads.scaled(w)
    s = {}
    s["q"], s["kc"], s["vc"] = workloads.canvas_qkv(ws0, 0)
    s["kp"], s["vp"], cu = workloads.prefix_kv(ws0)
    s["cu_host"] = cu.numpy()
    lg = workloads.logits(ws0, 0)
    ta, ts = [], []
    for i in range(args.warmup + args.steps):
        a, b = _oracle_sample(w, s, lg, npos, nrows, i)
        if i >= args.warmup:
            ta.append(a)
            ts.append(b)
    t_attn, t_samp = statistics.mean(ta), statistics.mean(ts)
    step_s = _extrapolate(w, t_attn, t_samp, npos, nrows)
    value = w.batch / step_s
    sample = (f"{npos}/{w.canvas} canvas positions of every batch row and head (attention) and "
              f"{nrows}/{w.rows} sampler rows per step, float64 oracle on {cores} host cores; "
              "extrapolated to a whole step")
    return {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "extrapolated": True,
            "timed_ms_per_step": (t_attn + t_samp) * 1e3,
            "config": {"workload": w.name, "batch_per_gpu": w.batch, "canvas": w.canvas,
                       "heads_q": w.heads_q, "heads_kv": w.heads_kv, "head_dim": w.head_dim,
                       "prefix": list(w.prefix_lens), "vocab": w.vocab,
                       "parallelism": "host cores (rank 0 only)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample, "cpu_model": _cpu_model()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}


def run_policy(w, reps: int = 10, max_steps: int = 12, budget: float = 0.1,
               stop_entropy: float = 0.005):
    """The pages' adaptive block (dd_denoise_block_adaptive) on the 12-step
    geometry (B=1, prefix 8192, V = 262144) with synthetic logits that sharpen
    step by step (N(0, 1.5^2) plus a spike of 3 + 4 s at one token per row),
    so the canvas halts early; temperatures annealed 0.8 -> 0.4 over a
    nominal 48 steps.  Also times dd_entropy_accept alone on 8 canvases."""
    import block_discrete_diffusion_dd_b200 as dd
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    g = torch.Generator(device=dev).manual_seed(w.seed)
    R, V = w.rows, w.vocab
    qs, ks, vs, ls = [], [], [], []
    hot = torch.randint(0, V, (R,), generator=g, device=dev)
    for s in range(max_steps):
        q, kc, vc = workloads.canvas_qkv(w, s, device=dev)
        lg = torch.randn((R, V), generator=g, device=dev) * 1.5
        lg[torch.arange(R, device=dev), hot] += 3.0 + 4.0 * s
        qs.append(q), ks.append(kc), vs.append(vc), ls.append(lg.to(torch.bfloat16))
        del lg
    q, kc, vc, lg = torch.stack(qs), torch.stack(ks), torch.stack(vs), torch.stack(ls)
    del qs, ks, vs, ls
    kp, vp, cu = workloads.prefix_kv(w, device=dev)
    cud = cu.to(dev)
    temps = [float(np.float32(0.8 - 0.4 * s / 47)) for s in range(max_steps)]
    desc = dd.attn_desc(q[0], kc[0], w.scale)
    ws = dd.new_workspace(int(dd.load().dd_denoise_block_adaptive_workspace(
        ctypes.byref(desc), cu.numpy().ctypes.data_as(ctypes.c_void_p), V)), dev)
    attn_out = torch.empty_like(q)

    def block():
        canvas = torch.zeros(R, dtype=torch.int32, device=dev)
        return dd.denoise_block_adaptive(q, kc, vc, kp, vp, cud, lg, temps, budget, stop_entropy,
                                         w.seed, cu_prefix_host=cu, scale=w.scale,
                                         attn_out=attn_out, canvas=canvas, keep_history=False,
                                         workspace=ws)

    for _ in range(2):
        res = block()
    torch.cuda.synchronize()
    wall, dev_ms = [], []
    for _ in range(reps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        t0 = time.perf_counter()
        e0.record()
        res = block()
        e1.record()
        torch.cuda.synchronize()
        wall.append((time.perf_counter() - t0) * 1e3)
        dev_ms.append(e0.elapsed_time(e1))
    n = res["steps_run"]
    # the same loop kept on the device (dd_denoise_block_adaptive_graph):
    # one graph launch per block, no per-step host read
    ag = dd.denoise_block_adaptive_graph(q, kc, vc, kp, vp, cud, lg, temps, budget, stop_entropy,
                                         w.seed, cu_prefix_host=cu, scale=w.scale,
                                         attn_out=attn_out, keep_history=False)
    for _ in range(2):
        t = ag.launch()
    torch.cuda.synchronize()
    g_wall, g_dev = [], []
    for _ in range(reps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        t0 = time.perf_counter()
        e0.record()
        t = ag.launch()
        e1.record()
        torch.cuda.synchronize()
        g_wall.append((time.perf_counter() - t0) * 1e3)
        g_dev.append(e0.elapsed_time(e1))
    g_steps = int(t["steps_run"].item())
    same = bool(torch.equal(t["canvas"], res["canvas"]) and
                torch.equal(t["halt_step"], res["halt_step"]))
    dd.query_device_error(t["workspace"])
    ag.destroy()
    # the acceptance kernel alone, 8 canvases of 256
    h = torch.rand(8 * 256, device=dev) * 0.01
    pr = torch.randint(0, V, (8 * 256,), dtype=torch.int32, device=dev)
    out = {"tokens": torch.empty(8 * 256, dtype=torch.int32, device=dev),
           "accepted": torch.empty(8 * 256, dtype=torch.uint8, device=dev)}
    for _ in range(5):
        dd.entropy_accept(h, pr, 256, budget, 0, 0, V, tokens=out["tokens"],
                          accepted=out["accepted"])
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()      # 100 back-to-back calls, no host in the way
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            for _ in range(100):
                dd.entropy_accept(h, pr, 256, budget, 0, 0, V, tokens=out["tokens"],
                                  accepted=out["accepted"], stream=side)
    torch.cuda.current_stream().wait_stream(side)
    graph.replay()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    graph.replay()
    e1.record()
    torch.cuda.synchronize()
    return {"metric": "adaptive block (the pages' policy): ms per block", "unit": "ms",
            "value": statistics.median(wall), "device_ms": statistics.median(dev_ms),
            "steps_run": n, "max_steps": max_steps, "ms_per_step": statistics.median(wall) / n,
            "halt_step": res["halt_step"].cpu().tolist(),
            "entropy_accept_us_8_canvases": e0.elapsed_time(e1) * 10.0,
            "device_loop": {"ms_per_block": statistics.median(g_dev),
                            "wall_ms_per_block": statistics.median(g_wall),
                            "steps_run": g_steps, "same_result_as_eager": same,
                            "timing": "median of %d replays of dd_denoise_block_adaptive_graph "
                                      "(one IF node per step), CUDA events" % reps},
            "config": {"workload": w.name + " geometry, sharpening synthetic logits",
                       "budget": budget, "stop_entropy": stop_entropy,
                       "temperature": "0.8 -> 0.4 over 48 nominal steps"},
            "timing": "median of %d calls; wall clock includes the per-step halt-flag reads" % reps}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="ragged_b8", choices=list(workloads.WORKLOADS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--policy", action="store_true",
                    help="time the pages' adaptive block loop instead (one JSON line)")
    ap.add_argument("--attn-e4m3", action="store_true",
                    help="time canvas attention on E4M3 inputs beside bf16 (one JSON line)")
    ap.add_argument("--soft-embed", action="store_true",
                    help="time the self-conditioning soft embedding (one JSON line)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    w = workloads.WORKLOADS[args.workload]
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        res = run_reference(args, w, None, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    from block_discrete_diffusion_dd_b200 import build as libbuild
    if not os.path.exists(libbuild.LIB):
        libbuild.build()
    if args.policy:
        print(json.dumps(run_policy(workloads.WORKLOADS["block12_L8192"])), flush=True)
        return
    if args.attn_e4m3:
        print(json.dumps(run_attn_e4m3(w)), flush=True)
        return
    if args.soft_embed:
        print(json.dumps(run_soft_embed(w)), flush=True)
        return
    dist, rank, world, local_rank = _dist()
    if world != args.gpus and rank == 0:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    res = run_ours(args, w, dist, rank, world, local_rank)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
