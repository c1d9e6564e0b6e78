#!/usr/bin/env python3
"""Throughput of the Gated DeltaNet-2 chunkwise forward (gdn2_chunk_fwd) on B200.

Workload: the long-context 16K x 1 token budget of the pages' throughput
figure -- B=1, T=16384, H=16, dk=dv=128, bf16 q/k/v/out, fp32 gates with
strong per-channel decay variety, seeded synthetic inputs (workloads.py,
workload 2).  A step is one gdn2_chunk_fwd call over the whole batch.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun (one process per GPU, NCCL for the barrier and the
max-over-ranks reduction only): every rank runs an independent replica of the
workload ("replicas only": the operator needs no exchange between sequences).
Prints one JSON line on rank 0.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "GDN2 chunk-fwd tokens/s (B·T) at H=16,dk=dv=128,bf16 on 1 B200; % of roofline"
UNIT = "tokens/s"
WORKLOAD_ID = 2
B, T, H, DK, DV = 1, 16384, 16, 128, 128
TH = B * T * H
# Algorithmic work of the method per token-head (bf16 I/O, d = 128, chunk 64):
# q, k, v in bf16 (768 B) + log_alpha, b, w in fp32 (1536 B) + O in bf16 (256 B);
# per (sequence, head) the fp32 final state (64 KiB); h0 is zero and not read.
ALG_BYTES_PER_TH = 2560
ALG_BYTES = TH * ALG_BYTES_PER_TH + B * H * DK * DV * 4
# Chunk-form FLOPs per token-head: 6*dk*dv + 5*C*d + C^2/3 with C = 64.
ALG_FLOPS = TH * (6 * DK * DV + 5 * 64 * 128 + 64 * 64 / 3)
# Compulsory bytes of the two stage kernels given the stored chunk factors of
# the affine set (bf16 Mp, Nc = 2 x 128 x 128 x 2 B per 64 tokens, Q_eff,
# O_part = 2 x 64 x 128 x 2 B: 1536 B per token-head; exp(g_n) fp32 8 B).
FACTOR_BYTES_PER_TH = 1536 + 8
# DRAM bytes (read + write) of one fused launch at 16K x 1, from one ncu
# capture (dram__bytes_read.sum 604,688,128 + dram__bytes_write.sum
# 429,519,104) of this build's fused kernel under this script's own command
# (profiles/ holds the command).  It is taken again (or set to None) whenever
# the fused kernel changes.
FUSED_TRAFFIC_BYTES = 604688128 + 429519104
PREP_BYTES = TH * (2304 + FACTOR_BYTES_PER_TH)
WALK_BYTES = TH * (FACTOR_BYTES_PER_TH + 256) + B * H * DK * DV * 4
L2_FLUSH_BYTES = 256 << 20


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        fd, self.path = tempfile.mkstemp(prefix="gdn2_clocks_", suffix=".csv")
        os.close(fd)
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = []
        self.cmd = ["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                    "-lms", "50"]

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(self.cmd, stdout=self.f, stderr=subprocess.DEVNULL)
            # the first sample is out before the timed region starts
            t0 = time.time()
            while time.time() - t0 < 5.0 and self.proc.poll() is None:
                if os.path.getsize(self.path) > 0:
                    break
                time.sleep(0.02)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return None
        rows = []
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
                except ValueError:
                    continue
        except OSError:
            return None
        finally:
            try:
                os.remove(self.path)
            except OSError:
                pass
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


def dist_setup(n_gpus):
    import torch
    if n_gpus <= 1 or "RANK" not in os.environ:
        torch.cuda.set_device(0)
        return 0, 1, 0
    import datetime

    import torch.distributed as dist
    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                            device_id=torch.device("cuda", local))
    return dist.get_rank(), dist.get_world_size(), local


def barrier_sync(world, cuda=True):
    """Every rank's device idle and every rank here (both sides of a timed
    region)."""
    import torch
    if cuda:
        torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if cuda:
        torch.cuda.synchronize()


def max_over_ranks(x, world, device="cuda"):
    """The slowest rank's value (times are taken per rank on its own device)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world, tokens_per_rank, ms_max):
    """Whole-job throughput: every rank runs a full replica, and the job takes
    as long as its slowest rank."""
    return world * tokens_per_rank / (ms_max / 1e3)


def cpu_oracle_sample(x, target_s, max_tokens=T):
    """Time the fp64 oracle (as it stands) on the first `t` tokens of every
    head, with `t` chosen so that one run takes about `target_s` seconds."""
    import oracle
    cores = min(oracle.default_threads(), H * B)
    t_tok = 256
    while True:
        s = slice(0, t_tok)
        args = [a[:, s] for a in (x.q, x.k, x.v, x.log_alpha, x.b, x.w)]
        t0 = time.perf_counter()
        oracle.recurrent(*args, x.scale, nthreads=cores)
        dt = time.perf_counter() - t0
        if dt >= target_s * 0.5 or t_tok >= max_tokens:
            return B * t_tok / dt, cores, t_tok, dt
        t_tok = int(min(max_tokens, max(t_tok * 2, t_tok * target_s / max(dt, 1e-3))))


def run_reference(args, rank):
    """The oracle as the reference arm: each step is a bounded sample of the
    workload (all 16 heads, the first t tokens), timed on the host cores."""
    if rank != 0:
        return
    from workloads import config
    x = config(WORKLOAD_ID)
    per_step = max(0.05, min(2.0, 150.0 / max(1, args.steps + args.warmup)))
    _, cores, t_tok, _ = cpu_oracle_sample(x, per_step)
    import oracle
    s = slice(0, t_tok)
    sample = [a[:, s] for a in (x.q, x.k, x.v, x.log_alpha, x.b, x.w)]
    for _ in range(args.warmup):
        oracle.recurrent(*sample, x.scale, nthreads=cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.recurrent(*sample, x.scale, nthreads=cores)
    dt = (time.perf_counter() - t0) / max(1, args.steps)
    value = B * t_tok / dt
    desc = f"fp64 C oracle on tokens [0,{t_tok}) of every head of the 16Kx1 workload"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "16Kx1 B=1 T=16384 H=16 dk=dv=128 (sampled)", "sample_tokens": t_tok},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_ours(args, rank, world, local):
    import torch

    import gated_delta_rule_129_b200 as gdn2
    from workloads import config
    gdn2.load_library()
    x = config(WORKLOAD_ID)
    dev = torch.device("cuda", local)
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)  # noqa: E731
    bf, f32 = torch.bfloat16, torch.float32
    q, k, v = t(x.q, bf), t(x.k, bf), t(x.v, bf)
    la, b, w = t(x.log_alpha, f32), t(x.b, f32), t(x.w, f32)
    out = torch.empty_like(v)
    hT = torch.empty((B, H, DK, DV), dtype=f32, device=dev)
    ws = torch.empty(gdn2.workspace_size(B, T, H, DK, DV, gdn2.GDN2_IO_BF16), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        gdn2.chunk_fwd(q, k, v, la, b, w, x.scale, out=out, hT=hT, workspace=ws, stream=stream)

    sampler = ClockSampler(local) if rank == 0 else None
    if sampler:
        sampler.__enter__()
    for _ in range(args.warmup):
        step()
        flush.zero_()
    # The timed steps; after each one (outside its events, like the L2 flush)
    # the fused launch alone is timed once, after its plan, so that the
    # kernel's and the step's medians come from the same loop.
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    k0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    k1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier_sync(world)
    for i in range(args.steps):
        flush.zero_()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
        flush.zero_()
        gdn2.chunk_plan((B, T, H, DK, DV), bf, ws, stream=stream)
        k0[i].record(stream)
        gdn2.chunk_fused(q, k, v, la, b, w, x.scale, ws, out=out, hT=hT, stream=stream)
        k1[i].record(stream)
    barrier_sync(world)
    if sampler:
        sampler.__exit__(None, None, None)
    step_ms = [s_.elapsed_time(e_) for s_, e_ in zip(starts, ends)]
    fused_ms = [a_.elapsed_time(b_) for a_, b_ in zip(k0, k1)]
    ms_mean = sum(step_ms) / args.steps
    ms = max_over_ranks(statistics.median(step_ms), world)
    # chunk_fwd here: plan, the fused prep + walk launch, and the two guards
    # after it (exact redo of steep-decay chunks; walk again if one occurred)
    launches_per_step = 4

    # the two stages run back to back through their own entry points
    kt = {"prep": [], "walk": []}
    nk = max(3, min(args.steps, 50))
    for i in range(nk):
        flush.zero_()
        e2, e3, e4 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e2.record(stream)
        gdn2.chunk_prep(q, k, v, la, b, w, workspace=ws, stream=stream)
        e3.record(stream)
        gdn2.chunk_walk(ws, (B, T, H, DK, DV), bf, x.scale, out=out, hT=hT, stream=stream)
        e4.record(stream)
        kt["prep"].append((e2, e3))
        kt["walk"].append((e3, e4))
    torch.cuda.synchronize()
    kern_ms = {kname: statistics.median(a.elapsed_time(bb) for a, bb in ev) for kname, ev in kt.items()}
    kern_ms["fused"] = statistics.median(fused_ms)

    # end to end: pinned host inputs -> device -> chunk_fwd -> O, hT back to pinned host
    host = {n: getattr(x, n) for n in ("q", "k", "v", "log_alpha", "b", "w")}
    pin = {}
    for n, a in host.items():
        dt = bf if n in ("q", "k", "v") else f32
        pin[n] = torch.from_numpy(np.ascontiguousarray(a)).to(dt).pin_memory()
    dev_in = {"q": q, "k": k, "v": v, "log_alpha": la, "b": b, "w": w}
    out_h = torch.empty(out.shape, dtype=bf).pin_memory()
    hT_h = torch.empty(hT.shape, dtype=f32).pin_memory()
    h2d = sum(p.numel() * p.element_size() for p in pin.values())
    d2h = out_h.numel() * out_h.element_size() + hT_h.numel() * hT_h.element_size()
    ne = max(2, min(args.steps, 10))
    barrier_sync(world)
    e_s, e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_s.record(stream)
    for _ in range(ne):
        for n in dev_in:
            dev_in[n].copy_(pin[n], non_blocking=True)
        step()
        out_h.copy_(out, non_blocking=True)
        hT_h.copy_(hT, non_blocking=True)
    e_e.record(stream)
    barrier_sync(world)
    e2e_ms = max_over_ranks(e_s.elapsed_time(e_e) / ne, world)

    decode = measure_decode(dev, stream, flush) if rank == 0 else None
    token_path = measure_token_path(dev, stream, flush, peaks()[0]) if rank == 0 else None
    others = measure_other_configs(dev, stream, flush, peaks()[0]) if (rank == 0 and not args.no_other_configs) else None
    backward = None
    if rank == 0 and not args.no_backward:
        try:
            backward = measure_backward(dev, stream, peaks()[0])
        except Exception as exc:  # the forward's line must print whatever happens here
            backward = {"error": str(exc)[:300]}
    if rank != 0:
        return
    hbm, tflops, src = peaks()
    tokens = B * T
    value = job_tokens_per_s(world, tokens, ms)
    t_roof = max(ALG_BYTES / (hbm * 1e9), ALG_FLOPS / (tflops * 1e12))
    # the fused launch is the step's one substantial kernel; its algorithmic
    # bytes are the method's own (inputs once, outputs and final state once)
    dom = "fused"
    dom_bytes = ALG_BYTES
    dom_gbs = dom_bytes / (kern_ms[dom] / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "ms_per_step_mean": ms_mean, "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "16Kx1 B=1 T=16384 H=16 dk=dv=128 bf16 I/O, fp32 gates (strong decay)",
                   "global_batch": world * B, "seq_len": T, "parallelism": f"replicas x{world}",
                   "l2": "flushed between timed steps (256 MiB write)"},
        "roofline": {"bound": "hbm", "achieved": dom_gbs, "peak": hbm, "unit": "GB/s",
                     "frac": dom_gbs / hbm, "traffic": FUSED_TRAFFIC_BYTES, "kernel": dom,
                     "kernel_ms": kern_ms[dom], "alg_bytes_per_launch": dom_bytes,
                     "peak_source": f"{src} (MEASURED_PEAKS hbm_gbs)" if src == "measured" else src},
        "roofline_step": {"alg_bytes": ALG_BYTES, "alg_flops": ALG_FLOPS, "t_roof_us": t_roof * 1e6,
                          "t_meas_us": ms * 1e3, "frac": t_roof / (ms / 1e3),
                          "achieved_gbs": ALG_BYTES / (ms / 1e3) / 1e9},
        "kernels_ms": kern_ms,
        "timing": "medians over the timed steps; the fused kernel alone is timed once after each timed step, "
                  "in the same loop",
        "e2e": {"value": job_tokens_per_s(world, tokens, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": ne},
        "gpu_launches": launches_per_step * args.steps,
    }
    clk = sampler.summary() if sampler else None
    line["clocks"] = clk
    if decode:
        decode["roofline"] = {"bound": "hbm", "achieved": decode["gbs"], "peak": hbm, "unit": "GB/s",
                              "frac": decode["gbs"] / hbm}
        line["decode_step"] = decode
    if token_path:
        line["token_path"] = token_path
    if others:
        line["other_configs"] = others
    if backward:
        line["backward_step"] = backward
    if world == 1 and not args.no_cpu_baseline:
        tps, cores, t_tok, dt = cpu_oracle_sample(x, args.cpu_seconds)
        line["cpu_baseline"] = {"value": tps, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": f"fp64 C oracle, tokens [0,{t_tok}) of all 16 heads "
                                          f"({dt:.1f} s)"}
    print(json.dumps(line), flush=True)


def measure_decode(dev, stream, flush, reps=20):
    """gdn2_recurrent_step on the 256-state decode batch (B=256, H=16,
    dk=dv=128, bf16 q/k/v/out, fp32 gates and states): its compulsory traffic
    is one read and one write of every fp32 state (2 x 256 x 16 x 128 x 128 x
    4 B) plus the token vectors."""
    import torch

    import gated_delta_rule_129_b200 as gdn2
    from workloads import decode_inputs
    di = decode_inputs(B=256, H=16, dk=128, dv=128, io="bf16", seed=41)
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)  # noqa: E731
    bf, f32 = torch.bfloat16, torch.float32
    args = (t(di.q, bf), t(di.k, bf), t(di.v, bf), t(di.log_alpha, f32), t(di.b, f32), t(di.w, f32))
    state = t(di.state, f32)
    out = torch.empty((256, 16, 128), dtype=bf, device=dev)
    nbytes = 2 * state.numel() * 4 + sum(a.numel() * a.element_size() for a in args) + out.numel() * 2
    for _ in range(3):
        gdn2.recurrent_step(*args, di.scale, state, out=out, stream=stream)
    tot = 0.0
    for _ in range(reps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        gdn2.recurrent_step(*args, di.scale, state, out=out, stream=stream)
        e1.record(stream)
        e1.synchronize()
        tot += e0.elapsed_time(e1)
    us = tot / reps * 1e3
    return {"workload": "decode B=256 H=16 dk=dv=128 (one token per state)", "us": us,
            "tokens_per_s": 256 / (us * 1e-6), "bytes": nbytes, "gbs": nbytes / (us * 1e-6) / 1e9}


def measure_backward(dev, stream, hbm, reps=3):
    """gdn2_chunk_bwd (the gradients of every input through the chunkwise WY
    form, fp32 on the CUDA cores) on the 16K x 1 workload with a random bf16 dO.  Its algorithmic traffic per
    token-head: the inputs (768 + 1536 B), dO (256 B) and the six fp32
    gradients (4 x 512 + 2 x 512 B), plus dh0."""
    import torch

    import gated_delta_rule_129_b200 as gdn2
    from workloads import config
    x = config(WORKLOAD_ID)
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)  # noqa: E731
    q, k, v = (t(a, torch.bfloat16) for a in (x.q, x.k, x.v))
    la, b, w = (t(a, torch.float32) for a in (x.log_alpha, x.b, x.w))
    gen = torch.Generator(device=dev).manual_seed(5)
    dO = torch.randn(v.shape, generator=gen, dtype=torch.float32, device=dev).to(torch.bfloat16)
    ws = torch.empty(gdn2.backward_workspace_size(B, T, H, DK, DV, gdn2.GDN2_IO_BF16), dtype=torch.uint8, device=dev)
    gdn2.chunk_bwd(q, k, v, la, b, w, x.scale, dO, workspace=ws, stream=stream)
    tot = 0.0
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        gdn2.chunk_bwd(q, k, v, la, b, w, x.scale, dO, workspace=ws, stream=stream)
        e1.record(stream)
        e1.synchronize()
        tot += e0.elapsed_time(e1)
    ms = tot / reps
    alg = TH * (768 + 1536 + 256 + 6 * 512) + B * H * DK * DV * 4
    gbs = alg / (ms / 1e3) / 1e9
    flops = backward_flops()
    tfs = flops / (ms / 1e3) / 1e12
    return {"workload": "16Kx1 backward (gdn2_chunk_bwd: chunkwise WY form, fp32 on the CUDA cores), bf16 inputs, "
                        "fp32 gradients",
            "ms": ms, "tokens_per_s": B * T / (ms / 1e3), "alg_bytes": alg, "alg_flops": flops,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm},
            "roofline_alu": {"bound": "alu", "achieved": tfs, "peak": FP32_FMA_TFLOPS, "unit": "TFLOP/s",
                             "frac": tfs / FP32_FMA_TFLOPS,
                             "peak_source": "nominal: 148 SMs x 128 fp32 lanes x 2 FLOP x 1.965 GHz"}}


# fp32 CUDA-core peak of one B200 (nominal, from the unit counts and the
# maximum SM clock): 148 SMs x 128 FMA lanes x 2 FLOP x 1.965 GHz
FP32_FMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def backward_flops(C=64):
    """Algorithmic FLOPs of the chunkwise backward at 16K x 1 (2 per
    multiply-add; triangular products counted at half):
      recompute: A, P (2 C^2/2 dk); T (C^3/6); W, Q_eff (2 C^2/2 dk);
                 U~, O_part (2 C^2/2 dv)
      the walks: U = U~ - W S0 and S1 (2 C dk dv); Kbar dS1 and the dS0
                 update (3 C dk dv)
      per chunk: P^T dO (C^2/2 dv); dQ~, dKbar, dW (3 C dk dv); dP (C^2 dv);
                 dT (C^2 dv + C^2 dk); dZ (C^2/2 dv); dE~ (C^2/2 dk);
                 dA (C^3); the three pairwise-decay sums (3 C^2/2 dk)"""
    dk, dv = DK, DV
    tri = C * C / 2
    macs = (2 * tri * dk + C ** 3 / 6 + 2 * tri * dk + 2 * tri * dv
            + 2 * C * dk * dv + 3 * C * dk * dv
            + tri * dv + 3 * C * dk * dv + C * C * dv + C * C * (dv + dk) + tri * dv + tri * dk + C ** 3
            + 3 * tri * dk)
    chunks = B * T // C
    return 2 * macs * chunks * H


def measure_token_path(dev, stream, flush, hbm, reps=20):
    """The token path around the operator at 16K x 1 (H=16, d=128, bf16):
    gdn2_token_prologue (reads q, k, v from the projections, writes the
    operator's q, k, v: 6 x 256 B per token-head) and gdn2_token_epilogue
    (reads o and the gate, writes the gated output: 3 x 256 B per token-head),
    each timed alone with CUDA events, L2 flushed, with its HBM roofline."""
    import torch

    import gated_delta_rule_129_b200 as gdn2
    gen = torch.Generator(device=dev).manual_seed(7)
    r = lambda *s: torch.randn(*s, generator=gen, device=dev)  # noqa: E731
    bf = torch.bfloat16
    q_raw, k_raw, v_raw = (r(B, T, H, DK).to(bf) for _ in range(3))
    wq, wk, wv = (0.5 * r(H * DK, 4) for _ in range(3))
    gate = r(B, T, H, DV).to(bf)
    wt = torch.ones(DV, device=dev)
    q, k, v = (torch.empty_like(q_raw) for _ in range(3))
    out = torch.empty_like(v_raw)

    def timed(fn):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)
    res = {}
    for name, fn, per_th in (
            ("prologue", lambda: gdn2.token_prologue(q_raw, k_raw, v_raw, wq, wk, wv, q=q, k=k, v=v, stream=stream),
             6 * 256),
            ("epilogue", lambda: gdn2.token_epilogue(v_raw, gate, wt, out=out, stream=stream), 3 * 256)):
        ms = timed(fn)
        nbytes = TH * per_th
        gbs = nbytes / (ms / 1e3) / 1e9
        res[name] = {"ms": ms, "alg_bytes": nbytes, "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm,
                                                                  "unit": "GB/s", "frac": gbs / hbm}}
    return res


def measure_other_configs(dev, stream, flush, hbm, steps=10):
    """gdn2_chunk_fwd on the other bf16 workloads (2K x 8, 4K x 4 with
    b = w = beta, 32 packed sequences) and on the gate ablations of the 16K x 1
    inputs (erase range [0, 2], channel-mean erase or write gate): tokens/s
    and the step roofline fraction, same timing rules as the headline number
    (median of the timed steps); the 16K x 1 workload through the two-level
    chunk scan (gdn2_chunk_fwd_segmented); and the 16K x 1 workload with fp32
    q, k, v and O (the fp32 CUDA-core path, 3,584 algorithmic bytes per
    token-head)."""
    import torch

    import gated_delta_rule_129_b200 as gdn2
    from workloads import config
    from workloads import make_inputs
    out_cfg = {}
    ablations = [
        ("16Kx1 erase range [0,2] (b scaled by 2)", dict(erase_range=2.0)),
        ("16Kx1 channel-mean erase gate", dict(mean_gate="erase")),
        ("16Kx1 channel-mean write gate", dict(mean_gate="write")),
    ]
    cases = [(lambda c=c, v_=v_: config(c, v_), False, "bf16") for c, v_ in ((1, "a"), (3, "a"), (4, "a"))]
    for name, kw in ablations:
        def mk(name=name, kw=kw):
            xi = make_inputs(1, 16384, 16, 128, 128, io="bf16", seed=2, decay="strong", **kw)
            xi.name = name
            return xi
        cases.append((mk, False, "bf16"))

    def mk_seg():
        xi = config(WORKLOAD_ID)
        xi.name = "16Kx1 through the two-level chunk scan (gdn2_chunk_fwd_segmented, 64-chunk segments)"
        return xi
    cases.append((mk_seg, True, "bf16"))

    def mk_f32():
        xi = make_inputs(1, 16384, 16, 128, 128, io="f32", seed=2, decay="strong")
        xi.name = "16Kx1 fp32 q, k, v and O (the fp32 CUDA-core path)"
        return xi
    cases.append((mk_f32, False, "f32"))
    for make, segmented, iot in cases:
        x = make()
        t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)  # noqa: E731
        bf, f32 = torch.bfloat16, torch.float32
        io_t = f32 if iot == "f32" else bf
        io_c = gdn2.GDN2_IO_F32 if iot == "f32" else gdn2.GDN2_IO_BF16
        q, k, v = t(x.q, io_t), t(x.k, io_t), t(x.v, io_t)
        la, b, w = t(x.log_alpha, f32), t(x.b, f32), t(x.w, f32)
        h0 = None if x.h0 is None else t(x.h0, f32)
        cu = None if x.cu_seqlens is None else t(x.cu_seqlens, torch.int32)
        Bc, Tc, Hc = x.q.shape[0], x.q.shape[1], x.q.shape[2]
        ns = 0 if cu is None else len(x.cu_seqlens) - 1
        nseq = ns if cu is not None else Bc
        ws = torch.empty(gdn2.workspace_size(Bc, Tc, Hc, DK, DV, io_c, ns), dtype=torch.uint8, device=dev)
        o = torch.empty_like(v)
        hT = torch.empty((nseq, Hc, DK, DV), dtype=f32, device=dev)

        if segmented:
            ws = torch.empty(gdn2.segmented_workspace_size(Bc, Tc, Hc, DK, DV, gdn2.GDN2_IO_BF16, ns), dtype=torch.uint8,
                             device=dev)

        def run():
            if segmented:
                gdn2.chunk_fwd_segmented(q, k, v, la, b, w, x.scale, h0=h0, cu_seqlens=cu, out=o, hT=hT,
                                         workspace=ws, stream=stream)
            else:
                gdn2.chunk_fwd(q, k, v, la, b, w, x.scale, h0=h0, cu_seqlens=cu, out=o, hT=hT, workspace=ws,
                               stream=stream)
        for _ in range(3):
            run()
        times = []
        for _ in range(steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            run()
            e1.record(stream)
            e1.synchronize()
            times.append(e0.elapsed_time(e1))
        ms = statistics.median(times)
        tokens = Bc * Tc
        per_th = ALG_BYTES_PER_TH if iot == "bf16" else 3 * DK * 4 + 3 * DK * 4 + DV * 4
        alg = tokens * Hc * per_th + nseq * Hc * DK * DV * 4 * (2 if h0 is not None else 1)
        out_cfg[x.name] = {"tokens_per_s": tokens / (ms / 1e3), "ms_per_step": ms,
                           "roofline_frac": (alg / (hbm * 1e9)) / (ms / 1e3)}
        del q, k, v, la, b, w, h0, cu, ws, o, hT
    return out_cfg


def ncu_case():
    """A small case of the fused kernel for full ncu captures (B=1, T=4096,
    H=16, dk=dv=128, strong decay, seed 2: 1,024 (chunk, head) tasks, inputs
    and factors ~0.4 GB on the device, larger than L2): three gdn2_chunk_fwd
    calls, nothing timed."""
    import torch

    import gated_delta_rule_129_b200 as gdn2
    from workloads import make_inputs
    torch.cuda.set_device(0)
    x = make_inputs(1, 4096, 16, 128, 128, io="bf16", seed=2, decay="strong")
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dt)  # noqa: E731
    q, k, v = (t(a, torch.bfloat16) for a in (x.q, x.k, x.v))
    la, b, w = (t(a, torch.float32) for a in (x.log_alpha, x.b, x.w))
    ws = torch.empty(gdn2.workspace_size(1, 4096, 16, 128, 128, gdn2.GDN2_IO_BF16), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(v)
    hT = torch.empty((1, 16, 128, 128), dtype=torch.float32, device="cuda")
    for _ in range(3):
        gdn2.chunk_fwd(q, k, v, la, b, w, x.scale, out=out, hT=hT, workspace=ws)
    torch.cuda.synchronize()
    print("ncu case ok", float(out.float().abs().mean()))


def ncu_kernels():
    """One launch of each kernel of the library on a small case, for per-kernel
    ncu captures (nothing timed): the two stages of the chunked forward
    (B=1, T=4096, H=16, dk=dv=128, strong decay: inputs and factors larger
    than L2), the decode step on 256 states, the token path's prologue and
    epilogue, the two-level chunk scan, and the backward on T=1024."""
    import torch

    import gated_delta_rule_129_b200 as gdn2
    from workloads import decode_inputs, make_inputs
    torch.cuda.set_device(0)
    bf, f32 = torch.bfloat16, torch.float32
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dt)  # noqa: E731
    x = make_inputs(1, 4096, 16, 128, 128, io="bf16", seed=2, decay="strong")
    q, k, v = (t(a, bf) for a in (x.q, x.k, x.v))
    la, b, w = (t(a, f32) for a in (x.log_alpha, x.b, x.w))
    ws = torch.empty(gdn2.workspace_size(1, 4096, 16, 128, 128), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(v)
    hT = torch.empty((1, 16, 128, 128), dtype=f32, device="cuda")
    gdn2.chunk_prep(q, k, v, la, b, w, workspace=ws)
    gdn2.chunk_walk(ws, (1, 4096, 16, 128, 128), bf, x.scale, out=out, hT=hT)
    di = decode_inputs(B=256, H=16, dk=128, dv=128, io="bf16", seed=41)
    state = t(di.state, f32)
    gdn2.recurrent_step(t(di.q, bf), t(di.k, bf), t(di.v, bf), t(di.log_alpha, f32), t(di.b, f32), t(di.w, f32),
                        di.scale, state)
    wconv = torch.full((16 * 128, 4), 0.25, device="cuda")
    q2, k2, v2 = gdn2.token_prologue(q, k, v, wconv, wconv, wconv)
    gdn2.token_epilogue(out, v, torch.ones(128, device="cuda"), out=out)
    gdn2.chunk_fwd_segmented(q, k, v, la, b, w, x.scale, segment_chunks=16)
    xs = make_inputs(1, 1024, 16, 128, 128, io="bf16", seed=3, decay="strong")
    gdn2.chunk_bwd(*(t(a, bf) for a in (xs.q, xs.k, xs.v)), *(t(a, f32) for a in (xs.log_alpha, xs.b, xs.w)),
                   xs.scale, t(xs.v, bf))
    torch.cuda.synchronize()
    print("ncu kernels ok", float(out.float().abs().mean()), float(q2.float().abs().mean()))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-configs", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--ncu-case", action="store_true",
                    help="run the small fused-kernel case for ncu captures and exit")
    ap.add_argument("--ncu-kernels", action="store_true",
                    help="run one launch of each kernel on small cases for ncu captures and exit")
    args = ap.parse_args()
    if args.ncu_case:
        ncu_case()
        return
    if args.ncu_kernels:
        ncu_kernels()
        return
    args.warmup = max(3, args.warmup)
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", 0))
        run_reference(args, rank)
        return
    rank, world, local = dist_setup(args.gpus)
    try:
        run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
