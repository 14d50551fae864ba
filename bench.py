#!/usr/bin/env python
"""Benchmark: MoE decode block on B200 -- microseconds per block and achieved
HBM GB/s of the distinct weights touched, against the measured B200 peak.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config full_b1] [--impl reference]

A step is one forward of the whole block (router + top-k + bucketing, shared
expert, routed SwiGLU experts, combine + residual) over one batch of
synthetic tokens, in the library's default plan (router kernel, one expert
kernel for the shared and the routed experts, combine kernel); --two-stream
times the plan with the shared expert on the aux stream instead.  Default
workload: the full-size block at batch 1 (hidden 7168, 384 experts top-8,
inter 2048, one shared expert).

Timing: the forward is captured once in a CUDA graph (both streams) and
replayed; L2 is flushed (a 2x-L2 write) before every step and each step is
bracketed by CUDA events on the launching stream, so the flush is not timed.
`value` = bytes of distinct weights touched (+ router, shared, activations)
per step x steps x ranks / max-over-ranks device time.  Under torchrun every
rank runs an independent replica of the block on its own batch (weak scaling,
no collective on the data path).

--impl reference times the fp64 CPU oracle on the host cores instead.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE decode block µs and achieved HBM GB/s vs B200 peak, batch 1–64, 1 GPU"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=3000)
    p.add_argument("--warmup", type=int, default=50)
    p.add_argument("--config", default="full_b1")
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--two-stream", action="store_true",
                   help="time the plan with the shared expert on the aux stream (MOE_FLAG_TWO_STREAM)")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def code_only(text: str) -> str:
    """C/C++/CUDA source without its comments, trailing blanks and empty lines:
    what the compiler sees, so that editing a comment keeps a capture valid."""
    out = []
    i, n = 0, len(text)
    while i < n:
        c = text[i]
        if text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            out.append(c)
            i += 1
    lines = (line.rstrip() for line in "".join(out).split("\n"))
    return "\n".join(line for line in lines if line)


def kernel_sources_sha() -> str:
    """Hash of the library's CUDA sources (code only, comments excluded)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "moe_decode_block_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, name), encoding="utf-8") as f:
                h.update(name.encode() + b"\0" + code_only(f.read()).encode())
    return h.hexdigest()


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or
    None if there is none or the kernel sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    ent = d.get(f"{kernel}/{workload}")
    if not ent or ent.get("sources_sha256") != kernel_sources_sha():
        return None
    return float(ent["dram_bytes_per_launch"])


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            self.path = os.path.join("/tmp", f"moe_clocks_{os.getpid()}.csv")
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ----------------------------------------------------------------- helpers --

def bytes_per_step(shape, ids, batch: int) -> tuple[int, int]:
    """Algorithmic HBM bytes of one forward: distinct routed experts' weights +
    shared expert + router + x read + out written.  Returns (bytes, distinct)."""
    distinct = len(set(ids.reshape(-1).tolist()))
    act = 2 * batch * shape.hidden * 2
    return distinct * shape.expert_bytes() + shape.shared_bytes() + shape.router_bytes() + act, distinct


def aggregate_over_ranks(total_ms: float, bytes_per_step: float, steps: int, device, world: int):
    """Whole-job throughput of independent replicas: bytes summed over ranks,
    time = the slowest rank's device time (all_reduce MAX).  Returns
    (value GB/s, max_total_ms, all_bytes).  Collective calls are the same on
    every rank, in the same order."""
    import torch
    if world > 1:
        t = torch.tensor([float(total_ms)], device=device, dtype=torch.float64)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        total_ms = float(t.item())
        bt = torch.tensor([float(bytes_per_step)], device=device, dtype=torch.float64)
        torch.distributed.all_reduce(bt)
        all_bytes = float(bt.item()) * steps
    else:
        all_bytes = float(bytes_per_step) * steps
    return all_bytes / (total_ms / 1e3) / 1e9, total_ms, all_bytes


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def host_oracle_inputs(wl, wts, x, ids_np):
    from moe_decode_block_b200 import synth
    E = wl.shape.n_experts
    h13 = [None] * E
    h2 = [None] * E
    for e in sorted(set(ids_np.reshape(-1).tolist())):
        h13[e] = synth.bf16_bits(wts.w13[e])
        h2[e] = synth.bf16_bits(wts.w2[e])
    bias = None if wts.router_bias is None else wts.router_bias.float().cpu().numpy()
    return dict(x=synth.bf16_bits(x), R=synth.bf16_bits(wts.router_w), h13=h13, h2=h2,
                sw13=synth.bf16_bits(wts.shared_w13), sw2=synth.bf16_bits(wts.shared_w2), bias=bias)


def time_oracle(wl, inp, bytes_step, min_seconds=10.0, max_runs=30, warmup=1, max_seconds=None, warmup_seconds=None):
    """The fp64 oracle, as it stands, on the host cores: router + block for
    the whole batch per run.  Returns (GB/s, seconds per run, runs, threads,
    warm-up runs done); warm-up stops early after warmup_seconds."""
    import oracle
    k = wl.shape.top_k

    def one():
        _, ids, w = oracle.router(inp["x"], inp["R"], k, inp["bias"])
        oracle.block(inp["x"], ids, w, inp["h13"], inp["h2"], inp["sw13"], inp["sw2"], n_experts=wl.shape.n_experts)

    done_warmup = 0
    t_w = time.perf_counter()
    for _ in range(warmup):
        one()
        done_warmup += 1
        if warmup_seconds is not None and time.perf_counter() - t_w >= warmup_seconds:
            break
    times = []
    t_start = time.perf_counter()
    while len(times) < max_runs:
        t0 = time.perf_counter()
        one()
        times.append(time.perf_counter() - t0)
        el = time.perf_counter() - t_start
        if el >= min_seconds and len(times) >= 3:
            break
        if max_seconds is not None and el >= max_seconds:
            break
    per = statistics.median(times)
    return bytes_step / per / 1e9, per, len(times), oracle.num_threads(), done_warmup


# -------------------------------------------------------------------- arms --

def run_reference(args):
    """CPU oracle arm: rank 0 only; other ranks exit without work."""
    world, rank, _ = dist_setup()
    if rank != 0:
        return 0
    import torch

    from moe_decode_block_b200 import synth
    wl = synth.WORKLOADS[args.config]
    # the same seeded generator as the CUDA arm (on the GPU when there is one:
    # drawing 34 GB of full-size weights on the host is slow); only the
    # touched experts are copied to the host for the oracle
    gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
    wts = synth.make_weights(wl.shape, seed=args.seed, device=gen_dev, routing=wl.routing)
    x = synth.make_x(wl.batch, wl.shape.hidden, seed=args.seed)
    import oracle
    bias = None if wts.router_bias is None else wts.router_bias.float().cpu().numpy()
    _, ids, _ = oracle.router(synth.bf16_bits(x), synth.bf16_bits(wts.router_w), wl.shape.top_k, bias)
    bstep, distinct = bytes_per_step(wl.shape, ids, wl.batch)
    inp = host_oracle_inputs(wl, wts, x, ids)
    budget = 120.0
    gbs, per, runs, threads, warm = time_oracle(wl, inp, bstep, min_seconds=float("inf"),
                                                max_runs=max(1, args.steps), warmup=args.warmup,
                                                max_seconds=budget, warmup_seconds=30.0)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": args.gpus,
        "steps": runs, "steps_requested": args.steps, "warmup": warm, "warmup_requested": args.warmup,
        "ms_per_step": round(per * 1e3, 3), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": _config_dict(wl, graph=False),
        "us_per_block": round(per * 1e6, 1), "bytes_per_step": bstep, "distinct_experts": distinct,
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": f"{runs} full forwards of the {wl.name} block (router + {distinct} routed + "
                                   f"shared expert MLPs), fp64 C oracle, wall-clock median, capped at "
                                   f"{int(budget)} s"},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _config_dict(wl, graph=True):
    s = wl.shape
    return {"workload": wl.name, "batch": wl.batch, "hidden": s.hidden, "n_experts": s.n_experts,
            "top_k": s.top_k, "inter": s.inter, "shared_inter": s.shared_inter, "n_shared": s.n_shared,
            "routing": wl.routing, "weights": "bf16 ~N(0,0.02), x bf16 ~N(0,1), seeded",
            "l2": "flushed before every step (2x L2 write + read back, untimed)", "cuda_graph": graph,
            "parallelism": "replicas (one independent block per GPU)"}


def run_ours(args):
    import numpy as np
    import torch

    world, rank, local = dist_setup()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    from moe_decode_block_b200 import MoEDecode, synth
    from moe_decode_block_b200.build import build_library
    if rank == 0:
        build_library()
    if world > 1:
        torch.distributed.barrier()

    wl = synth.WORKLOADS[args.config]
    s = wl.shape
    B = wl.batch
    wts = synth.make_weights(s, seed=args.seed, device=dev, routing=wl.routing)
    x = synth.make_x(B, s.hidden, seed=args.seed + 1000 * rank).to(dev)
    blk = MoEDecode(s.hidden, s.n_experts, s.top_k, s.inter, s.shared_inter, n_shared=s.n_shared,
                    max_batch=max(B, 1), router_bias=wts.router_bias, two_stream=args.two_stream)
    out = torch.empty_like(x)
    ids = torch.empty(B, s.top_k, dtype=torch.int32, device=dev)
    w = torch.empty(B, s.top_k, dtype=torch.float32, device=dev)
    main = torch.cuda.Stream()
    aux = torch.cuda.Stream()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = torch.empty(2 * l2 // 4, dtype=torch.float32, device=dev)
    flush_sum = torch.empty((), dtype=torch.float32, device=dev)

    class _Flush:
        """Write a 2x-L2 buffer, then read it back: the write evicts every
        weight line; the read leaves L2 holding clean lines, so the timed step
        pays no write-back of the flush's dirty lines."""

        @staticmethod
        def zero_():
            flush_buf.zero_()
            torch.sum(flush_buf, dim=0, out=flush_sum)

    flush = _Flush()
    fargs = (x, wts.router_w, wts.w13, wts.w2, wts.shared_w13, wts.shared_w2, out, ids, w)

    with torch.cuda.stream(main):
        blk.forward(*fargs, stream_main=main, stream_aux=aux)
    main.synchronize()
    if blk.status() != 0:
        raise RuntimeError("device status not OK after the first forward")
    bstep, distinct = bytes_per_step(s, ids.cpu().numpy(), B)
    kernels_per_step = blk.stats()["last_kernels"]

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=main):
        blk.forward(*fargs, stream_main=torch.cuda.current_stream(), stream_aux=aux)

    def timed_loop(n, step_fn):
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        with torch.cuda.stream(main):
            for i in range(n):
                flush.zero_()
                starts[i].record(main)
                step_fn()
                ends[i].record(main)
        return starts, ends

    # ---- warm-up
    with torch.cuda.stream(main):
        for _ in range(args.warmup):
            flush.zero_()
            g.replay()
    torch.cuda.synchronize()

    # ---- headline: graph replays, L2 flushed before each step
    sampler = ClockSampler(dev.index)
    sampler.start()
    time.sleep(0.2)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    starts, ends = timed_loop(args.steps, g.replay)
    torch.cuda.synchronize()
    wall1 = time.perf_counter()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    value, total_ms, all_bytes = aggregate_over_ranks(float(sum(step_ms)), bstep, args.steps, dev, world)
    ms_per_step = total_ms / args.steps

    # ---- per-kernel breakdown (eager forwards with timing events)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    blk.set_timing_events(evs)
    kt = {k: [] for k in ("router", "experts", "combine", "shared", "step")}
    nb = min(args.steps, 200)
    with torch.cuda.stream(main):
        for i in range(nb + 5):
            flush.zero_()
            blk.forward(*fargs, stream_main=main, stream_aux=aux)
            main.synchronize()
            aux.synchronize()
            if i < 5:
                continue
            kt["router"].append(evs[0].elapsed_time(evs[1]))
            if args.two_stream:
                kt["experts"].append(evs[1].elapsed_time(evs[2]))
                kt["combine"].append(evs[2].elapsed_time(evs[3]))
                kt["shared"].append(evs[4].elapsed_time(evs[5]))
            else:  # one expert kernel: shared + routed experts
                kt["experts"].append(evs[4].elapsed_time(evs[5]))
                kt["combine"].append(evs[2].elapsed_time(evs[3]))
            kt["step"].append(evs[0].elapsed_time(evs[3]))
    blk.set_timing_events(None)
    kern_us = {k: round(1e3 * statistics.mean(v), 2) for k, v in kt.items() if v}
    peak, peak_kind = peaks()
    # dominant kernel: the expert kernel.  Default plan: shared expert + every
    # active routed expert (UP + SwiGLU + DOWN); two-stream plan: the routed
    # experts only.
    exp_bytes = distinct * s.expert_bytes() + (0 if args.two_stream else s.shared_bytes())
    exp_gbs = exp_bytes / (kern_us["experts"] * 1e-6) / 1e9
    kname = "expert_mlp_routed" if args.two_stream else "expert_mlp"
    traffic = ncu_traffic(kname, wl.name)
    roofline = {"bound": "hbm",
                "kernel": "expert_mlp_kernel<routed only>" if args.two_stream
                else "expert_mlp_kernel<shared + routed>",
                "achieved": round(exp_gbs, 1),
                "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": round(exp_gbs / peak, 4),
                "traffic": traffic, "algorithmic_bytes_per_launch": exp_bytes,
                "launch_us": kern_us["experts"],
                "block_frac": round((bstep / (ms_per_step * 1e-3) / 1e9) / peak, 4)}

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        xh = x.cpu().pin_memory()
        oh = torch.empty_like(xh).pin_memory()
        ih = torch.empty(B, s.top_k, dtype=torch.int32).pin_memory()
        wh = torch.empty(B, s.top_k, dtype=torch.float32).pin_memory()
        ne = min(args.steps, 500)
        times = []
        with torch.cuda.stream(main):
            for i in range(ne + 5):
                flush.zero_()
                main.synchronize()
                t0 = time.perf_counter()
                blk.forward_host(xh, wts.router_w, wts.w13, wts.w2, wts.shared_w13, wts.shared_w2, oh, ih, wh,
                                 stream_main=main, stream_aux=aux)
                t1 = time.perf_counter()
                if i >= 5:
                    times.append(t1 - t0)
        e2e_s = statistics.mean(times)
        e2e_val = bstep / e2e_s / 1e9
        if world > 1:
            t = torch.tensor([e2e_s], device=dev, dtype=torch.float64)
            torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
            e2e_val = bstep * world / float(t.item()) / 1e9
        e2e = {"value": round(e2e_val, 2), "unit": "GB/s", "us_per_block": round(e2e_s * 1e6, 1),
               "h2d_bytes_per_step": B * s.hidden * 2, "d2h_bytes_per_step": B * s.hidden * 2 + B * s.top_k * 8,
               "api": "moe_decode_forward_host (pinned host buffers: x copied in; out, topk_ids, topk_w "
                      "stored into them by the kernels; synchronous)"}

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N == 1)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        inp = host_oracle_inputs(wl, wts, x, ids.cpu().numpy())
        gbs, per, runs, threads, _ = time_oracle(wl, inp, bstep, min_seconds=10.0, max_runs=30)
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": f"{runs} full forwards of the {wl.name} block (router + {distinct} routed + shared "
                         f"expert MLPs) by the fp64 C oracle, >= 10 s of CPU work, median "
                         f"{per * 1e3:.1f} ms per block"}

    status = blk.status()
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(_config_dict(wl), plan="two_stream" if args.two_stream else "default"),
            "us_per_block": round(ms_per_step * 1e3, 2), "tokens_per_s": round(B * 1e3 / ms_per_step, 1),
            "bytes_per_step": bstep, "distinct_experts": distinct,
            "roofline": roofline, "kernels_us": kern_us, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": kernels_per_step * args.steps, "kernels_per_step": kernels_per_step,
            "clocks": clocks, "bracket_ms_incl_flush": round((wall1 - wall0) * 1e3, 2),
            "device_status": status,
        }
        print(json.dumps(line), flush=True)
    del g
    blk.close()
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
