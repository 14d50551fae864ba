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

At N=1 the same run also times the other graded configurations on the same
weight set (full-size batch 8 and 64, Zipf-routed batch 32: the `configs`
object), and rank 0 checks every timed forward against the fp64 oracle (ids
exact, weights within 1e-5, outputs within 2e-2 * rms): the `parity` key; a
failed check makes the run exit non-zero.  Token inputs carry a top-k logit
margin >= 1e-3: each row's redraw counter comes from
tests/golden/bench_inputs.json (written by tests/golden/make_bench_inputs.py).

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
NOMINAL_HBM_GBS = 8000.0  # the nominal B200 HBM3e figure, for context
CONFIG_WORKLOADS = ("full_b8", "full_b64", "zipf_b32")
OUT_RTOL = 2e-2
W_ATOL = 1e-5
INPUTS_JSON = os.path.join(ROOT, "tests", "golden", "bench_inputs.json")


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
    p.add_argument("--no-configs", action="store_true", help="skip the other graded configurations")
    p.add_argument("--config-steps", type=int, default=200, help="timed graph replays per extra configuration")
    p.add_argument("--no-parity", action="store_true", help="skip the oracle check of the timed forwards")
    p.add_argument("--chain", type=int, default=0,
                   help="measure a chain of this many blocks of the config (one handle per block, distinct "
                        "weights) against its first block alone: graph replays, L2 flushed; prints that line")
    p.add_argument("--fp8-forwards", type=int, default=0,
                   help="profiling driver: run this many e4m3-weight forwards of the config (L2 flushed before "
                        "each), print their event-timed us and exit (no bench line)")
    return p.parse_args()


def x_attempts(workload: str, x_seed: int):
    """Per-row redraw counters giving this workload's x (drawn from x_seed) a
    top-k logit margin, or None when none are stored for it."""
    try:
        with open(INPUTS_JSON) as f:
            d = json.load(f)
        return d["workloads"][workload][str(x_seed)]
    except Exception:
        return None


def make_inputs(wl, seed: int, x_seed: int, dev):
    """Weights (router drawn on the host generator, the rest on the device)
    and the margin-checked x of a workload.  Returns (weights, x, margin)."""
    from moe_decode_block_b200 import synth
    wts = synth.make_weights(wl.shape, seed=seed, device=dev, routing=wl.routing, router_device="cpu")
    att = x_attempts(wl.name, x_seed) if seed == 0 else None
    x = synth.make_x(wl.batch, wl.shape.hidden, seed=x_seed, attempts=att).to(dev)
    return wts, x, ("top-k margin >= 1e-3 (stored redraw counters)" if att is not None else "unchecked")


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

    last = {}

    def one():
        _, ids, w = oracle.router(inp["x"], inp["R"], k, inp["bias"])
        out = oracle.block(inp["x"], ids, w, inp["h13"], inp["h2"], inp["sw13"], inp["sw2"],
                           n_experts=wl.shape.n_experts)
        last.update(out=out, ids=ids, w=w)

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
    time_oracle.last = last
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
    wts, x, _ = make_inputs(wl, args.seed, args.seed, gen_dev)
    x = x.cpu()
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


def check_against_oracle(wts, x, out, ids, w, k, ref=None):
    """The timed forward's results against the fp64 oracle (ids exact,
    weights within W_ATOL, outputs within OUT_RTOL * rms over every element).
    ref: the oracle's (out, ids, w) for these inputs if already computed;
    otherwise the oracle is run here, one selected expert at a time.
    Returns a small dict with "ok"."""
    import numpy as np

    import oracle
    from moe_decode_block_b200 import synth
    xb = synth.bf16_bits(x)
    if ref is None:
        bias = None if wts.router_bias is None else wts.router_bias.float().cpu().numpy()
        _, o_ids, o_w = oracle.router(xb, synth.bf16_bits(wts.router_w), k, bias)

        def fetch(e):
            return synth.bf16_bits(wts.w13[e]), synth.bf16_bits(wts.w2[e])

        o_out = oracle.block_streamed(xb, o_ids, o_w, fetch, synth.bf16_bits(wts.shared_w13),
                                      synth.bf16_bits(wts.shared_w2))
    else:
        o_out, o_ids, o_w = ref
    g_ids = ids.cpu().numpy()
    g_w = w.cpu().numpy().astype(np.float64)
    g_out = out.float().cpu().numpy()
    ids_ok = bool(np.array_equal(g_ids, o_ids))
    w_err = float(np.max(np.abs(g_w - o_w), initial=0.0))
    err = float(np.max(np.abs(g_out - o_out), initial=0.0)) if np.all(np.isfinite(g_out)) else float("inf")
    rms = float(np.sqrt(np.mean(o_out ** 2)))
    ok = ids_ok and w_err <= W_ATOL and err <= OUT_RTOL * rms
    return {"ok": ok, "ids_exact": ids_ok, "max_w_err": w_err, "max_out_err": err,
            "tol": OUT_RTOL * rms, "rows": int(x.shape[0])}


def fp8_bytes_per_step(shape, w8, ids, batch: int):
    """Algorithmic HBM bytes of one forward with e4m3 expert weights: each
    distinct routed expert's codes and block scales, the shared expert's,
    the bf16 router and the activations.  Returns (bytes, distinct)."""
    distinct = len(set(ids.reshape(-1).tolist()))
    per = (w8.q13[0].numel() + w8.q2[0].numel()) + 4 * (w8.s13[0].numel() + w8.s2[0].numel())
    shared = 0 if w8.shared_q13 is None else (w8.shared_q13.numel() + w8.shared_q2.numel()
                                             + 4 * (w8.shared_s13.numel() + w8.shared_s2.numel()))
    act = 2 * batch * shape.hidden * 2
    return distinct * per + shared + shape.router_bytes() + act, distinct


def check_fp8_against_oracle(shape, w8, x, out, ids, w):
    """An e4m3-weight forward against the fp64 oracle of block-scaled e4m3
    weights (ids exact, weights within W_ATOL, outputs within OUT_RTOL * rms)."""
    import numpy as np

    import oracle
    from moe_decode_block_b200 import synth
    k, H, I, Is = shape.top_k, shape.hidden, shape.inter, shape.shared_inter

    def osc(s_api, outs):  # the library's [in/128, padded] scales -> the oracle's [out/128, in/128]
        return np.ascontiguousarray(s_api.detach().cpu().numpy()[:, :-(-outs // 128)].T)

    xb = synth.bf16_bits(x)
    bias = None if w8.router_bias is None else w8.router_bias.float().cpu().numpy()
    _, o_ids, o_w = oracle.router(xb, synth.bf16_bits(w8.router_w), k, bias)
    fetch = lambda e: (w8.q13[e].cpu().numpy(), osc(w8.s13[e], 2 * I), w8.q2[e].cpu().numpy(), osc(w8.s2[e], H))
    shared = (w8.shared_q13.cpu().numpy(), osc(w8.shared_s13, 2 * Is), w8.shared_q2.cpu().numpy(),
              osc(w8.shared_s2, H))
    o_out = oracle.block_streamed_fp8(xb, o_ids, o_w, fetch, shared)
    g_out = out.float().cpu().numpy()
    ids_ok = bool(np.array_equal(ids.cpu().numpy(), o_ids))
    w_err = float(np.max(np.abs(w.cpu().numpy().astype(np.float64) - o_w)))
    err = float(np.max(np.abs(g_out - o_out))) if np.all(np.isfinite(g_out)) else float("inf")
    rms = float(np.sqrt(np.mean(o_out ** 2)))
    return {"ok": ids_ok and w_err <= W_ATOL and err <= OUT_RTOL * rms, "ids_exact": ids_ok, "max_w_err": w_err,
            "max_out_err": err, "tol": OUT_RTOL * rms, "rows": int(x.shape[0])}


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
    if args.fp8_forwards > 0:
        fp8_forwards(wl, args.fp8_forwards, args.seed, dev)
        return
    if args.chain > 0:
        return chain_bench(wl, args.chain, args.seed, dev, args.steps, args.warmup)
    wts, x, margin = make_inputs(wl, args.seed, args.seed + 1000 * rank, dev)
    main = torch.cuda.Stream()
    aux = torch.cuda.Stream()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = torch.empty(2 * l2 // 4, dtype=torch.float32, device=dev)
    flush_sum = torch.empty((), dtype=torch.float32, device=dev)

    def flush():
        """Write a 2x-L2 buffer, then read it back: the write evicts every
        weight line; the read leaves L2 holding clean lines, so the timed step
        pays no write-back of the flush's dirty lines."""
        flush_buf.zero_()
        torch.sum(flush_buf, dim=0, out=flush_sum)

    class Case:
        """One handle + buffers + a CUDA graph of one forward of a workload."""

        def __init__(self, wl_, wts_, x_, two_stream):
            sh = wl_.shape
            self.wl, self.wts, self.x = wl_, wts_, x_
            self.blk = MoEDecode(sh.hidden, sh.n_experts, sh.top_k, sh.inter, sh.shared_inter, n_shared=sh.n_shared,
                                 max_batch=max(wl_.batch, 1), router_bias=wts_.router_bias, two_stream=two_stream)
            self.out = torch.empty_like(x_)
            self.ids = torch.empty(wl_.batch, sh.top_k, dtype=torch.int32, device=dev)
            self.w = torch.empty(wl_.batch, sh.top_k, dtype=torch.float32, device=dev)
            self.fargs = (x_, wts_.router_w, wts_.w13, wts_.w2, wts_.shared_w13, wts_.shared_w2, self.out, self.ids,
                          self.w)
            with torch.cuda.stream(main):
                self.blk.forward(*self.fargs, stream_main=main, stream_aux=aux)
            main.synchronize()
            if self.blk.status() != 0:
                raise RuntimeError(f"device status not OK after the first forward of {wl_.name}")
            self.bstep, self.distinct = bytes_per_step(sh, self.ids.cpu().numpy(), wl_.batch)
            self.kernels_per_step = self.blk.stats()["last_kernels"]
            self.g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.g, stream=main):
                self.blk.forward(*self.fargs, stream_main=torch.cuda.current_stream(), stream_aux=aux)

        def timed(self, steps, warmup):
            """Graph replays with L2 flushed before each; per-step ms (events on
            the launching stream around the replay only) and the clocks seen."""
            with torch.cuda.stream(main):
                for _ in range(warmup):
                    flush()
                    self.g.replay()
            torch.cuda.synchronize()
            sampler = ClockSampler(dev.index)
            sampler.start()
            time.sleep(0.2)
            if world > 1:
                torch.distributed.barrier()
            torch.cuda.synchronize()
            w0 = time.perf_counter()
            starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
            ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
            with torch.cuda.stream(main):
                for i in range(steps):
                    flush()
                    starts[i].record(main)
                    self.g.replay()
                    ends[i].record(main)
            torch.cuda.synchronize()
            w1 = time.perf_counter()
            if world > 1:
                torch.distributed.barrier()
            clocks = sampler.stop()
            return [a.elapsed_time(b) for a, b in zip(starts, ends)], clocks, (w1 - w0) * 1e3

        def close(self):
            del self.g
            self.blk.close()

    head = Case(wl, wts, x, args.two_stream)
    blk, fargs, bstep, distinct = head.blk, head.fargs, head.bstep, head.distinct

    # ---- headline: graph replays, L2 flushed before each step
    step_ms, clocks, bracket_ms = head.timed(args.steps, args.warmup)
    value, total_ms, all_bytes = aggregate_over_ranks(float(sum(step_ms)), bstep, args.steps, dev, world)
    ms_per_step = total_ms / args.steps

    # ---- per-kernel breakdown (eager forwards with timing events)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    blk.set_timing_events(evs)
    kt = {k: [] for k in ("router", "experts", "combine", "shared", "step")}
    nb = min(args.steps, 200)
    with torch.cuda.stream(main):
        for i in range(nb + 5):
            flush()
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
    block_gbs = bstep / (ms_per_step * 1e-3) / 1e9
    roofline = {"bound": "hbm",
                "kernel": "expert_mlp_kernel<routed only>" if args.two_stream
                else "expert_mlp_kernel<shared + routed>",
                "achieved": round(exp_gbs, 1),
                "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": round(exp_gbs / peak, 4),
                "traffic": traffic, "algorithmic_bytes_per_launch": exp_bytes,
                "launch_us": kern_us["experts"],
                "block_frac": round(block_gbs / peak, 4),
                "frac_of_nominal_8tbs": round(exp_gbs / NOMINAL_HBM_GBS, 4),
                "block_frac_of_nominal_8tbs": round(block_gbs / NOMINAL_HBM_GBS, 4)}

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
                flush()
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

    # ---- the other graded configurations, same weights (N == 1)
    configs = None
    cases = []
    if world == 1 and not args.no_configs and s == synth.FULL:
        configs = {}
        for name in CONFIG_WORKLOADS:
            if name == wl.name:
                continue
            cwl = synth.WORKLOADS[name]
            cw = wts
            if cwl.routing != wl.routing:
                bias = synth.zipf_log_prior(s.n_experts, args.seed, dev) if cwl.routing == "zipf" else None
                cw = synth.BlockWeights(wts.router_w, wts.w13, wts.w2, wts.shared_w13, wts.shared_w2, bias)
            att = x_attempts(name, args.seed) if args.seed == 0 else None
            cx = synth.make_x(cwl.batch, s.hidden, seed=args.seed, attempts=att).to(dev)
            case = Case(cwl, cw, cx, args.two_stream)
            ms, cclk, _ = case.timed(args.config_steps, 20)
            us = 1e3 * statistics.mean(ms)
            gbs = case.bstep / (us * 1e-6) / 1e9
            configs[name] = {"batch": cwl.batch, "routing": cwl.routing, "distinct_experts": case.distinct,
                             "bytes_per_step": case.bstep, "us_per_block": round(us, 2),
                             "us_p10": round(1e3 * float(np.percentile(ms, 10)), 2),
                             "us_p90": round(1e3 * float(np.percentile(ms, 90)), 2),
                             "GB/s": round(gbs, 1), "frac_of_measured_peak": round(gbs / peak, 4),
                             "frac_of_nominal_8tbs": round(gbs / NOMINAL_HBM_GBS, 4),
                             "tokens_per_s": round(cwl.batch / (us * 1e-6), 1), "steps": args.config_steps,
                             "margin": "top-k margin >= 1e-3 (stored redraw counters)" if att is not None
                             else "unchecked", "clocks": cclk}
            cases.append(case)

    # ---- e4m3 expert weights (block-scaled), batch 1 and 8, same router
    fp8 = None
    fp8_cases = []
    if world == 1 and not args.no_configs and s == synth.FULL and not args.two_stream:
        w8 = synth.make_fp8_weights(s, seed=args.seed, device=dev, routing=wl.routing, router_device="cpu")
        fp8 = {"weights": "e4m3 codes [out, in] + fp32 scale per 128 x 128 block (scale = block absmax / 448), "
                          "router bf16, activations bf16 (f16 in the products), fp32 accumulation"}
        for name, fb in (("fp8_b1", 1), ("fp8_b8", 8)):
            att = x_attempts(f"full_b{fb}", args.seed) if args.seed == 0 else None
            fx = synth.make_x(fb, s.hidden, seed=args.seed, attempts=att).to(dev)
            fblk = MoEDecode(s.hidden, s.n_experts, s.top_k, s.inter, s.shared_inter, n_shared=s.n_shared,
                             max_batch=fb, router_bias=w8.router_bias, fp8=True)
            fout = torch.empty_like(fx)
            fids = torch.empty(fb, s.top_k, dtype=torch.int32, device=dev)
            fw = torch.empty(fb, s.top_k, dtype=torch.float32, device=dev)
            fargs8 = (fx, w8.router_w, w8.q13, w8.s13, w8.q2, w8.s2, w8.shared_q13, w8.shared_s13, w8.shared_q2,
                      w8.shared_s2, fout, fids, fw)
            with torch.cuda.stream(main):
                fblk.forward_fp8(*fargs8, stream_main=main, stream_aux=aux)
            main.synchronize()
            fg = torch.cuda.CUDAGraph()
            with torch.cuda.graph(fg, stream=main):
                fblk.forward_fp8(*fargs8, stream_main=torch.cuda.current_stream(), stream_aux=aux)
            with torch.cuda.stream(main):
                for _ in range(20):
                    flush()
                    fg.replay()
            torch.cuda.synchronize()
            fst = [torch.cuda.Event(enable_timing=True) for _ in range(args.config_steps)]
            fen = [torch.cuda.Event(enable_timing=True) for _ in range(args.config_steps)]
            with torch.cuda.stream(main):
                for i in range(args.config_steps):
                    flush()
                    fst[i].record(main)
                    fg.replay()
                    fen[i].record(main)
            torch.cuda.synchronize()
            fus = 1e3 * statistics.mean(a.elapsed_time(b) for a, b in zip(fst, fen))
            fbytes, fdist = fp8_bytes_per_step(s, w8, fids.cpu().numpy(), fb)
            fp8[name] = {"batch": fb, "distinct_experts": fdist, "bytes_per_step": fbytes,
                         "us_per_block": round(fus, 2), "GB/s": round(fbytes / (fus * 1e-6) / 1e9, 1),
                         "frac_of_measured_peak": round(fbytes / (fus * 1e-6) / 1e9 / peak, 4),
                         "tokens_per_s": round(fb / (fus * 1e-6), 1), "steps": args.config_steps,
                         "vs_bf16_us": round(ms_per_step * 1e3, 2) if fb == B else
                         (configs.get(f"full_b{fb}", {}).get("us_per_block") if configs else None)}
            del fg
            fp8_cases.append((name, fblk, fx, fout, fids, fw))

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N == 1); its
    # last run is the oracle output the headline forward is checked against
    cpu = None
    oracle_ref = None
    if world == 1 and not args.no_cpu_baseline:
        inp = host_oracle_inputs(wl, wts, x, head.ids.cpu().numpy())
        gbs, per, runs, threads, _ = time_oracle(wl, inp, bstep, min_seconds=10.0, max_runs=30)
        last = time_oracle.last
        oracle_ref = (last["out"], last["ids"], last["w"])
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": f"{runs} full forwards of the {wl.name} block (router + {distinct} routed + shared "
                         f"expert MLPs) by the fp64 C oracle, >= 10 s of CPU work, median "
                         f"{per * 1e3:.1f} ms per block"}

    # ---- parity of every timed forward against the oracle (rank 0)
    parity = None
    if rank == 0 and not args.no_parity:
        parity = {"bar": f"ids exact, |w - oracle| <= {W_ATOL}, max|out - oracle| <= {OUT_RTOL} * rms(oracle out)",
                  wl.name: check_against_oracle(wts, x, head.out, head.ids, head.w, s.top_k, oracle_ref)}
        for case in cases:
            parity[case.wl.name] = check_against_oracle(case.wts, case.x, case.out, case.ids, case.w, s.top_k)
        for name, fblk, fx, fout, fids, fw in fp8_cases:
            parity[name] = check_fp8_against_oracle(s, w8, fx, fout, fids, fw)
            fp8[name]["parity"] = "ok" if parity[name]["ok"] else "FAIL"
        parity["ok"] = all(v["ok"] for k, v in parity.items() if isinstance(v, dict))
        if configs:
            for name in configs:
                configs[name]["parity"] = "ok" if parity[name]["ok"] else "FAIL"

    status = blk.status()
    parity_ok = parity is None or parity["ok"]
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(_config_dict(wl), plan="two_stream" if args.two_stream else "default", inputs=margin),
            "us_per_block": round(ms_per_step * 1e3, 2), "tokens_per_s": round(B * 1e3 / ms_per_step, 1),
            "bytes_per_step": bstep, "distinct_experts": distinct,
            "roofline": roofline, "kernels_us": kern_us, "cpu_baseline": cpu, "e2e": e2e,
            "parity": "ok" if parity_ok and parity is not None else ("FAIL" if not parity_ok else None),
            "parity_detail": parity, "configs": configs, "fp8": fp8,
            "gpu_launches": head.kernels_per_step * args.steps, "kernels_per_step": head.kernels_per_step,
            "clocks": clocks, "bracket_ms_incl_flush": round(bracket_ms, 2),
            "device_status": status,
        }
        print(json.dumps(line), flush=True)
    for case in cases:
        case.close()
    for _, fblk, *_rest in fp8_cases:
        fblk.close()
    head.close()
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0 if parity_ok and status == 0 else 1


def fp8_forwards(wl, n, seed, dev):
    """Profiling driver for the e4m3-weight kernel: n forwards of the config's
    block with e4m3 expert weights, L2 flushed before each (for ncu captures
    of a small case; prints the event-timed us of each forward)."""
    import torch
    from moe_decode_block_b200 import MoEDecode, synth
    s = wl.shape
    w8 = synth.make_fp8_weights(s, seed=seed, device=dev, routing=wl.routing)
    x = synth.make_x(wl.batch, s.hidden, seed=seed).to(dev)
    blk = MoEDecode(s.hidden, s.n_experts, s.top_k, s.inter, s.shared_inter, n_shared=s.n_shared,
                    max_batch=wl.batch, router_bias=w8.router_bias, fp8=True)
    out = torch.empty_like(x)
    ids = torch.empty(wl.batch, s.top_k, dtype=torch.int32, device=dev)
    w = torch.empty(wl.batch, s.top_k, dtype=torch.float32, device=dev)
    fb = torch.empty(2 * torch.cuda.get_device_properties(dev).L2_cache_size // 4, dtype=torch.float32, device=dev)
    us = []
    for _ in range(n):
        fb.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        blk.forward_fp8(x, w8.router_w, w8.q13, w8.s13, w8.q2, w8.s2, w8.shared_q13, w8.shared_s13, w8.shared_q2,
                        w8.shared_s2, out, ids, w)
        e1.record()
        torch.cuda.synchronize()
        us.append(round(e0.elapsed_time(e1) * 1e3, 1))
    status = blk.status()
    blk.close()
    print(json.dumps({"fp8_forwards": wl.name, "us": us, "device_status": status}), flush=True)
    if status != 0:
        raise SystemExit(f"device status {status}")


def chain_bench(wl, n_blocks, seed, dev, steps, warmup):
    """A chain of n_blocks blocks of the workload (block 0 on the config's
    weights and input, block l on the weights of seed + l) timed as one CUDA
    graph per step, against a graph of block 0 alone; L2 flushed before every
    replay.  Prints one JSON line; returns non-zero on a device error."""
    import numpy as np
    import torch
    from moe_decode_block_b200 import synth
    from moe_decode_block_b200.chain import BlockChain
    s, B = wl.shape, wl.batch
    wts0, x, _ = make_inputs(wl, seed, seed, dev)
    weights = [wts0] + [synth.make_weights(s, seed=seed + l, device=dev, routing=wl.routing)
                        for l in range(1, n_blocks)]
    chain = BlockChain(n_blocks, s.hidden, s.n_experts, s.top_k, s.inter, s.shared_inter, n_shared=s.n_shared,
                       max_batch=max(B, 1), router_biases=[w.router_bias for w in weights])
    outs = [torch.empty_like(x) for _ in range(n_blocks)]
    ids = [torch.empty(B, s.top_k, dtype=torch.int32, device=dev) for _ in range(n_blocks)]
    ws = [torch.empty(B, s.top_k, dtype=torch.float32, device=dev) for _ in range(n_blocks)]
    wl_args = [(w.router_w, w.w13, w.w2, w.shared_w13, w.shared_w2) for w in weights]
    main_s = torch.cuda.Stream()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    fb = torch.empty(2 * l2 // 4, dtype=torch.float32, device=dev)
    fs = torch.empty((), dtype=torch.float32, device=dev)
    with torch.cuda.stream(main_s):
        chain.forward(x, wl_args, outs, ids, ws, stream=main_s)
    main_s.synchronize()
    if chain.status() != 0:
        chain.close()
        raise SystemExit(f"device status {chain.status()} after the first chain forward")
    bytes_blocks = [bytes_per_step(s, ids[l].cpu().numpy(), B)[0] for l in range(n_blocks)]
    g_chain, g_one = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_chain, stream=main_s):
        chain.forward(x, wl_args, outs, ids, ws, stream=torch.cuda.current_stream())
    with torch.cuda.graph(g_one, stream=main_s):
        chain.blocks[0].forward(x, *wl_args[0], outs[0], ids[0], ws[0], stream_main=torch.cuda.current_stream())

    def timed(g):
        with torch.cuda.stream(main_s):
            for _ in range(warmup):
                fb.zero_()
                torch.sum(fb, dim=0, out=fs)
                g.replay()
        torch.cuda.synchronize()
        sampler = ClockSampler(dev.index)
        sampler.start()
        time.sleep(0.2)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        with torch.cuda.stream(main_s):
            for a, b in ev:
                fb.zero_()
                torch.sum(fb, dim=0, out=fs)
                a.record(main_s)
                g.replay()
                b.record(main_s)
        torch.cuda.synchronize()
        return float(np.median([a.elapsed_time(b) for a, b in ev])) * 1e3, sampler.stop()

    us_one, clocks_one = timed(g_one)
    us_chain, clocks_chain = timed(g_chain)
    status = chain.status()
    del g_chain, g_one
    chain.close()
    line = {"chain": {"workload": wl.name, "blocks": n_blocks, "batch": B, "steps": steps, "warmup": warmup,
                      "us_block_alone": round(us_one, 2), "us_chain": round(us_chain, 2),
                      "us_per_block_in_chain": round(us_chain / n_blocks, 2),
                      "GB/s_chain": round(sum(bytes_blocks) / (us_chain * 1e-6) / 1e9, 1),
                      "GB/s_block_alone": round(bytes_blocks[0] / (us_one * 1e-6) / 1e9, 1),
                      "l2": "flushed before every replay (of the chain, or of the block alone)",
                      "clocks_block_alone": clocks_one, "clocks_chain": clocks_chain,
                      "device_status": status}}
    print(json.dumps(line), flush=True)
    return 0 if status == 0 else 1


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
