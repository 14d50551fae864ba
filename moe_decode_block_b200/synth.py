"""Seeded synthetic inputs for the MoE decode block.

This module only draws random numbers; it holds none of the block's
arithmetic.  The tests, the smoke check and the benchmark all take their
inputs from here, so the CUDA path and the fp64 oracle always see the same
tensors.

Distributions: weights ~ N(0, 0.02) and activations ~ N(0, 1), both rounded
once (round-to-nearest-even) from float32 to bf16.  Every tensor (and every
expert, and every row of x) draws from its own generator whose seed is a hash
of (seed, tensor name, index), so any subset can be regenerated on its own.
"""
from __future__ import annotations

import dataclasses
import hashlib
import math
from typing import Dict, Optional, Sequence

import torch

WEIGHT_STD = 0.02
ZIPF_S = 1.2


@dataclasses.dataclass(frozen=True)
class BlockShape:
    hidden: int
    n_experts: int
    top_k: int
    inter: int
    shared_inter: int
    n_shared: int = 1

    def expert_bytes(self) -> int:
        """bf16 bytes of one routed expert (w13 + w2)."""
        return 2 * (self.hidden * 2 * self.inter + self.inter * self.hidden)

    def shared_bytes(self) -> int:
        return self.n_shared * 2 * (self.hidden * 2 * self.shared_inter + self.shared_inter * self.hidden)

    def router_bytes(self) -> int:
        return 2 * self.hidden * self.n_experts


TINY = BlockShape(hidden=256, n_experts=16, top_k=2, inter=128, shared_inter=128)
FULL = BlockShape(hidden=7168, n_experts=384, top_k=8, inter=2048, shared_inter=2048)
# Same per-expert shapes as FULL with only 16 experts (1.4 GB of weights):
# the small case used for detailed profiler captures.
PROF = BlockShape(hidden=7168, n_experts=16, top_k=8, inter=2048, shared_inter=2048)
# The full-size router (hidden 7168, 384 experts top-8) with narrow experts
# (inter 64, ~1 GB of weights): the small case for profiling the router.
RPROF = BlockShape(hidden=7168, n_experts=384, top_k=8, inter=64, shared_inter=64)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    shape: BlockShape
    batch: int
    routing: str  # "uniform" (router weights only) or "zipf" (log-prior bias added)
    description: str


WORKLOADS: Dict[str, Workload] = {
    "tiny_b1": Workload("tiny_b1", TINY, 1, "uniform",
                        "tiny block: hidden 256, 16 experts top-2, inter 128, 1 shared (inter 128), batch 1"),
    "full_b1": Workload("full_b1", FULL, 1, "uniform",
                        "full-size block: hidden 7168, 384 experts top-8, inter 2048, 1 shared (inter 2048), batch 1"),
    "full_b8": Workload("full_b8", FULL, 8, "uniform", "full-size block, batch 8, uniform-ish routing"),
    "full_b64": Workload("full_b64", FULL, 64, "uniform", "full-size block, batch 64, uniform-ish routing"),
    "zipf_b32": Workload("zipf_b32", FULL, 32, "zipf",
                         "full-size block, batch 32, Zipf(1.2) per-expert log-prior added to router logits"),
    **{f"zipf_b{b}": Workload(f"zipf_b{b}", FULL, b, "zipf",
                              f"full-size block, batch {b}, Zipf(1.2) log-prior (batch sweep)")
       for b in (1, 2, 4, 8, 16, 64)},
    "prof_b1": Workload("prof_b1", PROF, 1, "uniform",
                        "profiling case: full-size experts, 16 of them (1.4 GB), batch 1"),
    "prof_b8": Workload("prof_b8", PROF, 8, "uniform",
                        "profiling case: full-size experts, 16 of them (1.4 GB), batch 8"),
    "prof_b64": Workload("prof_b64", PROF, 64, "uniform",
                         "profiling case: full-size experts, 16 of them (1.4 GB), batch 64 (~32 tokens per expert)"),
    **{f"rprof_b{b}": Workload(f"rprof_b{b}", RPROF, b, "uniform",
                               f"router profiling case: hidden 7168, 384 experts top-8, inter 64 (~1 GB), batch {b}")
       for b in (1, 64)},
}


def seed_for(seed: int, name: str, index: int = 0) -> int:
    """Deterministic 63-bit sub-seed for (seed, tensor name, index)."""
    h = hashlib.blake2b(f"{seed}/{name}/{index}".encode(), digest_size=8).digest()
    return int.from_bytes(h, "little") & ((1 << 63) - 1)


def _normal_bf16(shape: Sequence[int], std: float, seed: int, device) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def make_x(batch: int, hidden: int, seed: int = 0, device="cpu",
           attempts: Optional[Sequence[int]] = None) -> torch.Tensor:
    """Activations x [batch, hidden] bf16 ~ N(0,1).  Row b is drawn from
    sub-seed (seed, "x", b, attempts[b]); a caller that rejects a row redraws it
    by raising its attempt counter."""
    rows = []
    for b in range(batch):
        a = 0 if attempts is None else int(attempts[b])
        rows.append(_normal_bf16((hidden,), 1.0, seed_for(seed, f"x/{a}", b), device))
    if not rows:
        return torch.zeros(0, hidden, dtype=torch.bfloat16, device=device)
    return torch.stack(rows)


@dataclasses.dataclass
class BlockWeights:
    router_w: torch.Tensor          # [H, E]
    w13: torch.Tensor               # [E, H, 2I] (expert e at w13[e])
    w2: torch.Tensor                # [E, I, H]
    shared_w13: Optional[torch.Tensor]  # [H, 2Is]
    shared_w2: Optional[torch.Tensor]   # [Is, H]
    router_bias: Optional[torch.Tensor]  # [E] float32 or None


def make_weights(shape: BlockShape, seed: int = 0, device="cpu", routing: str = "uniform",
                 router_device=None) -> BlockWeights:
    """All weights of one block, bf16 ~ N(0, 0.02), each expert from its own
    sub-seed.  ``routing == "zipf"`` adds the Zipf log-prior bias.
    ``router_device``: where the router weights are drawn (default: ``device``);
    the CPU and CUDA generators give different streams, so drawing them on
    the CPU makes them reproducible without a GPU (the benchmark does, so
    its inputs' top-k margins can be checked ahead of time)."""
    H, E, I, Is = shape.hidden, shape.n_experts, shape.inter, shape.shared_inter
    rdev = device if router_device is None else router_device
    router_w = _normal_bf16((H, E), WEIGHT_STD, seed_for(seed, "router_w"), rdev).to(device)
    w13 = torch.empty(E, H, 2 * I, dtype=torch.bfloat16, device=device)
    w2 = torch.empty(E, I, H, dtype=torch.bfloat16, device=device)
    for e in range(E):
        w13[e] = _normal_bf16((H, 2 * I), WEIGHT_STD, seed_for(seed, "w13", e), device)
        w2[e] = _normal_bf16((I, H), WEIGHT_STD, seed_for(seed, "w2", e), device)
    sw13 = sw2 = None
    if shape.n_shared:
        sw13 = _normal_bf16((H, 2 * Is), WEIGHT_STD, seed_for(seed, "shared_w13"), device)
        sw2 = _normal_bf16((Is, H), WEIGHT_STD, seed_for(seed, "shared_w2"), device)
    bias = zipf_log_prior(E, seed, device) if routing == "zipf" else None
    return BlockWeights(router_w, w13, w2, sw13, sw2, bias)


def zipf_log_prior(n_experts: int, seed: int = 0, device="cpu", s: float = ZIPF_S) -> torch.Tensor:
    """Per-expert bias log(q_rank(e)), q_r = r^-s / sum_r' r'^-s, with the ranks
    assigned to experts by a seeded random permutation (so the heavy experts
    are not simply the lowest ids).  float32 [E]."""
    z = sum(r ** -s for r in range(1, n_experts + 1))
    logq = [math.log((r ** -s) / z) for r in range(1, n_experts + 1)]
    g = torch.Generator(device="cpu")
    g.manual_seed(seed_for(seed, "zipf_perm"))
    perm = torch.randperm(n_experts, generator=g)  # expert e gets rank perm[e] + 1
    bias = torch.tensor([logq[int(perm[e])] for e in range(n_experts)], dtype=torch.float32)
    return bias.to(device)


def bf16_bits(t: torch.Tensor):
    """numpy uint16 view of a bf16 tensor's bit patterns (copied to host)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")


def make_router(shape: BlockShape, seed: int = 0, routing: str = "uniform"):
    """The router weights and bias of ``make_weights(..., router_device="cpu")``
    alone, on the CPU: (router_w [H, E] bf16, bias [E] float32 or None)."""
    router_w = _normal_bf16((shape.hidden, shape.n_experts), WEIGHT_STD, seed_for(seed, "router_w"), "cpu")
    bias = zipf_log_prior(shape.n_experts, seed, "cpu") if routing == "zipf" else None
    return router_w, bias


@dataclasses.dataclass
class Fp8BlockWeights:
    """Expert weights as e4m3 codes with fp32 block scales (the layout the
    library's fp8 entry point takes): q13 [E, 2I, H] and q2 [E, H, I] uint8
    ([out, in]); s13 [E, ceil(H/128), P13] and s2 [E, ceil(I/128), P2]
    float32, scale[i/128, o/128] of output o and input i, rows padded to a
    multiple of 4 floats; the shared expert's likewise without the E axis."""
    router_w: torch.Tensor
    q13: torch.Tensor
    s13: torch.Tensor
    q2: torch.Tensor
    s2: torch.Tensor
    shared_q13: Optional[torch.Tensor]
    shared_s13: Optional[torch.Tensor]
    shared_q2: Optional[torch.Tensor]
    shared_s2: Optional[torch.Tensor]
    router_bias: Optional[torch.Tensor]


def scale_pitch(outs: int) -> int:
    """Floats per row of an e4m3 matrix's block scales (padded to 16 bytes)."""
    return -(-(-(-outs // 128)) // 4) * 4


def _fp8_matrix(outs: int, ins: int, std: float, seed: int, device):
    """One [outs, ins] matrix ~ N(0, std) drawn in fp32 and stored as e4m3
    codes with one fp32 scale per 128 x 128 block (scale = block absmax / 448,
    so the block's largest magnitude maps to e4m3's largest finite value)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    w = torch.randn(outs, ins, generator=g, device=device, dtype=torch.float32).mul_(std)
    ob, ib = -(-outs // 128), -(-ins // 128)
    wp = torch.zeros(ob * 128, ib * 128, device=device, dtype=torch.float32)
    wp[:outs, :ins] = w
    blocks = wp.view(ob, 128, ib, 128)
    amax = blocks.abs().amax(dim=(1, 3))                       # [ob, ib]
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    q = (blocks / scale[:, None, :, None]).to(torch.float8_e4m3fn).view(torch.uint8)
    q = q.reshape(ob * 128, ib * 128)[:outs, :ins].contiguous()
    s = torch.zeros(ib, scale_pitch(outs), device=device, dtype=torch.float32)
    s[:, :ob] = scale.t()
    return q, s


def make_fp8_weights(shape: BlockShape, seed: int = 0, device="cpu", routing: str = "uniform",
                     router_device=None) -> Fp8BlockWeights:
    """A block with e4m3 expert weights (routed and shared) and bf16 router
    weights, each matrix from its own sub-seed (different from make_weights')."""
    H, E, I, Is = shape.hidden, shape.n_experts, shape.inter, shape.shared_inter
    rdev = device if router_device is None else router_device
    router_w = _normal_bf16((H, E), WEIGHT_STD, seed_for(seed, "router_w"), rdev).to(device)
    q13 = torch.empty(E, 2 * I, H, dtype=torch.uint8, device=device)
    s13 = torch.empty(E, -(-H // 128), scale_pitch(2 * I), dtype=torch.float32, device=device)
    q2 = torch.empty(E, H, I, dtype=torch.uint8, device=device)
    s2 = torch.empty(E, -(-I // 128), scale_pitch(H), dtype=torch.float32, device=device)
    for e in range(E):
        q13[e], s13[e] = _fp8_matrix(2 * I, H, WEIGHT_STD, seed_for(seed, "fp8_w13", e), device)
        q2[e], s2[e] = _fp8_matrix(H, I, WEIGHT_STD, seed_for(seed, "fp8_w2", e), device)
    sq13 = ss13 = sq2 = ss2 = None
    if shape.n_shared:
        sq13, ss13 = _fp8_matrix(2 * Is, H, WEIGHT_STD, seed_for(seed, "fp8_shared_w13"), device)
        sq2, ss2 = _fp8_matrix(H, Is, WEIGHT_STD, seed_for(seed, "fp8_shared_w2"), device)
    bias = zipf_log_prior(E, seed, device) if routing == "zipf" else None
    return Fp8BlockWeights(router_w, q13, s13, q2, s2, sq13, ss13, sq2, ss2, bias)
