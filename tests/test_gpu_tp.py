"""The tensor-parallel split of the block on one B200: the ranks' partial-sum
forwards (MOE_FLAG_PARTIAL_SUM, each on its slice of every expert's
intermediate dimension) run one after another on the same GPU, and
moe_decode_reduce_residual adds their fp32 sums to the residual -- the step
that, across GPUs, reads the other ranks' buffers over NVLink.  The result
must match the fp64 oracle of the whole block on every element (the same bar
as the single-GPU parity tests)."""
import pytest
import torch

from moe_decode_block_b200 import MOE_OK, MoEDecode, reduce_residual, synth
from moe_decode_block_b200.tp import TPBlock, shard_intermediate
from gpu_helpers import margin_x, oracle_check

pytestmark = pytest.mark.gpu


def test_reduce_residual_adds_the_parts_in_rank_order_bitwise():
    g = torch.Generator(device="cuda").manual_seed(3)
    B, H = 5, 7168
    x = torch.randn(B, H, device="cuda", generator=g).to(torch.bfloat16)
    parts = [torch.randn(B, H, device="cuda", generator=g) * s for s in (1.0, 0.5, 1e-3)]
    out = torch.empty_like(x)
    reduce_residual(parts, x, out)
    ref = (x.float() + ((parts[0] + parts[1]) + parts[2])).to(torch.bfloat16)  # fp32, rank order, one rounding
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    # in place: out is x
    y = x.clone()
    reduce_residual(parts[:1], y, y)
    torch.cuda.synchronize()
    assert torch.equal(y, (x.float() + parts[0]).to(torch.bfloat16))


def _rank_forwards(shape, wts, x, tp, max_batch):
    """Every rank's partial sum (and routing), ranks run one after another."""
    B = x.shape[0]
    parts, routes = [], []
    for r in range(tp):
        w13, w2 = shard_intermediate(wts.w13, wts.w2, r, tp)
        sw13, sw2 = shard_intermediate(wts.shared_w13, wts.shared_w2, r, tp)
        blk = MoEDecode(shape.hidden, shape.n_experts, shape.top_k, shape.inter // tp, shape.shared_inter // tp,
                        max_batch=max_batch, router_bias=wts.router_bias, partial=True)
        try:
            p = torch.full((B, shape.hidden), float("nan"), dtype=torch.float32, device="cuda")
            ids = torch.full((B, shape.top_k), -1, dtype=torch.int32, device="cuda")
            w = torch.empty(B, shape.top_k, dtype=torch.float32, device="cuda")
            blk.forward(x, wts.router_w, w13, w2, sw13, sw2, p, ids, w)
            torch.cuda.synchronize()
            assert blk.status() == MOE_OK
            parts.append(p)
            routes.append((ids, w))
        finally:
            blk.close()
        del w13, w2
    for ids, w in routes[1:]:  # the same routing on every rank (the weights up to reduction order)
        assert torch.equal(ids, routes[0][0])
        assert float((w - routes[0][1]).abs().max()) <= 1e-6
    return parts, routes[0]


@pytest.mark.parametrize("tp", [2, 4])
def test_tiny_tp_ranks_match_the_block(tp):
    s = synth.TINY
    wts = synth.make_weights(s, seed=31, device="cuda")
    for B in (1, 5, 13, 40):
        x = margin_x(B, s.hidden, wts, s.top_k, seed=300 + B)
        parts, (ids, w) = _rank_forwards(s, wts, x, tp, max_batch=64)
        out = torch.full_like(x, float("nan"))
        reduce_residual(parts, x, out)
        torch.cuda.synchronize()
        oracle_check(wts, s.top_k, x, out, ids, w)


def test_tp_block_of_one_rank_is_the_block():
    s = synth.TINY
    wts = synth.make_weights(s, seed=32, device="cuda")
    tpb = TPBlock(s.hidden, s.n_experts, s.top_k, s.inter, s.shared_inter, tp=1, rank=0, max_batch=8)
    try:
        x = margin_x(6, s.hidden, wts, s.top_k, seed=320)
        out = torch.full_like(x, float("nan"))
        ids = torch.empty(6, s.top_k, dtype=torch.int32, device="cuda")
        w = torch.empty(6, s.top_k, dtype=torch.float32, device="cuda")
        tpb.forward(x, wts.router_w, wts.w13, wts.w2, wts.shared_w13, wts.shared_w2, out, ids, w)
        torch.cuda.synchronize()
        oracle_check(wts, s.top_k, x, out, ids, w)
    finally:
        tpb.close()


def test_full_size_tp2_ranks_match_the_block():
    s = synth.FULL
    wts = synth.make_weights(s, seed=0, device="cuda")
    try:
        B = 8
        x = margin_x(B, s.hidden, wts, s.top_k, seed=330)
        parts, (ids, w) = _rank_forwards(s, wts, x, 2, max_batch=8)
        out = torch.full_like(x, float("nan"))
        reduce_residual(parts, x, out)
        torch.cuda.synchronize()
        oracle_check(wts, s.top_k, x, out, ids, w)
    finally:
        del wts
        torch.cuda.empty_cache()
