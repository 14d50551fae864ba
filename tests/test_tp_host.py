"""The tensor-parallel split of the block (moe_decode_block_b200.tp) on CPU,
checked against the fp64 oracle: rank r of tp takes the slice [r I/tp,
(r+1) I/tp) of every expert's intermediate dimension, and the ranks' expert
sums add up to the whole block's.  Two gloo ranks run the exchange (an
all-reduce of the partial sums) the way TPBlock does on GPUs."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from moe_decode_block_b200 import synth
from moe_decode_block_b200.tp import shard_intermediate

S = synth.TINY


def _bits(t):
    return synth.bf16_bits(t)


def _shard_partial(wts, x, ids, w, rank, tp):
    """Oracle expert sum (no residual) of rank `rank`'s slice."""
    w13, w2 = shard_intermediate(wts.w13, wts.w2, rank, tp)
    sw13, sw2 = shard_intermediate(wts.shared_w13, wts.shared_w2, rank, tp)
    xb = _bits(x)
    out = oracle.block(xb, ids, w, [_bits(t) for t in w13], [_bits(t) for t in w2], _bits(sw13), _bits(sw2))
    return out - x.double().numpy()  # x (bf16) is exact in fp64


def test_shard_slices_gate_and_up_columns_and_down_rows():
    w13 = torch.arange(2 * 3 * 8, dtype=torch.float32).reshape(2, 3, 8)  # E 2, H 3, I 4
    w2 = torch.arange(2 * 4 * 3, dtype=torch.float32).reshape(2, 4, 3)
    a13, a2 = shard_intermediate(w13, w2, 1, 2)
    assert a13.shape == (2, 3, 4) and a2.shape == (2, 2, 3)
    assert torch.equal(a13[..., :2], w13[..., 2:4])      # gate columns 2, 3
    assert torch.equal(a13[..., 2:], w13[..., 6:8])      # up columns I + 2, I + 3
    assert torch.equal(a2, w2[:, 2:4, :])
    # the slices of all ranks put back together are the expert again
    parts = [shard_intermediate(w13, w2, r, 4) for r in range(4)]
    assert torch.equal(torch.cat([p[0][..., :1] for p in parts], -1), w13[..., :4])
    assert torch.equal(torch.cat([p[0][..., 1:] for p in parts], -1), w13[..., 4:])
    assert torch.equal(torch.cat([p[1] for p in parts], -2), w2)
    with pytest.raises(ValueError):
        shard_intermediate(w13, w2, 0, 3)  # 4 rows do not split in 3
    with pytest.raises(ValueError):
        shard_intermediate(w13, w2, 2, 2)


@pytest.mark.parametrize("tp", [2, 4])
def test_rank_partial_sums_add_up_to_the_block(tp):
    wts = synth.make_weights(S, seed=5, device="cpu")
    x = synth.make_x(3, S.hidden, seed=6)
    xb = _bits(x)
    _, ids, w = oracle.router(xb, _bits(wts.router_w), S.top_k)
    full = oracle.block(xb, ids, w, [_bits(t) for t in wts.w13], [_bits(t) for t in wts.w2],
                        _bits(wts.shared_w13), _bits(wts.shared_w2))
    xf = x.double().numpy()
    total = sum(_shard_partial(wts, x, ids, w, r, tp) for r in range(tp))
    # the intermediate dimension splits exactly: only fp64 summation order differs
    np.testing.assert_allclose(xf + total, full, rtol=0, atol=1e-12 * max(1.0, float(np.abs(full).max())))
    # and no rank alone is the block (each slice carries a real share)
    assert np.abs(_shard_partial(wts, x, ids, w, 0, tp)).max() > 1e-6


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        wts = synth.make_weights(S, seed=7, device="cpu")
        x = synth.make_x(4, S.hidden, seed=8)
        _, ids, w = oracle.router(_bits(x), _bits(wts.router_w), S.top_k)
        part = torch.from_numpy(_shard_partial(wts, x, ids, w, rank, world))
        dist.all_reduce(part, op=dist.ReduceOp.SUM)  # the exchange TPBlock runs without peer buffers
        results[rank] = (x.double().numpy() + part.numpy()).tolist()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reproduce_the_block():
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    wts = synth.make_weights(S, seed=7, device="cpu")
    x = synth.make_x(4, S.hidden, seed=8)
    full, _, _, _ = oracle.moe_forward(_bits(x), _bits(wts.router_w), [_bits(t) for t in wts.w13],
                                       [_bits(t) for t in wts.w2], _bits(wts.shared_w13), _bits(wts.shared_w2),
                                       S.top_k)
    for r in range(world):
        got = np.array(results[r])
        np.testing.assert_allclose(got, full, rtol=0, atol=1e-12 * max(1.0, float(np.abs(full).max())))
    assert results[0] == results[1]  # every rank holds the same sum
