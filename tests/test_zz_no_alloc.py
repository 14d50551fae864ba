"""The allocation-free router entry point (moe_router_topk_noalloc).

Some callers cannot call cudaMalloc: code running while a CUDA graph is being
captured, or a host framework that owns all device memory through its own
pool and does not let plug-ins allocate.  They cannot create a handle with
moe_decode_init, so the library also offers the router step (scores, softmax,
top-k, renormalised weights) with its scratch in a fixed static device array.
This test calls it through the C ABI twice in a row (different batches, so the
second call must clear what the first left in the shared scratch) and checks
each result against the handle-based moe_decode_forward: ids exact, weights
within 1e-5, and the entry point's device status (read back with
moe_router_topk_noalloc_status) OK.  The sizes reach the limits the fixed
scratch is sized for (batch 64, 1,024 experts, top-32), and one case captures
the call in a CUDA graph after a warm call and replays it on new inputs.  It
lives in its own file, collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import moe_decode_block_b200 as mdb
from moe_decode_block_b200 import synth
from moe_decode_block_b200.build import build_library
from gpu_helpers import margin_x

pytestmark = pytest.mark.gpu

W_ATOL = 1e-5


def _reference_routing(blk, wts, x):
    """ids and weights from the existing entry point (a full forward)."""
    B = x.shape[0]
    k = blk.shapes.top_k
    out = torch.empty_like(x)
    ids = torch.empty(B, k, dtype=torch.int32, device=x.device)
    w = torch.empty(B, k, dtype=torch.float32, device=x.device)
    blk.forward(x, wts.router_w, wts.w13, wts.w2, wts.shared_w13, wts.shared_w2, out, ids, w)
    torch.cuda.synchronize()
    return ids, w


def _noalloc(lib, wts, x, k):
    """One call of the C entry point on the current stream."""
    B, H = x.shape
    E = wts.router_w.shape[1]
    ids = torch.full((B, k), -1, dtype=torch.int32, device=x.device)
    w = torch.full((B, k), float("nan"), dtype=torch.float32, device=x.device)
    bias = None if wts.router_bias is None else wts.router_bias.data_ptr()
    rc = lib.moe_router_topk_noalloc(x.data_ptr(), wts.router_w.data_ptr(), bias, ids.data_ptr(), w.data_ptr(),
                                     B, H, E, k, torch.cuda.current_stream().cuda_stream)
    assert rc == mdb.MOE_OK, lib.moe_decode_error_string(rc)
    return ids, w


def _status(lib):
    return lib.moe_router_topk_noalloc_status(torch.cuda.current_stream().cuda_stream)


# 1,024 experts (the scratch's limit) at batch 64; hidden 2048 spreads the
# logits (std ~0.9) enough that rows with every top-33 gap >= 1e-3 are common
WIDE_8 = synth.BlockShape(hidden=256, n_experts=1024, top_k=8, inter=64, shared_inter=64)
WIDE_32 = synth.BlockShape(hidden=2048, n_experts=1024, top_k=32, inter=64, shared_inter=64)


@pytest.mark.parametrize("shape,routing,batches", [
    (synth.TINY, "uniform", (5, 2)),
    (synth.FULL, "zipf", (8, 3)),
    (WIDE_8, "uniform", (64, 1)),
    (WIDE_32, "uniform", (64, 7)),
])
def test_noalloc_router_matches_forward_twice_in_a_row(shape, routing, batches):
    build_library()
    lib = mdb.load_library()
    wts = synth.make_weights(shape, seed=7, device="cuda", routing=routing)
    blk = mdb.MoEDecode(shape.hidden, shape.n_experts, shape.top_k, shape.inter, shape.shared_inter,
                        max_batch=max(batches), router_bias=wts.router_bias)
    try:
        for call, B in enumerate(batches):
            x = margin_x(B, shape.hidden, wts, shape.top_k, seed=100 + call)
            ref_ids, ref_w = _reference_routing(blk, wts, x)
            ids, w = _noalloc(lib, wts, x, shape.top_k)
            assert _status(lib) == mdb.MOE_OK, f"call {call}"
            assert torch.equal(ids, ref_ids), f"call {call}"
            assert float(torch.max(torch.abs(w - ref_w))) <= W_ATOL, f"call {call}"
    finally:
        blk.close()
        del wts
        torch.cuda.empty_cache()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    build_library()
    lib = mdb.load_library()
    p = ctypes.c_void_p(16)  # never dereferenced: the size checks come first
    too_big = [(mdb_b, 256, 16, 2) for mdb_b in (65, 1000)] + [(4, 256, 2048, 2), (4, 256, 16, 33)]
    for B, H, E, k in too_big:
        rc = lib.moe_router_topk_noalloc(p, p, None, p, p, B, H, E, k, None)
        assert rc == mdb.MOE_ERR_UNSUPPORTED_SHAPE, (B, H, E, k)


def test_noalloc_router_in_a_cuda_graph():
    # the first call on the device (set-up included) is made outside capture;
    # the captured call allocates nothing, so capture succeeds, and each
    # replay recomputes the routing of whatever x holds
    build_library()
    lib = mdb.load_library()
    shape = synth.TINY
    wts = synth.make_weights(shape, seed=8, device="cuda")
    blk = mdb.MoEDecode(shape.hidden, shape.n_experts, shape.top_k, shape.inter, shape.shared_inter, max_batch=6)
    try:
        B, k = 6, shape.top_k
        xbuf = synth.make_x(B, shape.hidden, seed=200).cuda()
        ids = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
        w = torch.full((B, k), float("nan"), dtype=torch.float32, device="cuda")
        stream = torch.cuda.Stream()

        def call():
            rc = lib.moe_router_topk_noalloc(xbuf.data_ptr(), wts.router_w.data_ptr(), None, ids.data_ptr(),
                                             w.data_ptr(), B, shape.hidden, shape.n_experts, k,
                                             torch.cuda.current_stream().cuda_stream)
            assert rc == mdb.MOE_OK

        with torch.cuda.stream(stream):
            call()  # warm, outside capture
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            call()
        for seed in (201, 202):
            xbuf.copy_(margin_x(B, shape.hidden, wts, k, seed=seed))
            ids.fill_(-1)
            g.replay()
            torch.cuda.synchronize()
            ref_ids, ref_w = _reference_routing(blk, wts, xbuf.clone())
            assert torch.equal(ids, ref_ids), seed
            assert float(torch.max(torch.abs(w - ref_w))) <= W_ATOL, seed
            assert _status(lib) == mdb.MOE_OK
        del g
    finally:
        blk.close()
