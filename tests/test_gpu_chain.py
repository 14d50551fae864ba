"""A chain of blocks (moe_decode_block_b200.chain): one handle per block, the
blocks back to back on one stream with block l's output as block l + 1's
input.  Every block is compared with the fp64 oracle applied to the input that
block actually read (the previous block's bf16 output)."""
import numpy as np
import pytest
import torch

import oracle
from moe_decode_block_b200 import synth
from moe_decode_block_b200.chain import BlockChain
from gpu_helpers import OUT_RTOL, W_ATOL, bias_np, margin_x

pytestmark = pytest.mark.gpu

TIE = 1e-4  # a row whose top-(k+1) logits are closer than this may pick either side


def chain_block_check(wts, k, x, out, ids, w):
    """ids exact, weights within W_ATOL and outputs within OUT_RTOL * rms for
    every row whose top-k is separated by at least TIE; a row closer than that
    (possible only after the first block, whose input is not drawn with a
    margin) must select a valid top-k and is not compared further.  Returns
    the number of rows compared."""
    xb = synth.bf16_bits(x)
    logits, o_ids, o_w = oracle.router(xb, synth.bf16_bits(wts.router_w), k, bias_np(wts))
    sure = oracle.topk_margin(logits, k) >= TIE
    g_ids = ids.cpu().numpy()
    g_w = w.cpu().numpy().astype(np.float64)
    np.testing.assert_array_equal(g_ids[sure], o_ids[sure])
    assert np.max(np.abs(g_w[sure] - o_w[sure]), initial=0.0) <= W_ATOL
    for b in np.flatnonzero(~sure):
        kth = np.sort(logits[b])[::-1][k - 1]
        assert len(set(g_ids[b].tolist())) == k and np.all(logits[b][g_ids[b]] >= kth - TIE)

    def fetch(e):
        return synth.bf16_bits(wts.w13[e]), synth.bf16_bits(wts.w2[e])

    o_out = oracle.block_streamed(xb, o_ids, o_w, fetch, synth.bf16_bits(wts.shared_w13),
                                  synth.bf16_bits(wts.shared_w2))
    g_out = out.float().cpu().numpy()
    assert np.all(np.isfinite(g_out))
    rms = float(np.sqrt(np.mean(o_out[sure] ** 2))) if sure.any() else 0.0
    err = np.abs(g_out[sure] - o_out[sure])
    assert err.max(initial=0.0) <= OUT_RTOL * rms, f"max|err| {err.max():.4g} > {OUT_RTOL} * rms {rms:.4g}"
    return int(sure.sum())


def _run_chain(shape, n_blocks, B, seed0, max_batch=64):
    weights = [synth.make_weights(shape, seed=seed0 + l, device="cuda") for l in range(n_blocks)]
    x = margin_x(B, shape.hidden, weights[0], shape.top_k, seed=seed0 + 100)
    chain = BlockChain(n_blocks, shape.hidden, shape.n_experts, shape.top_k, shape.inter, shape.shared_inter,
                       max_batch=max_batch, router_biases=[w.router_bias for w in weights])
    try:
        outs = [torch.full_like(x, float("nan")) for _ in range(n_blocks)]
        ids = [torch.full((B, shape.top_k), -1, dtype=torch.int32, device="cuda") for _ in range(n_blocks)]
        ws = [torch.empty(B, shape.top_k, dtype=torch.float32, device="cuda") for _ in range(n_blocks)]
        wl = [(w.router_w, w.w13, w.w2, w.shared_w13, w.shared_w2) for w in weights]
        chain.forward(x, wl, outs, ids, ws)
        torch.cuda.synchronize()
        assert chain.status() == 0
        compared = 0
        for l in range(n_blocks):
            xin = x if l == 0 else outs[l - 1]
            compared += chain_block_check(weights[l], shape.top_k, xin, outs[l], ids[l], ws[l])
        assert compared >= n_blocks * B - max(1, n_blocks * B // 20)  # near-ties are rare
    finally:
        chain.close()


@pytest.mark.parametrize("B", [1, 5, 13])
def test_tiny_chain_of_three_blocks(B):
    _run_chain(synth.TINY, 3, B, seed0=40 + B)


def test_full_size_experts_chain_of_two_blocks():
    _run_chain(synth.PROF, 2, 8, seed0=60, max_batch=8)
    torch.cuda.empty_cache()


def test_chain_in_a_cuda_graph():
    s = synth.TINY
    weights = [synth.make_weights(s, seed=70 + l, device="cuda") for l in range(2)]
    xa = margin_x(6, s.hidden, weights[0], s.top_k, seed=71)
    xb = margin_x(6, s.hidden, weights[0], s.top_k, seed=72)
    chain = BlockChain(2, s.hidden, s.n_experts, s.top_k, s.inter, s.shared_inter, max_batch=8,
                       router_biases=[w.router_bias for w in weights])
    try:
        xbuf = xa.clone()
        outs = [torch.empty_like(xa) for _ in range(2)]
        ids = [torch.empty(6, s.top_k, dtype=torch.int32, device="cuda") for _ in range(2)]
        ws = [torch.empty(6, s.top_k, dtype=torch.float32, device="cuda") for _ in range(2)]
        wl = [(w.router_w, w.w13, w.w2, w.shared_w13, w.shared_w2) for w in weights]
        stream = torch.cuda.Stream()
        with torch.cuda.stream(stream):
            chain.forward(xbuf, wl, outs, ids, ws, stream=stream)  # warm-up outside capture
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            chain.forward(xbuf, wl, outs, ids, ws, stream=torch.cuda.current_stream())
        for xin in (xa, xb, xa):
            xbuf.copy_(xin)
            for o in outs:
                o.fill_(float("nan"))
            g.replay()
            torch.cuda.synchronize()
            assert chain.status() == 0
            chain_block_check(weights[0], s.top_k, xbuf, outs[0], ids[0], ws[0])
            chain_block_check(weights[1], s.top_k, outs[0], outs[1], ids[1], ws[1])
        del g
    finally:
        chain.close()
