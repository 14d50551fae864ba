"""The block with e4m3 expert weights (moe_decode_forward_fp8) on a B200
against the fp64 oracle of block-scaled e4m3 weights.

Bar as for bf16 weights: ids exact (the router is unchanged: bf16 weights,
inputs with a top-k logit margin), weights within 1e-5, outputs within
2e-2 * rms of the oracle, which decodes every code exactly and applies the
block scales in fp64.  The tiny block is compared element by element at
batches that reach every token class; the full-size block on every row.
"""
import numpy as np
import pytest
import torch

import oracle
import moe_decode_block_b200 as mdb
from moe_decode_block_b200 import MOE_OK, MoEDecode, synth
from gpu_helpers import OUT_RTOL, W_ATOL, expected_stages, margin_x

pytestmark = pytest.mark.gpu


def _oracle_scales(s_api, outs):
    """API scale layout [ceil(in/128), padded] -> the oracle's [ceil(out/128), ceil(in/128)]."""
    ob = -(-outs // 128)
    return np.ascontiguousarray(s_api.detach().cpu().numpy()[:, :ob].T)


def fp8_check(shape, w8, x, out, ids, w):
    k = shape.top_k
    xb = synth.bf16_bits(x)
    bias = None if w8.router_bias is None else w8.router_bias.float().cpu().numpy()
    _, o_ids, o_w = oracle.router(xb, synth.bf16_bits(w8.router_w), k, bias)
    np.testing.assert_array_equal(ids.cpu().numpy(), o_ids)
    assert np.max(np.abs(w.cpu().numpy().astype(np.float64) - o_w)) <= W_ATOL
    H, I, Is = shape.hidden, shape.inter, shape.shared_inter

    def fetch(e):
        return (w8.q13[e].cpu().numpy(), _oracle_scales(w8.s13[e], 2 * I),
                w8.q2[e].cpu().numpy(), _oracle_scales(w8.s2[e], H))

    shared = None
    if w8.shared_q13 is not None:
        shared = (w8.shared_q13.cpu().numpy(), _oracle_scales(w8.shared_s13, 2 * Is),
                  w8.shared_q2.cpu().numpy(), _oracle_scales(w8.shared_s2, H))
    o_out = oracle.block_streamed_fp8(xb, o_ids, o_w, fetch, shared)
    g_out = out.float().cpu().numpy()
    assert np.all(np.isfinite(g_out))
    rms = float(np.sqrt(np.mean(o_out ** 2)))
    err = float(np.max(np.abs(g_out - o_out)))
    assert err <= OUT_RTOL * rms, (err, rms)
    return err, rms


def run_fp8(blk, w8, x):
    B, k = x.shape[0], w8.router_w.shape[1] and blk.shapes.top_k
    out = torch.full_like(x, float("nan"))
    ids = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
    w = torch.full((B, k), float("nan"), dtype=torch.float32, device="cuda")
    blk.forward_fp8(x, w8.router_w, w8.q13, w8.s13, w8.q2, w8.s2, w8.shared_q13, w8.shared_s13, w8.shared_q2,
                    w8.shared_s2, out, ids, w)
    torch.cuda.synchronize()
    return out, ids, w


@pytest.fixture(scope="module")
def tiny8():
    s = synth.TINY
    w8 = synth.make_fp8_weights(s, seed=0, device="cuda")
    return s, w8


@pytest.mark.parametrize("plan", ["default", "two_stream"])
@pytest.mark.parametrize("B", [1, 2, 5, 8, 13, 32, 64])
def test_tiny_fp8_every_element(tiny8, plan, B):
    s, w8 = tiny8
    blk = MoEDecode(s.hidden, s.n_experts, s.top_k, s.inter, s.shared_inter, max_batch=64, fp8=True,
                    two_stream=plan == "two_stream")
    try:
        x = margin_x(B, s.hidden, w8, s.top_k, seed=90 + B)
        before = blk.stats()
        out, ids, w = run_fp8(blk, w8, x)
        fp8_check(s, w8, x, out, ids, w)
        st = blk.stats()
        up, down = expected_stages(s, ids.cpu().numpy(), B, fp8=True)
        assert [a - b for a, b in zip(st["stages_up"], before["stages_up"])] == up
        assert [a - b for a, b in zip(st["stages_down"], before["stages_down"])] == down
        assert blk.status() == MOE_OK
    finally:
        blk.close()


def test_fp8_and_bf16_entry_points_reject_the_other_handle(tiny8):
    s, w8 = tiny8
    b8 = MoEDecode(s.hidden, s.n_experts, s.top_k, s.inter, s.shared_inter, max_batch=4, fp8=True)
    b16 = MoEDecode(s.hidden, s.n_experts, s.top_k, s.inter, s.shared_inter, max_batch=4)
    try:
        x = margin_x(2, s.hidden, w8, s.top_k, seed=99)
        out = torch.empty_like(x)
        ids = torch.empty(2, s.top_k, dtype=torch.int32, device="cuda")
        w = torch.empty(2, s.top_k, dtype=torch.float32, device="cuda")
        with pytest.raises(mdb.MoEDecodeError):
            b8.forward(x, w8.router_w, w8.q13, w8.q2, w8.shared_q13, w8.shared_q2, out, ids, w)
        with pytest.raises(mdb.MoEDecodeError):
            b16.forward_fp8(x, w8.router_w, w8.q13, w8.s13, w8.q2, w8.s2, w8.shared_q13, w8.shared_s13,
                            w8.shared_q2, w8.shared_s2, out, ids, w)
    finally:
        b8.close()
        b16.close()


@pytest.mark.parametrize("B", [1, 8])
def test_full_size_fp8_every_row(B):
    s = synth.FULL
    w8 = synth.make_fp8_weights(s, seed=0, device="cuda")
    blk = MoEDecode(s.hidden, s.n_experts, s.top_k, s.inter, s.shared_inter, max_batch=8, fp8=True)
    try:
        x = margin_x(B, s.hidden, w8, s.top_k, seed=100 + B)
        out, ids, w = run_fp8(blk, w8, x)
        fp8_check(s, w8, x, out, ids, w)
        assert blk.status() == MOE_OK
    finally:
        blk.close()
        del w8
        torch.cuda.empty_cache()
