"""Shared helpers for the GPU parity tests: seeded inputs with a top-k logit
margin (checked with the oracle's router on the host) and comparison of the
CUDA path against the fp64 oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from moe_decode_block_b200 import MoEDecode, synth

OUT_RTOL = 2e-2      # max|out - oracle| <= 2e-2 * rms(oracle out)
W_ATOL = 1e-5        # |topk_w - oracle| (fp32 softmax vs fp64)
MIN_MARGIN = 1e-3    # top-(k+1) logit gaps of every generated row


def bias_np(wts):
    return None if wts.router_bias is None else wts.router_bias.detach().float().cpu().numpy()


def margin_x(batch, hidden, wts, k, seed=0, device="cuda", min_gap=MIN_MARGIN):
    """x [batch, hidden] whose rows all have top-(k+1) logit gaps >= min_gap
    (fp64 logits of the bf16 values); failing rows are redrawn."""
    attempts = np.zeros(batch, dtype=np.int64)
    rb = synth.bf16_bits(wts.router_w)
    bias = bias_np(wts)
    for _ in range(256):
        x = synth.make_x(batch, hidden, seed=seed, attempts=attempts)
        if batch == 0:
            return x.to(device)
        logits, _, _ = oracle.router(synth.bf16_bits(x), rb, k, bias)
        bad = oracle.topk_margin(logits, k) < min_gap
        if not bad.any():
            return x.to(device)
        attempts[bad] += 1
    raise RuntimeError("could not draw inputs with the required top-k margin")


class Run:
    """Device buffers and one handle for a block shape."""

    def __init__(self, shape: synth.BlockShape, wts, max_batch=64, two_stream=False, tcgen05=False, extra_flags=0):
        self.s = shape
        self.wts = wts
        self.blk = MoEDecode(shape.hidden, shape.n_experts, shape.top_k, shape.inter, shape.shared_inter,
                             n_shared=shape.n_shared, max_batch=max_batch, router_bias=wts.router_bias,
                             two_stream=two_stream, tcgen05=tcgen05, extra_flags=extra_flags)

    def kernels_per_forward(self):
        """Kernels one forward enqueues: router, expert kernel, combine by default;
        router, routed experts, [shared expert], combine with two streams."""
        if self.blk.two_stream:
            return 4 if self.s.n_shared else 3
        return 3

    def forward(self, x, stream_aux=None, w13=None, w2=None):
        B = x.shape[0]
        k = self.s.top_k
        out = torch.full_like(x, float("nan"))
        ids = torch.full((B, k), -1, dtype=torch.int32, device=x.device)
        w = torch.full((B, k), float("nan"), dtype=torch.float32, device=x.device)
        self.blk.forward(x, self.wts.router_w, self.wts.w13 if w13 is None else w13,
                         self.wts.w2 if w2 is None else w2, self.wts.shared_w13, self.wts.shared_w2,
                         out, ids, w, stream_aux=stream_aux)
        torch.cuda.synchronize()
        return out, ids, w


# Panel geometry of the expert kernels' token classes (columns x rows of a
# 64 KB weight stage), restated to predict the device-side stage counters.
CLASS_LW = (1024, 1024, 512)
CLASS_ROWS = (32, 32, 64)
# e4m3 weights: 128 input rows (one 128-byte line per weight row) by 512,
# 512 and 256 columns
CLASS_LW_FP8 = (512, 512, 256)
ROWS_FP8 = 128
UNIT_TOKENS = 32


def token_class(n):
    return 0 if n <= 8 else (1 if n <= 16 else 2)


def unit_stages(c, up, H, I, fp8=False):
    """Stages of a unit's UP list (panels of lw/2 gate + up columns, r-row
    stages) or DOWN list (panels of lw columns, r-row stages)."""
    lw, r = (CLASS_LW_FP8[c], ROWS_FP8) if fp8 else (CLASS_LW[c], CLASS_ROWS[c])
    cdiv = lambda a, b: -(-a // b)
    if up:
        return cdiv(I, lw // 2) * cdiv(H, r)
    return cdiv(H, lw) * cdiv(I, r)


def expected_stages(shape, ids, batch, fp8=False):
    """(up[3], down[3]) stages one forward streams per token class: the shared
    expert in units of up to 32 tokens, each selected expert in units of up to
    32 of the tokens that chose it."""
    up, down = [0, 0, 0], [0, 0, 0]
    units = []  # (tokens, intermediate size)
    if shape.n_shared:
        units += [(min(UNIT_TOKENS, batch - u), shape.shared_inter) for u in range(0, batch, UNIT_TOKENS)]
    counts = np.bincount(np.asarray(ids).ravel(), minlength=shape.n_experts)
    for n in counts[counts > 0]:
        units += [(min(UNIT_TOKENS, int(n) - u), shape.inter) for u in range(0, int(n), UNIT_TOKENS)]
    for n, I in units:
        c = token_class(n)
        up[c] += unit_stages(c, True, shape.hidden, I, fp8)
        down[c] += unit_stages(c, False, shape.hidden, I, fp8)
    return up, down


def oracle_check(wts, k, x, out, ids, w, w13=None, w2=None):
    """ids exact and weights within W_ATOL, and the outputs of every row within
    OUT_RTOL * rms, against the fp64 oracle.  The oracle holds one selected
    expert's weights at a time (copied from the device as it needs them), so
    full-size batches are compared element by element without holding every
    touched expert in host memory."""
    xb = synth.bf16_bits(x)
    o_logits, o_ids, o_w = oracle.router(xb, synth.bf16_bits(wts.router_w), k, bias_np(wts))
    g_ids = ids.cpu().numpy()
    np.testing.assert_array_equal(g_ids, o_ids)
    g_w = w.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(g_w - o_w), initial=0.0) <= W_ATOL
    assert np.max(np.abs(g_w.sum(axis=1) - 1.0), initial=0.0) <= 1e-6
    W13 = wts.w13 if w13 is None else w13
    W2 = wts.w2 if w2 is None else w2

    def fetch(e):
        return synth.bf16_bits(W13[e]), synth.bf16_bits(W2[e])

    sw13 = None if wts.shared_w13 is None else synth.bf16_bits(wts.shared_w13)
    sw2 = None if wts.shared_w2 is None else synth.bf16_bits(wts.shared_w2)
    o_out = oracle.block_streamed(xb, o_ids, o_w, fetch, sw13, sw2)
    g_out = out.float().cpu().numpy()
    assert g_out.shape == o_out.shape
    err = np.abs(g_out - o_out)
    rms = float(np.sqrt(np.mean(o_out ** 2)))
    assert np.all(np.isfinite(g_out))
    assert err.max(initial=0.0) <= OUT_RTOL * rms, f"max|err| {err.max():.4g} > {OUT_RTOL} * rms {rms:.4g}"
    return float(err.max(initial=0.0)), rms
