"""Numpy fp64 restatement of the MoE decode-block oracle.

TEST INFRASTRUCTURE ONLY: a second, independently written oracle used to
cross-check the C oracle on small shapes.  Only tests, the smoke check and the
benchmark's CPU-baseline leg may import it.

It follows the same reading of the pages as ``moe_oracle.c`` ("Hyper
Optimizing Kimi K3 in vLLM: Moving Fast and Responsibly", commentary, section
"Recovering time between operators": router scores, selected experts, a shared
expert beside them; the formulas themselves are the plainest standard reading):

1. logits = x R (+ bias)
2. p = softmax(logits) over all experts
3. S = top-k logits, descending, equal logits to the smaller id
4. w = p[S] / sum p[S]
5. y_j = (silu(x W13[:, :I]) * (x W13[:, I:])) W2 for each selected expert
6. s = the same MLP with the shared weights
7. out = x + sum_j w_j y_j + s

Matrix products use ``numpy.matmul`` in float64 as a library primitive; the
bf16 inputs (uint16 bit patterns) are widened exactly.
"""
from __future__ import annotations

import numpy as np


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def router(x, router_w, k, bias=None):
    """Steps 1-4. Returns (logits [B,E], ids [B,k] int32, w [B,k])."""
    X = bf16_bits_to_f64(x)
    R = bf16_bits_to_f64(router_w)
    logits = X @ R
    if bias is not None:
        logits = logits + np.asarray(bias, dtype=np.float32).astype(np.float64)[None, :]
    B, E = logits.shape
    ids = np.zeros((B, k), dtype=np.int32)
    w = np.zeros((B, k), dtype=np.float64)
    for b in range(B):
        lg = logits[b]
        p = np.exp(lg - lg.max())
        p = p / p.sum()
        # lexsort: last key is primary -> logit descending, then id ascending
        order = np.lexsort((np.arange(E), -lg))
        sel = order[:k]
        ids[b] = sel
        w[b] = p[sel] / p[sel].sum()
    return logits, ids, w


def swiglu_mlp(xrow: np.ndarray, W13, W2) -> np.ndarray:
    """Step 5/6 for one token: xrow float64 [H], W13/W2 bf16 bits."""
    W13f = bf16_bits_to_f64(W13)
    W2f = bf16_bits_to_f64(W2)
    inter = W13f.shape[1] // 2
    gu = xrow @ W13f
    a = silu(gu[:inter]) * gu[inter:]
    return a @ W2f


def block(x, ids, w, w13, w2, sw13=None, sw2=None):
    """Steps 5-7 for the given routing.  w13/w2 are sequences indexed by expert."""
    X = bf16_bits_to_f64(x)
    B = X.shape[0]
    out = X.copy()
    for b in range(B):
        for j in range(ids.shape[1]):
            e = int(ids[b, j])
            out[b] += w[b, j] * swiglu_mlp(X[b], w13[e], w2[e])
        if sw13 is not None:
            out[b] += swiglu_mlp(X[b], sw13, sw2)
    return out


def moe_forward(x, router_w, w13, w2, sw13, sw2, k, bias=None):
    """Steps 1-7.  Returns (out [B,H] float64, ids, w, logits)."""
    logits, ids, w = router(x, router_w, k, bias)
    out = block(x, ids, w, w13, w2, sw13, sw2)
    return out, ids, w, logits
