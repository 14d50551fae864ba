"""A stack of MoE decode blocks run back to back on one stream: argument
marshalling only.

The pages overlap consecutive operators of a decode step instead of draining
the GPU between them ("Hyper Optimizing Kimi K3 in vLLM", section
"Recovering time between operators": dependent work starts as soon as it
can, and upcoming weights are fetched before their consumer starts).  Here
each block has its own handle -- its own workspace and tensor maps, bound to
that block's weights and never rewritten -- and block l's output is block
l + 1's input.  Every kernel of a forward is launched with programmatic
dependent launch and the router stages its slab of router_w before it waits
for the grid before it, so block l + 1's router weights stream in while block
l's combine is still running, and block l + 1's shared expert starts as soon
as its router has passed that wait.
"""
from typing import Optional, Sequence

from . import MoEDecode


def check_chain_args(n_blocks: int, weights: Sequence, outs: Sequence, topk_ids: Sequence, topk_w: Sequence):
    """Raise ValueError unless every per-block sequence has one entry per block
    and every weight entry is (router_w, w13, w2, shared_w13, shared_w2)."""
    if n_blocks < 1:
        raise ValueError("a chain needs at least one block")
    for name, seq in (("weights", weights), ("outs", outs), ("topk_ids", topk_ids), ("topk_w", topk_w)):
        if len(seq) != n_blocks:
            raise ValueError(f"{name}: {len(seq)} entries for {n_blocks} blocks")
    for l, w in enumerate(weights):
        if len(w) != 5:
            raise ValueError(f"weights[{l}]: expected (router_w, w13, w2, shared_w13, shared_w2), got {len(w)} items")
    for l in range(n_blocks):
        if outs[l] is None:
            raise ValueError(f"outs[{l}] is None")
        if l + 1 < n_blocks and outs[l] is outs[l + 1]:
            raise ValueError(f"outs[{l}] and outs[{l + 1}]: a block's input and output must be distinct buffers")


class BlockChain:
    """n_blocks blocks of one shape, one handle each (router_biases: one
    per block, or None)."""

    def __init__(self, n_blocks: int, hidden: int, n_experts: int, top_k: int, inter: int, shared_inter: int,
                 n_shared: int = 1, max_batch: int = 64, router_biases: Optional[Sequence] = None):
        if n_blocks < 1:
            raise ValueError("a chain needs at least one block")
        if router_biases is not None and len(router_biases) != n_blocks:
            raise ValueError(f"router_biases: {len(router_biases)} entries for {n_blocks} blocks")
        self.blocks = []
        try:
            for l in range(n_blocks):
                self.blocks.append(MoEDecode(hidden, n_experts, top_k, inter, shared_inter, n_shared=n_shared,
                                             max_batch=max_batch,
                                             router_bias=None if router_biases is None else router_biases[l]))
        except Exception:
            self.close()
            raise

    def forward(self, x, weights: Sequence, outs: Sequence, topk_ids: Sequence, topk_w: Sequence,
                batch: Optional[int] = None, stream=None):
        """Enqueue the chain: block 0 reads x, block l > 0 reads outs[l - 1];
        block l writes outs[l], topk_ids[l], topk_w[l].  weights[l] =
        (router_w, w13, w2, shared_w13, shared_w2) of block l."""
        check_chain_args(len(self.blocks), weights, outs, topk_ids, topk_w)
        if outs[0] is x:
            raise ValueError("outs[0] is x: a block's input and output must be distinct buffers")
        for l, blk in enumerate(self.blocks):
            blk.forward(x if l == 0 else outs[l - 1], *weights[l], outs[l], topk_ids[l], topk_w[l], batch=batch,
                        stream_main=stream)

    def status(self):
        """The first non-OK device status of the blocks (MOE_OK when none)."""
        for blk in self.blocks:
            st = blk.status()
            if st != 0:
                return st
        return 0

    def close(self):
        for blk in self.blocks:
            blk.close()
        self.blocks = []
