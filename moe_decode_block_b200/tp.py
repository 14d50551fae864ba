"""Tensor-parallel split of one MoE decode block: argument marshalling only.

The pages run the block tensor-parallel (TP8 / TP16) with the ranks' expert
outputs exchanged over NVLink ("Hyper Optimizing Kimi K3 in vLLM", sections
"Recovering time between operators" and "Three performance comparisons
answer different questions").  Here rank r of tp holds the slice
[r * I / tp, (r + 1) * I / tp) of every expert's intermediate dimension --
the gate and up columns of w13 and the same rows of w2, for the routed and
the shared experts -- so the block's expert sum is the sum over ranks of
each rank's sum: SwiGLU acts column by column, and the down projection is a
sum over the intermediate rows.  Each rank runs an MOE_FLAG_PARTIAL_SUM
forward on its slice (the routing is the same on every rank: same x, same
router weights), then the partial sums are added and the residual applied by
moe_decode_reduce_residual -- reading the other ranks' buffers directly when
the caller has them mapped (peer memory over NVLink), or after an NCCL
all-reduce of the fp32 partials otherwise.
"""
from typing import Optional

from . import MoEDecode, reduce_residual


def shard_intermediate(w13, w2, rank: int, tp: int):
    """Rank `rank`'s slice of one expert (w13 [..., H, 2I], w2 [..., I, H])
    or of a stack of them ([E, H, 2I], [E, I, H]): (w13 [..., H, 2I/tp] --
    gate columns [r c, (r+1) c) then the same up columns, c = I / tp --,
    w2 [..., I/tp, H]), contiguous."""
    import torch
    inter = w2.shape[-2]
    if tp < 1 or inter % tp or not 0 <= rank < tp:
        raise ValueError(f"cannot give rank {rank} of {tp} a slice of inter {inter}")
    if w13.shape[-1] != 2 * inter:
        raise ValueError(f"w13 has {w13.shape[-1]} columns, expected {2 * inter}")
    c = inter // tp
    gate = w13[..., rank * c:(rank + 1) * c]
    up = w13[..., inter + rank * c:inter + (rank + 1) * c]
    return torch.cat([gate, up], dim=-1).contiguous(), w2[..., rank * c:(rank + 1) * c, :].contiguous()


class TPBlock:
    """One rank of a tensor-parallel block: a partial-sum handle for this
    rank's slice (inter / tp, shared_inter / tp) and the exchange.

    forward() runs the rank's forward into an fp32 buffer, then either
      * peers given: out = bf16(x + sum of the ranks' buffers) read directly.
        `peer_partials(rank_buffer)` is called once this rank's forward is
        enqueued and returns every rank's buffer, this one included, in rank
        order (device pointers the caller has mapped), after every rank's
        forward has completed (e.g. a stream synchronise, then a process-group
        barrier); the caller keeps the buffers until every rank's reduction
        has completed;
      * otherwise: an all-reduce of the buffer over `group`
        (torch.distributed, NCCL on GPUs) and the residual from the result.
    With tp == 1 it is the plain block (residual from the one buffer)."""

    def __init__(self, hidden: int, n_experts: int, top_k: int, inter: int, shared_inter: int, tp: int, rank: int,
                 n_shared: int = 1, max_batch: int = 64, router_bias=None, group=None, peer_partials=None):
        if inter % tp or (n_shared and shared_inter % tp):
            raise ValueError(f"inter {inter} / shared_inter {shared_inter} not divisible by tp {tp}")
        self.tp, self.rank, self.group, self.peer_partials = tp, rank, group, peer_partials
        self.hidden = hidden
        self.blk = MoEDecode(hidden, n_experts, top_k, inter // tp, shared_inter // tp if n_shared else 0,
                             n_shared=n_shared, max_batch=max_batch, router_bias=router_bias, partial=True)
        self.partial = None

    def forward(self, x, router_w, w13, w2, shared_w13, shared_w2, out, topk_ids, topk_w,
                batch: Optional[int] = None, stream=None):
        """w13 / w2 / shared_*: this rank's slices (shard_intermediate)."""
        import torch
        B = x.shape[0] if batch is None else batch
        if self.partial is None or self.partial.shape[0] < B:
            self.partial = torch.empty(max(B, 1), self.hidden, dtype=torch.float32, device=x.device)
        part = self.partial[:B]
        self.blk.forward(x, router_w, w13, w2, shared_w13, shared_w2, part, topk_ids, topk_w, batch=B,
                         stream_main=stream)
        if self.tp > 1 and self.peer_partials is not None:
            parts = self.peer_partials(part)
            if len(parts) != self.tp:
                raise ValueError(f"peer_partials gave {len(parts)} buffers for tp {self.tp}")
            reduce_residual(parts, x, out, stream=stream)
            return
        if self.tp > 1:
            import torch.distributed as dist
            with torch.cuda.stream(stream if stream is not None else torch.cuda.current_stream()):
                dist.all_reduce(part, op=dist.ReduceOp.SUM, group=self.group)
        reduce_residual([part], x, out, stream=stream)

    def close(self):
        self.blk.close()
