"""Expert-parallel execution of the layer across ranks (one process per GPU).

MAX DeepseekV41Config's ep_config shards the routed experts "only under data
parallelism": every rank brings its own tokens, holds one window of the routed
experts and the whole router. One step:

  1. all-gather the ranks' token rows (every rank then routes every token with
     the same router, so all ranks agree on the selection without exchanging it);
  2. each rank runs the selected slots whose expert lies in its window (and the
     shared experts, on the one rank that holds them): a partial output in fp32
     for every gathered token;
  3. reduce-scatter the partial outputs: each rank receives the sum for its own
     tokens, which is the layer's output.

The collectives are torch.distributed's (NCCL between GPUs). The partial
computation is the library's moe_forward_partial; a test may pass any function
of the gathered tokens instead (the host-side plumbing is then exercised with
gloo on CPU).
"""
from __future__ import annotations

from typing import Callable, Optional

import torch
import torch.distributed as dist


def expert_window(n_routed: int, world: int, rank: int):
    """(first expert, expert count) of `rank`'s window: n_routed split into `world`
    contiguous windows as evenly as possible (the first n_routed % world get one more)."""
    if not (1 <= world <= n_routed) or not (0 <= rank < world):
        raise ValueError("need 1 <= world <= n_routed and 0 <= rank < world")
    base, extra = divmod(n_routed, world)
    begin = rank * base + min(rank, extra)
    return begin, base + (1 if rank < extra else 0)


class ExpertParallelLayer:
    """The layer over a process group: each rank holds one expert window.

    partial: a function of the gathered tokens x_all [world * T, H] (BF16) giving
    this rank's fp32 partial output [world * T, H]; normally MoELayer.forward_partial
    of a layer created with this rank's expert_window.
    """

    def __init__(self, partial: Callable[[torch.Tensor], torch.Tensor], group: Optional[dist.ProcessGroup] = None):
        self.partial = partial
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        """x: this rank's tokens [T, H] (the same T on every rank). Returns its output
        rows [T, H] in fp32 (the sum of every rank's partial output)."""
        T, H = x.shape
        x_all = torch.empty((self.world * T, H), dtype=x.dtype, device=x.device)
        dist.all_gather_into_tensor(x_all, x.contiguous(), group=self.group)
        y_all = self.partial(x_all)
        if tuple(y_all.shape) != (self.world * T, H) or y_all.dtype != torch.float32:
            raise ValueError("the partial output must be fp32 [world * T, H]")
        y = torch.empty((T, H), dtype=torch.float32, device=x.device)
        dist.reduce_scatter_tensor(y, y_all.contiguous(), op=dist.ReduceOp.SUM, group=self.group)
        return y

    __call__ = forward
