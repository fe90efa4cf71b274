"""Expert-parallel routed-expert layer across ranks (one process per GPU).

"Tech2wild/Nex-N2.5-mini-Int4-Int8Mix", Serving: the model is served with
expert parallelism over a pair of GPUs.  Here rank g of G holds the packed
banks of one contiguous block of experts (expert_range) and its own tokens.
One layer forward:

  1. all-gather the ranks' tokens (NCCL), in rank order;
  2. moe_forward_partial on every rank: routing over all E experts (the router
     weight is replicated, so every rank routes identically) and the fp32
     contribution of the rank's own experts;
  3. reduce-scatter (sum) of the fp32 contributions: each rank receives the
     sum for its own tokens;
  4. moe_partial_to_bf16: the single bf16 rounding of the layer output.

Every step of the layer runs in the library's kernels; torch.distributed only
moves the tokens and the partial sums.  The exchange is plain NCCL (or, for
host-side tests, gloo); no kernel here reads another GPU's memory.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch
import torch.distributed as dist

from . import _binding as moe


def expert_range(num_experts: int, rank: int, world: int):
    """(first expert, number of experts) of `rank`: contiguous blocks, the
    first num_experts % world ranks holding one expert more."""
    if world < 1 or not 0 <= rank < world or num_experts < world:
        raise ValueError("need 0 <= rank < world <= num_experts")
    base, extra = divmod(num_experts, world)
    begin = rank * base + min(rank, extra)
    return begin, base + (1 if rank < extra else 0)


def _all_gather_rows(x_local: torch.Tensor, world: int, group) -> torch.Tensor:
    if dist.get_backend(group) == "nccl":
        out = torch.empty((world * x_local.shape[0],) + tuple(x_local.shape[1:]), dtype=x_local.dtype,
                          device=x_local.device)
        dist.all_gather_into_tensor(out, x_local.contiguous(), group=group)
        return out
    parts = [torch.empty_like(x_local) for _ in range(world)]
    dist.all_gather(parts, x_local.contiguous(), group=group)
    return torch.cat(parts)


def _reduce_scatter_rows(partial: torch.Tensor, rank: int, world: int, group) -> torch.Tensor:
    rows = partial.shape[0] // world
    if dist.get_backend(group) == "nccl":
        out = torch.empty((rows,) + tuple(partial.shape[1:]), dtype=partial.dtype, device=partial.device)
        dist.reduce_scatter_tensor(out, partial.contiguous(), op=dist.ReduceOp.SUM, group=group)
        return out
    # gloo has no reduce-scatter: the full sum, then this rank's rows
    dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=group)
    return partial[rank * rows:(rank + 1) * rows].contiguous()


class ExpertParallelLayer:
    """One routed-expert layer sharded by experts over the ranks of `group`.

    shape: the layer's moe_shape_t (num_experts = all E); router_w [E, H] bf16
    (replicated); gate_up_local / down_local: this rank's packed banks of the
    experts expert_range(E, rank, world).  Every rank calls forward() with the
    same number of tokens.  `partial_fn(x_all) -> fp32 [T, H]` and
    `finalize_fn(fp32 [T_local, H]) -> output` replace the CUDA calls only in
    host-side tests of the exchange.
    """

    def __init__(self, shape, router_w, gate_up_local, down_local, group=None, bias=None, path=None,
                 partial_fn: Optional[Callable] = None, finalize_fn: Optional[Callable] = None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.shape, self.router_w, self.bias, self.path = shape, router_w, bias, path
        self.expert_begin, self.num_local = expert_range(shape.num_experts, self.rank, self.world)
        self.gate_up, self.down = gate_up_local, down_local
        self.partial_fn = partial_fn or self._partial
        self.finalize_fn = finalize_fn or moe.moe_partial_to_bf16
        self._ws, self._ws_T = None, -1

    def _partial(self, x_all: torch.Tensor) -> torch.Tensor:
        T = x_all.shape[0]
        if self._ws_T != T:
            self._ws = moe.alloc_workspace(self.shape, T, device=x_all.device)
            self._ws_T = T
        return moe.moe_forward_partial(self.shape, x_all, self.router_w, self.expert_begin, self.num_local,
                                       self.gate_up, self.down, self._ws, bias=self.bias, path=self.path)

    def forward(self, x_local: torch.Tensor) -> torch.Tensor:
        x_all = _all_gather_rows(x_local, self.world, self.group)
        partial = self.partial_fn(x_all)
        mine = _reduce_scatter_rows(partial, self.rank, self.world, self.group)
        return self.finalize_fn(mine)
