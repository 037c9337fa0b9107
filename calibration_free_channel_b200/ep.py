"""Expert parallelism for the reader: one process per GPU, expert e owned by
rank e % world.  The router is replicated, so every rank routes the whole
step; each rank reads and computes only the (token, slot) pairs of the
experts it owns and produces an fp32 partial of the block output.  One
all-reduce (NCCL over NVLink on GPUs) sums the partials; the finish adds the
residual and rounds once to bf16.  The only data exchange of the block is
that sum of [B, d] fp32 per layer.

The step is split into `ep_step` (the exchange, independent of how the
partial was computed) and `ep_forward` (the CUDA path through the C ABI)."""
from __future__ import annotations

import torch
import torch.distributed as dist


def owned_experts(E: int, rank: int, world: int) -> list[int]:
    """The experts rank `rank` reads: e % world == rank."""
    return [e for e in range(E) if e % world == rank]


def shard_weights(W: dict, rank: int, world: int):
    """The weights rank `rank` holds: the router whole, w_gate / w_up /
    w_down of the experts e % world == rank stacked in that order, and the
    [E] int32 slot map (e // world for them, -1 elsewhere) that
    moe_reader_layer.expert_slot takes."""
    E = W["w_router"].shape[0]
    own = list(range(rank, E, world))
    idx = torch.tensor(own, dtype=torch.long)
    out = {n: (v if v is None or n in ("w_router", "router_bias") else v.index_select(0, idx.to(v.device)))
           for n, v in W.items()}
    slot = torch.full((E,), -1, dtype=torch.int32)
    slot[idx] = torch.arange(len(own), dtype=torch.int32)
    return out, slot


def ep_step(partial: torch.Tensor, finish, group=None):
    """Sums this rank's fp32 partial [B, d] over the group in place (one
    all-reduce) and returns finish(sum)."""
    dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=group)
    return finish(partial)


def ep_forward(layer, x: torch.Tensor, k: int, c: int, residual: torch.Tensor | None = None, group=None,
               recovery_input: int = 0, stream=None) -> torch.Tensor:
    """One expert-parallel MoE block on this rank's GPU: partial through the
    C ABI, all-reduce over `group`, finish on the GPU; returns y [B, d] bf16."""
    from calibration_free_channel_b200 import moe_reader as M
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    B, d = x.shape
    yp = layer.forward_ep(x, k, c, rank, world, stream=stream, recovery_input=recovery_input)

    def finish(y_sum):
        y = torch.empty_like(x)
        M.moe_reader_ep_finish(B, d, y_sum, residual, y, stream)
        return y

    return ep_step(yp, finish, group)
