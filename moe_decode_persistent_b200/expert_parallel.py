"""Expert parallelism: one MoE decode layer split over the ranks of a torch.distributed
group by ranges of routed experts, router and shared expert replicated on every rank.

The pages spread the expert work over the GPUs and fold the cross-GPU exchange into the
computation (page post.smzdm.com/p/a6zppe4g, section "改了什么：每层 23 个 kernel 砍到
13 个", items "把通信缝进计算" and "MoE 去重"). Here rank r holds only the weights of
experts [e0_r, e1_r); every rank routes every row in full (the router is replicated), runs
its experts' share of the layer in one persistent launch (moe_decode_step_partial), and
one all-reduce of the fp32 partial outputs [batch, hidden] per step -- NCCL over
NVLink / NVSwitch on GPUs, gloo on the CPU -- gives the layer's output, rounded to bf16 by
moe_decode_partial_to_bf16. Exactly one rank (rank 0) adds the residual and the shared
expert. Since the sum is in fp32 before the one rounding to bf16, the result equals the
single-GPU layer up to the fp32 summation order.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import MoeDecode, partial_to_bf16


def expert_range(n_experts: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous experts [e0, e1) of `rank`: near-equal parts, the first n_experts mod
    world ranks one expert more."""
    if world < 1 or not 0 <= rank < world or n_experts < world:
        raise ValueError(f"expert_range: {n_experts} experts over {world} ranks, rank {rank}")
    base, extra = divmod(n_experts, world)
    e0 = rank * base + min(rank, extra)
    return e0, e0 + base + (1 if rank < extra else 0)


def adds_residual_shared(rank: int) -> bool:
    """Whether `rank`'s partial carries the residual x and the shared expert (rank 0)."""
    return rank == 0


def local_experts(layer: dict, e0: int, e1: int) -> dict:
    """The layer mapping with w_gate, w_up and w_down cut to experts [e0, e1) (views of
    expert-major tensors [E, ...]); everything else as given."""
    out = dict(layer)
    for name in ("w_gate", "w_up", "w_down"):
        out[name] = layer[name][e0:e1]
    return out


def reduce_partials(part: torch.Tensor, group=None) -> None:
    """In place: the sum of every rank's partial output (one all-reduce)."""
    dist.all_reduce(part, op=dist.ReduceOp.SUM, group=group)


class ExpertParallelLayer:
    """This rank's share of one expert-parallel layer on `device`.

    layer: gamma, w_router, router_bias, ws_gate, ws_up, ws_down of the whole layer and
    w_gate, w_up, w_down of this rank's experts only ([e1 - e0, ...], see
    local_experts and expert_range). Every rank calls step with the same rows."""

    def __init__(self, hidden, n_experts, top_k_max, inter, shared_inter, max_batch, layer, group=None,
                 eps=1e-6, device=0):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.e0, self.e1 = expert_range(n_experts, self.world, self.rank)
        self.device = int(device)
        self.hidden = hidden
        self.handle = MoeDecode(hidden, n_experts, top_k_max, inter, shared_inter, max_batch, [layer], eps=eps,
                                device=device, expert_range=(self.e0, self.e1))
        self.part = torch.empty((max_batch, hidden), dtype=torch.float32, device=f"cuda:{self.device}")

    def step(self, x, y, batch, top_k) -> None:
        """y <- the layer's output for rows x (device bf16 [batch, hidden] each), on the
        current stream of this rank's device; every rank of the group must call it."""
        stream = torch.cuda.current_stream(self.device)
        part = self.part[:batch]
        self.handle.step_partial(x, part, batch, top_k, residual_shared=adds_residual_shared(self.rank),
                                 stream=stream)
        reduce_partials(part, self.group)
        partial_to_bf16(part, y, self.device, stream)

    def close(self) -> None:
        self.handle.close()
