"""Expert-parallel sharding of the block over a process group (one process per GPU).

Each rank holds one contiguous range of the routed experts (their stacked planes only) and
a replica of every dense plane (router, coefficient head, shared expert, latent
projections); every rank receives the same token batch. One step:

  1. route every token (moe_route) and permute the slots by expert (moe_permute);
  2. latent block: z = x Wdp^T (moe_latent_down);
  3. run the local experts into a partial fp32 routed sum y_acc [T, K]
     (moe_grouped_ffn_experts);
  4. reduce-scatter the partial sums over the ranks along the token dimension: rank r
     receives the complete routed sum of its token shard (the one exchange step; NCCL over
     NVLink on GPUs);
  5. finish the shard (moe_combine): shared expert, add or blend, and for the latent block
     RMSNorm and the up projection.

Argument marshalling and the collective only: every step of the block runs in the CUDA
library. The pages run the block on one device; this split follows the block's own
structure (the routed sum is the only quantity that needs every expert).
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Tuple

import torch

from . import moe as M

# moe_weights fields that hold stacked routed-expert planes [E, ...]
ROUTED_PLANES = frozenset({
    "gate_w", "up_w", "gate_up_w", "gate_b", "up_b", "gate_up_b", "down_w", "down_b",
    "gate_s", "gate_z", "up_s", "up_z", "down_s", "down_z", "gate_up_s", "gate_up_z",
})


def expert_range(num_experts: int, world: int, rank: int) -> Tuple[int, int]:
    """[begin, end) of the routed experts rank `rank` holds: contiguous ranges whose sizes
    differ by at most one and cover [0, num_experts) once."""
    if not (0 <= rank < world) or num_experts < world:
        raise ValueError("every rank needs at least one expert")
    base, rem = divmod(num_experts, world)
    begin = rank * base + min(rank, rem)
    return begin, begin + base + (1 if rank < rem else 0)


def shard_rows(T: int, world: int) -> int:
    """Token rows per rank in the reduce-scatter: T rounded up to a multiple of `world`
    shards, each a multiple of 8 rows (every shard's slices stay 16-byte aligned)."""
    return max(8, 8 * math.ceil(T / (8 * world)))


def token_range(T: int, world: int, rank: int) -> Tuple[int, int]:
    """[t0, t1) of the tokens whose block output rank `rank` produces (may be empty)."""
    per = shard_rows(T, world)
    t0 = min(T, rank * per)
    return t0, min(T, t0 + per)


def local_weights(weights: Dict[str, torch.Tensor], begin: int, end: int) -> Dict[str, torch.Tensor]:
    """The rank's weights: routed planes cut to experts [begin, end), dense planes whole."""
    return {k: (v[begin:end].contiguous() if k in ROUTED_PLANES else v) for k, v in weights.items()}


def reduce_scatter_routed(partial: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """Sum the ranks' partial routed sums [world * rows, K] and return this rank's
    [rows, K] shard (rank r gets rows [r * rows, (r + 1) * rows))."""
    rows = partial.shape[0] // world
    if world == 1:
        return partial
    import torch.distributed as dist
    out = torch.empty((rows, partial.shape[1]), dtype=partial.dtype, device=partial.device)
    dist.reduce_scatter_tensor(out, partial.contiguous(), group=group)
    return out


class ExpertParallelBlock:
    """One rank's share of an expert-parallel block (see the module docstring)."""

    def __init__(self, spec, weights: Dict[str, torch.Tensor], max_tokens: int, group=None,
                 device: str = "cuda"):
        import torch.distributed as dist
        initialized = dist.is_available() and dist.is_initialized()
        self.world = dist.get_world_size(group) if initialized else 1
        self.rank = dist.get_rank(group) if initialized else 0
        self.group = group
        self.spec = spec
        self.begin, self.end = expert_range(spec.num_experts, self.world, self.rank)
        self.block = M.MoeBlock(spec, local_weights(weights, self.begin, self.end),
                                max_tokens=max(max_tokens, shard_rows(max_tokens, self.world)), device=device)

    def forward(self, x: torch.Tensor, stream=None) -> Tuple[torch.Tensor, Tuple[int, int]]:
        """x [T, hidden] (the same on every rank) -> (this rank's output rows, (t0, t1))."""
        b, spec = self.block, self.spec
        T, dev = x.shape[0], x.device
        k, E, K = spec.top_k, spec.num_experts, spec.expert_in
        i32 = dict(dtype=torch.int32, device=dev)
        idx = torch.empty((T, k), **i32)
        wts = torch.empty((T, k), dtype=torch.float32, device=dev)
        coef = torch.empty((T, 2), dtype=torch.float32, device=dev)
        off, ss, sp = torch.empty(E + 1, **i32), torch.empty(T * k, **i32), torch.empty(T * k, **i32)
        M.moe_route(b.cfg, b.w, x, T, idx, wts, coef, b.ws, stream)
        M.moe_permute(b.cfg, idx, T, off, ss, sp, b.ws, stream)
        u = x
        if spec.latent_dim:
            u = torch.empty((T, spec.latent_dim), dtype=b.act_dtype, device=dev)
            M.moe_latent_down(b.cfg, b.w, x, T, u, b.ws, stream)
        rows = shard_rows(T, self.world)
        partial = torch.zeros((rows * self.world, K), dtype=torch.float32, device=dev)
        M.moe_grouped_ffn_experts(b.cfg, b.w, u, T, off, ss, wts, self.begin, self.end, partial, b.ws, stream)
        if stream is not None:
            torch.cuda.current_stream().wait_stream(stream)
        shard = reduce_scatter_routed(partial, self.world, self.group)
        t0, t1 = token_range(T, self.world, self.rank)
        y = torch.empty((t1 - t0, spec.hidden), dtype=b.act_dtype, device=dev)
        if t1 > t0:
            M.moe_combine(b.cfg, b.w, shard, x[t0:t1], coef[t0:t1], t1 - t0, y, b.ws, stream)
        return y, (t0, t1)
