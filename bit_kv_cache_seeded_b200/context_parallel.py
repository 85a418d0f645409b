"""Context-parallel decode: the context of every sequence split over ranks, one cache shard each.

Each rank's cache holds a disjoint, contiguous range of every sequence's tokens (same configuration
and seeds on every rank). A decode step is then:
  1. kvq_decode_partials on the local shard: the softmax state (m, l, unnormalised o) of every
     (sequence, query head) over the local tokens, [batch, n_q_heads, 2 + dv] floats;
  2. one all-gather of those states over the process group (NCCL over NVLink on GPUs) -- for the
     64-head MLA cache that is 64 x 514 floats per sequence and rank;
  3. kvq_combine_partials: the log-sum-exp merge of all ranks' states, giving every rank the
     output over the whole context.
This is argument marshalling and the exchange only; the arithmetic runs in libkvq.so's kernels.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import kvq_combine_partials


def shard_range(ctx: int, rank: int, world: int) -> tuple[int, int]:
    """The contiguous token range [begin, end) of a ctx-token context that rank `rank` holds: the
    first ctx % world ranks take one token more."""
    base, extra = divmod(ctx, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def exchange_states(local: torch.Tensor, group=None) -> torch.Tensor:
    """All ranks' states in rank order: [world, *local.shape] on local's device."""
    world = dist.get_world_size(group)
    out = torch.empty((world, *local.shape), dtype=local.dtype, device=local.device)
    if local.is_cuda:
        dist.all_gather_into_tensor(out, local.contiguous(), group=group)
    else:  # gloo: list form
        dist.all_gather(list(out.unbind(0)), local.contiguous(), group=group)
    return out


def context_parallel_decode(cache, q: torch.Tensor, out: torch.Tensor | None = None, group=None,
                            stream=None) -> torch.Tensor:
    """Decode attention of q over the context of all ranks' shards (every rank gets out)."""
    local = cache.decode_partials(q, stream=stream)
    states = exchange_states(local, group)
    if out is None:
        out = torch.empty((cache.batch, cache.cfg.n_q_heads, cache.out_dim), dtype=torch.float32, device=q.device)
    kvq_combine_partials(states, out, stream=stream)
    return out
