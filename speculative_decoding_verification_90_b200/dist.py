"""Host-side plumbing of the multi-GPU run: one process per GPU.

Sequences of a verification batch are independent, so the step shards with no
data-path collective: each rank verifies its own sequences and the only
communication is the timing reduction (max over ranks) and, when a caller wants
the whole batch's outputs on one rank, a gather of the small int32 outputs.
"""
from __future__ import annotations

import os
from datetime import timedelta


def env_rank() -> tuple[int, int, int]:
    """(rank, local_rank, world_size) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def init(backend: str, device=None, timeout_s: float = 120.0):
    """Initialise the default process group (short timeout: ranks that wait on
    one another end with an error instead of hanging)."""
    import torch.distributed as dist
    kw = {"timeout": timedelta(seconds=timeout_s)}
    if device is not None:
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def shard(batch: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous sequence range [lo, hi) of `rank` when one batch is split."""
    if world < 1 or not (0 <= rank < world):
        raise ValueError("rank outside the world")
    return batch * rank // world, batch * (rank + 1) // world


def rank_seed(seed: int, rank: int) -> int:
    """Seed of rank `rank`'s own batch in a weak-scaling run."""
    return seed + 1000003 * rank


def max_over_ranks(value: float, device=None) -> float:
    """The largest value over all ranks (e.g. a device time)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def gather_outputs(out_tokens, out_num_accepted):
    """All ranks' (out_tokens, out_num_accepted) concatenated in rank order
    (int32 tensors of equal shape on every rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return out_tokens, out_num_accepted
    w = dist.get_world_size()
    toks = [torch.empty_like(out_tokens) for _ in range(w)]
    nums = [torch.empty_like(out_num_accepted) for _ in range(w)]
    dist.all_gather(toks, out_tokens.contiguous())
    dist.all_gather(nums, out_num_accepted.contiguous())
    return torch.cat(toks), torch.cat(nums)
