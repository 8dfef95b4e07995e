"""Host logic for running the decode path on several GPUs, one process per GPU.

Every decode sequence is independent of every other, and each data-parallel
group keeps a full copy of the MLA layer and runs it on its own inputs ("Lower
latency and higher throughput with multi-node DeepSeek deployment", section
"Data parallelism").  So the attention path has no exchange step: ranks
never talk on the data path.  The only collectives are for bookkeeping after
the timed region: the max over ranks of each timing and the OR of the device
status words.

Two ways to give ranks work:
  * weak scaling (what the benchmark does): every rank decodes its own batch of
    the same shape, drawn with `replica_seed(seed, rank)`;
  * strong scaling: one global batch of sequences split across ranks by
    `shard_sequences`, which balances the cached tokens each rank reads.
"""
from __future__ import annotations

from typing import List, Sequence

import torch


def replica_seed(seed: int, rank: int) -> int:
    """Seed of rank `rank`'s synthetic batch (distinct per rank, same shape)."""
    return int(seed) + 1000 * int(rank)


def shard_sequences(seq_lens: Sequence[int], world: int) -> List[List[int]]:
    """Split sequence indices over `world` ranks, balancing the sum of T.

    The attention kernel reads each cached token once, so a rank's time is
    close to proportional to its total T.  This is a longest-first greedy:
    sequences in descending T (ties: lower index first) each go to the rank
    with the least total so far (ties: lower rank).  Each rank's list comes
    back in ascending index order.  A rank may get no sequence when there
    are fewer sequences than ranks.
    """
    if world < 1:
        raise ValueError("world must be >= 1")
    lens = [int(t) for t in seq_lens]
    if any(t < 0 for t in lens):
        raise ValueError("sequence lengths must be non-negative")
    load = [0] * world
    shards: List[List[int]] = [[] for _ in range(world)]
    for i in sorted(range(len(lens)), key=lambda k: (-lens[k], k)):
        r = min(range(world), key=lambda q: (load[q], q))
        shards[r].append(i)
        load[r] += lens[i]
    return [sorted(s) for s in shards]


def reduce_max(values: Sequence[float], device=None) -> List[float]:
    """Element-wise max over all ranks (one all-reduce); identity when not distributed."""
    vals = [float(v) for v in values]
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def reduce_status(status: int, device=None) -> int:
    """Bitwise OR of every rank's device status word (one all-gather).

    NCCL has no bitwise reduction, so the words are gathered and OR-ed on the host.
    """
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return int(status)
    world = torch.distributed.get_world_size()
    mine = torch.tensor([int(status)], dtype=torch.int32, device=device)
    parts = [torch.empty_like(mine) for _ in range(world)]
    torch.distributed.all_gather(parts, mine)
    out = 0
    for p in parts:
        out |= int(p.item())
    return out
