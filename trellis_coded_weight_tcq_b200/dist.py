"""Host-side helpers for running the encoder on several GPUs, one process each.

Coding blocks are independent (each block's Viterbi search and its stored start
state concern that block alone), so the work shards by block with no exchange
on the data path.  Two ways to split:

* weak scaling: every rank encodes a whole matrix of its own
  (``workload_for_rank``), the way ``bench.py --gpus N`` runs;
* strong scaling: one matrix, contiguous block ranges per rank
  (``block_range``).

The only collective is the timing reduction (``max_over_ranks``), taken after
the timed region.
"""
from __future__ import annotations


def block_range(n_blocks: int, rank: int, world: int) -> tuple[int, int]:
    """[begin, end) of the blocks rank owns: contiguous, balanced to one block."""
    if world < 1 or not 0 <= rank < world or n_blocks < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(n_blocks, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def workload_for_rank(name: str, rank: int):
    """The rank's own matrix of the named workload (seeds offset by rank)."""
    from . import workloads

    return workloads.NAMED[name](rank)


def max_over_ranks(values, device=None):
    """Element-wise maximum of a list of floats over all ranks (all_reduce MAX).

    With one process (or no process group) the values come back unchanged.
    """
    import torch
    import torch.distributed as dist

    vals = [float(v) for v in values]
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu().tolist()]
