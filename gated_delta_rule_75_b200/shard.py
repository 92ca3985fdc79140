"""Host-side partitioning of KDA work across GPUs.

Every (sequence, head) pair of the recurrence is independent, so a batch
shards across ranks with no exchange on the data path: each rank runs the
ordinary single-GPU call on its slice and the caller owns placement.  These
helpers pick the slices.  Pure Python, no CUDA.
"""
from typing import List, Sequence, Tuple


def head_range(H: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous, balanced split of H heads: rank gets [start, stop)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(H, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def sequence_assignment(lengths: Sequence[int], world: int) -> List[List[int]]:
    """Greedy longest-first assignment of packed sequences to ranks, balancing
    tokens (the sequential chunk loop of a sequence cannot be split further
    without a cross-rank scan).  Returns one sorted index list per rank."""
    if world < 1:
        raise ValueError("bad world")
    load = [0] * world
    out: List[List[int]] = [[] for _ in range(world)]
    for i in sorted(range(len(lengths)), key=lambda j: (-lengths[j], j)):
        r = min(range(world), key=lambda k: (load[k], k))
        out[r].append(i)
        load[r] += lengths[i]
    return [sorted(x) for x in out]
