"""Sharding packed sequences across ranks (one process per GPU, no data exchange).

Sequences and heads of the KDA recurrence are independent, so a multi-GPU run
gives each rank a subset of the sequences of a packed batch and runs the 1-GPU
library on it; nothing crosses ranks but the timing reduction.
"""
from __future__ import annotations

import numpy as np


def partition_sequences(lengths, world_size: int):
    """Longest-processing-time assignment of sequences to ranks.

    Returns a list (one per rank) of sorted sequence indices. Every sequence is
    assigned to exactly one rank; ties go to the lowest rank, so the result is
    deterministic and identical on every rank.
    """
    if world_size <= 0:
        raise ValueError("world_size must be positive")
    lengths = [int(x) for x in lengths]
    order = sorted(range(len(lengths)), key=lambda i: (-lengths[i], i))
    load = [0] * world_size
    shards = [[] for _ in range(world_size)]
    for i in order:
        r = min(range(world_size), key=lambda k: (load[k], k))
        shards[r].append(i)
        load[r] += lengths[i]
    return [sorted(s) for s in shards]


def gather_shard(cu_seqlens, seqs):
    """Token index array and cu_seqlens of the packed sub-batch made of sequences `seqs`."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    idx = np.concatenate([np.arange(cu[s], cu[s + 1]) for s in seqs]) if seqs else np.zeros(0, np.int64)
    lens = [int(cu[s + 1] - cu[s]) for s in seqs]
    sub = np.zeros(len(seqs) + 1, dtype=np.int64)
    if lens:
        sub[1:] = np.cumsum(lens)
    return idx, sub
