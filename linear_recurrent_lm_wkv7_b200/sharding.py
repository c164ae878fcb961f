"""Splitting a batch of independent sequences across ranks.

Every (sequence, head) unit of the WKV-7 recurrence is independent of every
other one (the state is per sequence and head), so a batch shards across GPUs
without any exchange on the data path: each rank runs ``wkv7_forward`` on its
own sequences and owns their outputs and final states.  The only host-side
decision is which sequences go where; for packed variable-length batches the
assignment balances token counts (longest sequences first, each to the least
loaded rank).

Nothing here computes the operator; the collective helpers below exist only to
gather shards for checking and are not on the compute path.
"""
from __future__ import annotations

from typing import List, Sequence


def assign_sequences(lengths: Sequence[int], world_size: int) -> List[List[int]]:
    """Indices of the sequences each rank owns, balanced by length.

    Greedy longest-processing-time assignment; ties go to the lower rank and
    each rank's list is returned in ascending sequence order, so the result is
    deterministic and identical on every rank."""
    if world_size <= 0:
        raise ValueError("world_size must be positive")
    loads = [0] * world_size
    owned: List[List[int]] = [[] for _ in range(world_size)]
    order = sorted(range(len(lengths)), key=lambda i: (-int(lengths[i]), i))
    for i in order:
        rk = min(range(world_size), key=lambda q: (loads[q], q))
        owned[rk].append(i)
        loads[rk] += int(lengths[i])
    return [sorted(o) for o in owned]


def packed_shard(offsets: Sequence[int], owned: Sequence[int]):
    """Token ranges and new offsets for a rank's sequences of a packed batch.

    Returns ``(ranges, new_offsets)``: ``ranges`` lists the (start, end) token
    slices of the original packed axis in the order of ``owned``, and
    ``new_offsets`` (len(owned) + 1 entries) describes the rank's own packed
    batch made by concatenating those slices."""
    ranges = [(int(offsets[i]), int(offsets[i + 1])) for i in owned]
    new = [0]
    for s, e in ranges:
        new.append(new[-1] + (e - s))
    return ranges, new


def dense_shard(batch: int, world_size: int, rank: int) -> range:
    """Contiguous block of sequences of a dense [B, T, H, D] batch for one rank
    (sizes differ by at most one)."""
    base, extra = divmod(batch, world_size)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))
