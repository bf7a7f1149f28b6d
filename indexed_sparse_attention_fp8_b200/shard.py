"""Sharding plans for running one DSA layer-group workload on several GPUs, one process per GPU.

Every query row of the path is independent: its indexer row, its top-k and its attention read
only the (replicated) key caches and its own inputs.  So the work shards with no exchange at
all.
  * Prefill (one long sequence of T new queries): the rows are cut into 2*world contiguous
    chunks of nearly equal length and rank r takes chunks r and 2*world-1-r ("zig-zag").  The
    indexer's work per row grows with the row's position (it scores every visible key), so
    pairing an early chunk with a late one gives every rank about the same number of visible
    (query, key) pairs; the attention's work is k keys per row, the same for every row.
  * Decode (B sequences of one new token): rank r takes a contiguous slice of the batch.
A chunk runs as its own dsa_group_forward call whose T is the chunk length and whose
ctx_len is the chunk's end, so the position rule pos = ctx_len - T + t places every row at its
position in the whole sequence and the call computes exactly what the unsharded call computes
for those rows.

This module only plans: it holds none of the method's arithmetic.
"""
from __future__ import annotations

from typing import List, Tuple


def _cut(n: int, parts: int) -> List[Tuple[int, int]]:
    """[0, n) cut into `parts` contiguous pieces whose lengths differ by at most one."""
    base, extra = divmod(n, parts)
    out, s = [], 0
    for i in range(parts):
        e = s + base + (1 if i < extra else 0)
        out.append((s, e))
        s = e
    return out


def zigzag_chunks(T: int, world: int, rank: int) -> List[Tuple[int, int]]:
    """Query-row ranges [t0, t1) of rank `rank` for a prefill of T rows over `world` ranks:
    chunks rank and 2*world-1-rank of 2*world contiguous chunks (empty ranges dropped)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    cuts = _cut(T, 2 * world)
    picks = [cuts[rank], cuts[2 * world - 1 - rank]]
    return [(a, b) for a, b in picks if b > a]


def batch_slice(B: int, world: int, rank: int) -> Tuple[int, int]:
    """Sequence range [b0, b1) of rank `rank` for a decode batch of B sequences."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    return _cut(B, world)[rank]


def visible_pairs(ctx: int, T: int, t0: int, t1: int, S: int, pool: int = 1) -> int:
    """Indexer work of rows t0..t1-1 of a sequence whose T new queries end at position ctx-1:
    the number of visible (query, key row) pairs, key rows being pooled blocks when pool > 1."""
    n = 0
    for t in range(t0, t1):
        pos = ctx - T + t
        if pos >= 0:
            n += min(S // pool, pos // pool + 1)
    return n


def plan(workload, world: int, rank: int):
    """The shards of one workload for one rank: a list of (b0, b1, t0, t1) boxes of
    (sequence, query-row) ranges.  Prefill (T > 1) shards the rows zig-zag over every
    sequence; decode (T == 1) shards the batch."""
    if workload.T == 1:
        b0, b1 = batch_slice(workload.B, world, rank)
        return [(b0, b1, 0, 1)] if b1 > b0 else []
    return [(0, workload.B, t0, t1) for t0, t1 in zigzag_chunks(workload.T, world, rank)]
