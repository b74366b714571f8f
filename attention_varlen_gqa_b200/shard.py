"""Partition of one packed varlen batch across ranks (one process per GPU).

The sequences of a varlen batch are independent problems: the attention of a
sequence reads only its own queries, keys and values.  A batch therefore
shards by whole sequences with no data exchange between ranks: every rank
gathers its sequences' rows, runs the same kernels on them and keeps its
outputs.  The partition balances work, not sequence counts: a sequence costs
its number of allowed (query, key) pairs, which the forward's FLOPs are
proportional to (causal masking is bottom-right aligned, as in the kernels),
and sequences are dealt heaviest first, each to the rank with the least work
so far (longest-processing-time list scheduling, which ends within 4/3 of
the best possible largest load).

Host logic only (numpy); nothing here touches a GPU.
"""
from __future__ import annotations

import numpy as np


def sequence_cost(s_q: int, s_k: int, causal: bool) -> int:
    """Allowed (query, key) pairs of one sequence: s_q * s_k without a mask;
    with bottom-right causal alignment row i sees keys j <= i + s_k - s_q."""
    s_q, s_k = int(s_q), int(s_k)
    if s_q <= 0 or s_k <= 0:
        return 0
    if not causal:
        return s_q * s_k
    return int(np.clip(np.arange(s_q, dtype=np.int64) + (s_k - s_q + 1), 0, s_k).sum())


def lpt_partition(costs, world: int) -> list[list[int]]:
    """Indices of `costs` dealt to `world` ranks: heaviest first (ties in index
    order), each to the least-loaded rank (ties to the lower rank).  Returns,
    per rank, its indices in ascending order."""
    if world < 1:
        raise ValueError("world must be >= 1")
    costs = [int(c) for c in costs]
    order = sorted(range(len(costs)), key=lambda i: (-costs[i], i))
    load = [0] * world
    parts: list[list[int]] = [[] for _ in range(world)]
    for i in order:
        r = min(range(world), key=lambda x: (load[x], x))
        parts[r].append(i)
        load[r] += costs[i]
    return [sorted(p) for p in parts]


def shard_varlen(lens_q, lens_k, causal: bool, world: int) -> list[list[int]]:
    """Per rank, the sequences of a varlen batch it computes."""
    return lpt_partition([sequence_cost(q, k, causal) for q, k in zip(lens_q, lens_k)], world)


def shard_rows(cu_seqlens, seqs):
    """Packed-row indices and cu_seqlens of the sub-batch made of sequences
    `seqs` (in that order) of a batch with prefix sums `cu_seqlens`.  Gather
    q (or k, v, out) rows with the indices; the shard's cu_seqlens starts at 0."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    rows = [np.arange(cu[b], cu[b + 1], dtype=np.int64) for b in seqs]
    idx = np.concatenate(rows) if rows else np.zeros(0, dtype=np.int64)
    lens = np.array([cu[b + 1] - cu[b] for b in seqs], dtype=np.int64)
    sub = np.zeros(len(seqs) + 1, dtype=np.int32)
    sub[1:] = np.cumsum(lens)
    return idx, sub
