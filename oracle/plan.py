"""Independent shard planner and ring schedules (test infrastructure).

Written from "Context Parallelism for Scalable Million-Token Inference"
(section 3 ring pass-KV / pass-Q; section 4 load-balanced sharding). The
figure for the load-balanced layout did not survive on the page; the reading
used is the standard one for causal ring attention: a sequence of length L is
cut into 2N chunks, chunk c = [floor(c*L/2N), floor((c+1)*L/2N)), and rank i
holds chunks i and 2N-1-i, so each rank holds one early and one late chunk and
the causal work per rank is equal. The contiguous layout (rank i holds
[floor(i*L/N), floor((i+1)*L/N)), i.e. chunks 2i and 2i+1) is the unbalanced
layout the pages contrast it with.

Ring direction: rank r sends to r+1, so at step t rank r holds the shard of
rank (r - t) mod N; step 0 is the local shard (N compute steps, N-1 hops).
  * pass-KV: rank i keeps its Q shard; at step t it computes against the KV
    shard of rank (i - t) mod N; that partial is arrival number t.
  * pass-Q: rank i keeps its KV shard; at step t it computes the Q shard of
    rank (i - t) mod N; after the all-to-all the Q owner holds one partial per
    KV owner, indexed by the KV owner.
"""
from __future__ import annotations

from dataclasses import dataclass

LOAD_BALANCED = 0
CONTIGUOUS = 1

PASS_KV = 0
PASS_Q = 1

FULL = 0
PARTIAL = 1
SKIP = 2


@dataclass(frozen=True)
class Segment:
    length: int
    row0: int      # first row of the segment in its buffer
    pos0: int      # global causal position of that first row
    seq: int       # sequence id


@dataclass(frozen=True)
class Range:
    row0: int
    pos0: int
    length: int
    seq: int


@dataclass(frozen=True)
class Block:
    q_begin: int
    q_count: int
    kv_begin: int
    kv_count: int
    out_row0: int


def chunk_bounds(length: int, n_ranks: int) -> list[int]:
    n_chunks = 2 * n_ranks
    return [(c * length) // n_chunks for c in range(n_chunks + 1)]


def rank_chunks(rank: int, n_ranks: int, mode: int) -> tuple[int, int]:
    if mode == LOAD_BALANCED:
        return (rank, 2 * n_ranks - 1 - rank)
    if mode == CONTIGUOUS:
        return (2 * rank, 2 * rank + 1)
    raise ValueError(mode)


def rank_ranges(segs, n_ranks: int, mode: int, rank: int) -> list[Range]:
    """Ranges a rank holds: per segment in order, its chunks in ascending
    chunk order; empty chunks are left out."""
    out = []
    for s in segs:
        b = chunk_bounds(s.length, n_ranks)
        for c in sorted(rank_chunks(rank, n_ranks, mode)):
            n = b[c + 1] - b[c]
            if n > 0:
                out.append(Range(s.row0 + b[c], s.pos0 + b[c], n, s.seq))
    return out


def shard_plan(segs, n_ranks: int, mode: int):
    """(chunk bounds per segment, rank row offsets [N+1], buffer rows in rank order)."""
    bounds = [chunk_bounds(s.length, n_ranks) for s in segs]
    rank_rows = [0]
    token_index = []
    for r in range(n_ranks):
        for rg in rank_ranges(segs, n_ranks, mode, r):
            token_index.extend(range(rg.row0, rg.row0 + rg.length))
        rank_rows.append(len(token_index))
    return bounds, rank_rows, token_index


def ring_schedule(q_segs, kv_segs, n_ranks: int, mode: int, variant: int):
    """Ranges (all Q shards then all KV shards), blocks [N*N] by step, and the
    partial index of each block."""
    q_sh = [rank_ranges(q_segs, n_ranks, mode, r) for r in range(n_ranks)]
    kv_sh = [rank_ranges(kv_segs, n_ranks, mode, r) for r in range(n_ranks)]
    ranges, q_off, kv_off = [], [], []
    for r in range(n_ranks):
        q_off.append(len(ranges))
        ranges.extend(q_sh[r])
    q_off.append(len(ranges))
    for r in range(n_ranks):
        kv_off.append(len(ranges))
        ranges.extend(kv_sh[r])
    kv_off.append(len(ranges))
    blocks, parts = [], []
    for t in range(n_ranks):
        for i in range(n_ranks):
            if variant == PASS_KV:
                qr, kr, part = i, (i - t) % n_ranks, t
            elif variant == PASS_Q:
                kr, qr, part = i, (i - t) % n_ranks, i
            else:
                raise ValueError(variant)
            blocks.append(Block(q_off[qr], q_off[qr + 1] - q_off[qr],
                                kv_off[kr], kv_off[kr + 1] - kv_off[kr], 0))
            parts.append(part)
    return ranges, blocks, parts


def pair_class(qr: Range, kr: Range, causal: bool = True) -> int:
    """FULL: every query row sees every key; PARTIAL: mask needed; SKIP: none."""
    if qr.seq != kr.seq or qr.length == 0 or kr.length == 0:
        return SKIP
    if not causal:
        return FULL
    q_lo, q_hi = qr.pos0, qr.pos0 + qr.length - 1
    k_lo, k_hi = kr.pos0, kr.pos0 + kr.length - 1
    if k_lo > q_hi:
        return SKIP
    if k_hi <= q_lo:
        return FULL
    return PARTIAL


def visible_pairs(qr: Range, kr: Range, causal: bool = True) -> int:
    """Number of (query, key) pairs of the two ranges the mask keeps, by counting."""
    if qr.seq != kr.seq:
        return 0
    if not causal:
        return qr.length * kr.length
    total = 0
    for p in range(qr.pos0, qr.pos0 + qr.length):
        total += max(0, min(kr.pos0 + kr.length, p + 1) - kr.pos0)
    return total


def block_pairs(ranges, block: Block, causal: bool = True) -> int:
    total = 0
    for a in range(block.q_begin, block.q_begin + block.q_count):
        for b in range(block.kv_begin, block.kv_begin + block.kv_count):
            total += visible_pairs(ranges[a], ranges[b], causal)
    return total
