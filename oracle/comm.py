"""Communication volume of the ring schedules (test infrastructure).

On one GPU the virtual ring moves no bytes; these counts say what a real ring
of N GPUs would move, so they can be checked against the closed forms of
"Context Parallelism for Scalable Million-Token Inference":
  * section 3, parallelism comparison table: per transformer block TP moves
    2*(T*N_H*D_H) elements, CP moves T*N_KV*D_H;
  * section 3, ring communication model: pass-KV moves (N-1)*T*N_KV*D_H in
    total, overlapped with attention;
  * section 3 / Algorithm 1: pass-KV is chosen when the KV-cache miss rate
    T/(T+P) exceeds 2*N_KV/N_H (12.5% for 128 query heads and 8 KV heads).

Reading of the factor 2: the table's CP entry counts one tensor (K or V) and
its TP entry counts two all-reduces; the page's "16x smaller" for 128/8 heads
only holds when both sides count two tensors (K and V against two
all-reduces), so counts here are per tensor unless named otherwise.
"""
from __future__ import annotations

from .plan import PASS_KV, PASS_Q


def tp_block_elems(t: int, n_h: int, d: int) -> int:
    """Elements all-reduced per transformer block under tensor parallelism."""
    return 2 * t * n_h * d


def cp_block_elems(t: int, n_kv: int, d: int) -> int:
    """Elements of one KV tensor (K or V) for T tokens: the CP message size."""
    return t * n_kv * d


def cp_over_tp_ratio(n_h: int, n_kv: int) -> float:
    """TP volume over CP volume with both counting two tensors (K and V)."""
    return tp_block_elems(1, n_h, 1) / (2 * cp_block_elems(1, n_kv, 1))


def miss_rate_threshold(n_h: int, n_kv: int) -> float:
    return 2.0 * n_kv / n_h


def select_variant(t: int, p: int, n_h: int, n_kv: int) -> int:
    """Algorithm 1, condition 1 (the volume crossover): pass-KV when the miss
    rate T/(T+P) is above 2*N_KV/N_H, else pass-Q. Condition 2 (pass-KV when
    its SendRecv hides under compute) needs timing and is not modelled."""
    return PASS_KV if t / (t + p) > miss_rate_threshold(n_h, n_kv) else PASS_Q


def kv_hop_seconds(t: int, p: int, n_kv: int, d: int, n_ranks: int, elem_bytes: int,
                   link_bytes_per_s: float) -> float:
    """Time of one pass-KV ring hop: one rank's KV shard, (T+P)/N tokens of K
    and of V, over a link of the given bandwidth."""
    return (t + p) / n_ranks * n_kv * d * 2 * elem_bytes / link_bytes_per_s


def select_variant_alg1(t: int, p: int, n_h: int, n_kv: int, d: int, n_ranks: int, elem_bytes: int,
                        link_bytes_per_s: float, step_attn_s: float):
    """Algorithm 1 of the method page (section 3), both conditions, in order:
    1. pass-KV if the miss rate T/(T+P) is above 2*N_KV/N_H;
    2. pass-KV if one ring hop's SendRecv of a KV shard takes no longer than
       one ring step of attention (step_attn_s), i.e. it hides under compute;
    otherwise pass-Q. Returns (variant, condition that chose pass-KV or 0)."""
    if t / (t + p) > miss_rate_threshold(n_h, n_kv):
        return PASS_KV, 1
    if kv_hop_seconds(t, p, n_kv, d, n_ranks, elem_bytes, link_bytes_per_s) <= step_attn_s:
        return PASS_KV, 2
    return PASS_Q, 0


def schedule_volume(ranges, blocks, n_ranks: int, variant: int, n_h: int, n_kv: int, d: int):
    """Per hop and per rank, the elements a rank receives (per tensor for
    pass-KV; the Q tensor for pass-Q), plus pass-Q's all-to-all of (O, LSE).

    blocks are the ring schedule [N*N] ordered by step (blocks[t*N + i] runs on
    rank i at step t). Step 0 uses local data and moves nothing.
    """
    def rows(begin, count):
        return sum(ranges[j].length for j in range(begin, begin + count))

    hops = []
    for t in range(1, n_ranks):
        per_rank = []
        for i in range(n_ranks):
            b = blocks[t * n_ranks + i]
            if variant == PASS_KV:
                per_rank.append(rows(b.kv_begin, b.kv_count) * n_kv * d)
            else:
                per_rank.append(rows(b.q_begin, b.q_count) * n_h * d)
        hops.append(per_rank)
    a2a = 0
    if variant == PASS_Q:
        for t in range(1, n_ranks):
            for i in range(n_ranks):
                b = blocks[t * n_ranks + i]
                a2a += rows(b.q_begin, b.q_count) * n_h * (d + 1)
    total = sum(sum(h) for h in hops)
    return {"hops": hops, "total": total, "all_to_all": a2a}
