"""Context-parallel ring attention across processes, one per GPU.

"Context Parallelism for Scalable Million-Token Inference", section 3. Every
rank holds its shard of Q and of K/V under the shard plan (load-balanced:
chunks i and 2N-1-i of every segment; or contiguous).

* Pass-KV: in N steps each rank attends its Q shard to the KV shard it holds
  while sending that shard to rank r+1 and receiving the next one from r-1
  into a second buffer, so the transfer of step t overlaps the attention of
  step t; at the end it merges its N partials.
* Pass-Q: the Q shards travel instead and the KV stays; each rank attends
  every Q shard that reaches it to its local KV, then an all-to-all returns
  the partials to the owners of the queries, which merge them.

* CP groups per KV head (section 5, key implementation details, item 1: one
  CP communication group per KV head): with the heads split across G groups
  of ranks (a KV head and the query heads that share it per group, as tensor
  parallelism splits them), each group runs its own ring over its heads'
  slices; kv_head_groups() forms the groups and head_slices() names each
  group's heads.

This module is plumbing: torch.distributed moves the shards (NCCL between
GPUs, point-to-point sends into a local buffer; no remote loads); the
attention and the merge are the library's kernels (cp_attn_partial,
cp_attn_merge). A caller may substitute functions with the same arguments
(the CPU tests do, to check the exchange logic on gloo ranks).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import binding as B


@dataclass
class Segment:
    """`length` tokens of one sequence at global rows row0.. and positions pos0.."""
    length: int
    row0: int
    pos0: int
    seq: int = 0


def kv_head_groups(n_groups: int):
    """Split the world into `n_groups` CP rings of world/n_groups consecutive
    ranks each: ring i serves KV-head group i. Every rank must call this (each
    group is created collectively, in the same order on all ranks). Returns
    (this rank's process group, its group index)."""
    world, rank = dist.get_world_size(), dist.get_rank()
    if n_groups < 1 or world % n_groups:
        raise ValueError(f"world size {world} is not a multiple of {n_groups} KV-head groups")
    cp = world // n_groups
    mine = None
    for i in range(n_groups):
        g = dist.new_group(list(range(i * cp, (i + 1) * cp)))
        if rank // cp == i:
            mine = g
    return mine, rank // cp


def head_slices(n_h: int, n_kv: int, n_groups: int, index: int):
    """Query-head and KV-head slices of KV-head group `index`: n_kv/n_groups
    consecutive KV heads and the n_h/n_kv query heads of each (GQA: query head
    h uses KV head floor(h / (n_h/n_kv)))."""
    if n_h % n_kv or n_kv % n_groups:
        raise ValueError("n_kv must be a multiple of the group count and n_h of n_kv")
    kv_per = n_kv // n_groups
    g = n_h // n_kv
    return slice(index * kv_per * g, (index + 1) * kv_per * g), slice(index * kv_per, (index + 1) * kv_per)


def _local(ranges, base: int = 0):
    """The same ranges with rows renumbered to a packed local buffer from `base`."""
    out, row = [], base
    for g in ranges:
        out.append(B.cp_range(row, g.pos0, g.len, g.seq, 0))
        row += g.len
    return out


def _rows(ranges) -> torch.Tensor:
    idx = [torch.arange(g.row0, g.row0 + g.len, dtype=torch.int64) for g in ranges if g.len > 0]
    return torch.cat(idx) if idx else torch.zeros(0, dtype=torch.int64)


class RingAttention:
    """One rank's side of a ring over `group` (default: the whole world)."""

    def __init__(self, q_segs, kv_segs, n_h: int, n_kv: int, d: int, variant: int = B.CP_PASS_KV,
                 mode: int = B.CP_SHARD_LOAD_BALANCED, group=None, partial_fn=None, merge_fn=None):
        if variant not in (B.CP_PASS_KV, B.CP_PASS_Q):
            raise ValueError("variant must be CP_PASS_KV or CP_PASS_Q")
        self.group = group
        self.rank = dist.get_rank(group)
        self.n = dist.get_world_size(group)
        self.n_h, self.n_kv, self.d = n_h, n_kv, d
        self.variant = variant
        qs = B.segments([(s.length, s.row0, s.pos0, s.seq) for s in q_segs])
        ks = B.segments([(s.length, s.row0, s.pos0, s.seq) for s in kv_segs])
        self.q_ranges = [B.cp_rank_ranges(qs, len(q_segs), self.n, mode, r) for r in range(self.n)]
        self.kv_ranges = [B.cp_rank_ranges(ks, len(kv_segs), self.n, mode, r) for r in range(self.n)]
        self.q_rows = [sum(g.len for g in rr) for rr in self.q_ranges]
        self.kv_rows = [sum(g.len for g in rr) for rr in self.kv_ranges]
        self.max_q = max(1, max(self.q_rows))
        self.max_kv = max(1, max(self.kv_rows))
        self.partial_fn = partial_fn or B.cp_attn_partial
        self.merge_fn = merge_fn or B.cp_attn_merge

    # ------------------------------------------------------------------ shards
    def q_shard_rows(self, rank: int | None = None) -> torch.Tensor:
        """Global rows of a rank's Q shard, in its local order."""
        return _rows(self.q_ranges[self.rank if rank is None else rank])

    def kv_shard_rows(self, rank: int | None = None) -> torch.Tensor:
        return _rows(self.kv_ranges[self.rank if rank is None else rank])

    # ----------------------------------------------------------------- forward
    def forward(self, q_local, k_local, v_local, softmax_scale: float | None = None, causal: bool = True,
                workspace=None):
        """q_local [q_rows, n_h, d], k_local/v_local [kv_rows, n_kv, d] (this rank's
        shards, rows as q_shard_rows / kv_shard_rows order them). Returns this
        rank's (out [q_rows, n_h, d] in q's dtype, lse [q_rows, n_h] fp32)."""
        if softmax_scale is None:
            softmax_scale = 1.0 / math.sqrt(self.d)
        if workspace is None:
            workspace = torch.zeros(256, dtype=torch.uint8, device=q_local.device)
        if self.variant == B.CP_PASS_KV:
            return self._pass_kv(q_local, k_local, v_local, softmax_scale, causal, workspace)
        return self._pass_q(q_local, k_local, v_local, softmax_scale, causal, workspace)

    def _exchange(self, send, recv):
        """Start sending `send` tensors to rank r+1 and receiving `recv` from r-1."""
        nxt = dist.get_global_rank(self.group, (self.rank + 1) % self.n) if self.group else (self.rank + 1) % self.n
        prv = dist.get_global_rank(self.group, (self.rank - 1) % self.n) if self.group else (self.rank - 1) % self.n
        ops = [dist.P2POp(dist.isend, t, nxt, self.group) for t in send]
        ops += [dist.P2POp(dist.irecv, t, prv, self.group) for t in recv]
        return dist.batch_isend_irecv(ops)

    def _block(self, q_ranges, kv_ranges, out_row0: int):
        ranges = (B.cp_range * max(1, len(q_ranges) + len(kv_ranges)))(*q_ranges, *kv_ranges)
        blocks = (B.cp_block * 1)(B.cp_block(0, len(q_ranges), len(q_ranges), len(kv_ranges), out_row0))
        return ranges, len(q_ranges) + len(kv_ranges), blocks

    def _pass_kv(self, q, k, v, scale, causal, ws):
        n, r = self.n, self.rank
        nq = self.q_rows[r]
        kb = [k.new_empty((self.max_kv, self.n_kv, self.d)) for _ in range(2)]
        vb = [v.new_empty((self.max_kv, self.n_kv, self.d)) for _ in range(2)]
        kb[0][:k.shape[0]].copy_(k)
        vb[0][:v.shape[0]].copy_(v)
        o_parts = torch.empty((n * max(1, nq), self.n_h, self.d), dtype=torch.float32, device=q.device)
        l_parts = torch.empty((n * max(1, nq), self.n_h), dtype=torch.float32, device=q.device)
        qr = _local(self.q_ranges[r])
        cur = 0
        for t in range(n):
            src = (r - t) % n
            reqs = self._exchange([kb[cur], vb[cur]], [kb[1 - cur], vb[1 - cur]]) if t < n - 1 else []
            if nq > 0:
                ranges, n_ranges, blocks = self._block(qr, _local(self.kv_ranges[src]), t * nq)
                self.partial_fn(q, kb[cur], vb[cur], self.n_h, self.n_kv, scale, causal, ranges, n_ranges, blocks,
                                1, o_parts, l_parts, ws)
            for w in reqs:
                w.wait()
            cur = 1 - cur
        out = torch.empty((nq, self.n_h, self.d), dtype=q.dtype, device=q.device)
        lse = torch.empty((nq, self.n_h), dtype=torch.float32, device=q.device)
        if nq > 0:
            self.merge_fn(o_parts, l_parts, n, nq, nq, self.n_h, self.d, out, lse)
        return out, lse

    def _pass_q(self, q, k, v, scale, causal, ws):
        n, r, mq = self.n, self.rank, self.max_q
        qb = [q.new_empty((mq, self.n_h, self.d)) for _ in range(2)]
        qb[0][:q.shape[0]].copy_(q)
        # slot o holds the partial of rank o's queries against this rank's KV
        o_send = torch.zeros((n * mq, self.n_h, self.d), dtype=torch.float32, device=q.device)
        l_send = torch.full((n * mq, self.n_h), float("-inf"), dtype=torch.float32, device=q.device)
        kvr = _local(self.kv_ranges[r])
        cur = 0
        for t in range(n):
            owner = (r - t) % n
            reqs = self._exchange([qb[cur]], [qb[1 - cur]]) if t < n - 1 else []
            if self.q_rows[owner] > 0 and self.kv_rows[r] > 0:
                ranges, n_ranges, blocks = self._block(_local(self.q_ranges[owner]), kvr, owner * mq)
                self.partial_fn(qb[cur], k, v, self.n_h, self.n_kv, scale, causal, ranges, n_ranges, blocks, 1,
                                o_send, l_send, ws)
            for w in reqs:
                w.wait()
            cur = 1 - cur
        # all-to-all: slot o goes to rank o; slot s of the result came from rank s
        o_recv = torch.empty_like(o_send)
        l_recv = torch.empty_like(l_send)
        dist.all_to_all_single(o_recv, o_send, group=self.group)
        dist.all_to_all_single(l_recv, l_send, group=self.group)
        nq = self.q_rows[r]
        out = torch.empty((nq, self.n_h, self.d), dtype=q.dtype, device=q.device)
        lse = torch.empty((nq, self.n_h), dtype=torch.float32, device=q.device)
        if nq > 0:
            self.merge_fn(o_recv, l_recv, n, mq, nq, self.n_h, self.d, out, lse)
        return out, lse
