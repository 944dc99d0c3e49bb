"""Ring schedules over the C ABI: N virtual context-parallel ranks on one GPU.

"Context Parallelism for Scalable Million-Token Inference", section 3: in
pass-KV every rank keeps its query shard while the KV shards travel around
the ring; in pass-Q the KV shards stay and the query shards travel, and an
all-to-all returns the partials to their owners, which merge them. On one
GPU every shard already sits in the same buffers, so a ring step is one
cp_attn_partial launch covering the N blocks of that step, and the exchange
moves no bytes. The merge is cp_attn_merge.

This module only sequences C-ABI calls; all arithmetic runs in the kernels.
"""
from __future__ import annotations

import ctypes
import math
from dataclasses import dataclass

import torch

from . import binding as B


@dataclass
class Segment:
    """`length` rows of a buffer from `row0`, tokens of sequence `seq` at
    positions pos0.. (a persistent-KV prefill has a cached segment and a new
    one in the same sequence)."""
    length: int
    row0: int
    pos0: int
    seq: int = 0


class RingSchedule:
    def __init__(self, q_segs, kv_segs, n_ranks: int, variant: int = B.CP_PASS_KV,
                 mode: int = B.CP_SHARD_LOAD_BALANCED):
        self.n_ranks = n_ranks
        self.variant = variant
        self.mode = mode
        self.q_segs = B.segments([(s.length, s.row0, s.pos0, s.seq) for s in q_segs])
        self.kv_segs = B.segments([(s.length, s.row0, s.pos0, s.seq) for s in kv_segs])
        self.ranges, self.n_ranges, self.blocks, self.parts = B.cp_ring_schedule(
            self.q_segs, len(q_segs), self.kv_segs, len(kv_segs), n_ranks, mode, variant)

    def step_blocks(self, t: int, part_rows: int, part_of=None) -> ctypes.Array:
        """The N blocks of ring step t, writing partial `part_of(part)` at row
        offset part * part_rows of one stacked partial buffer."""
        n = self.n_ranks
        arr = (B.cp_block * n)()
        for i in range(n):
            src = self.blocks[t * n + i]
            part = self.parts[t * n + i] if part_of is None else part_of(self.parts[t * n + i])
            arr[i] = B.cp_block(src.q_begin, src.q_count, src.kv_begin, src.kv_count, part * part_rows)
        return arr

    def pairs(self, causal: bool = True) -> int:
        """Visible (query, key) pairs per query head over the whole schedule."""
        return sum(B.cp_block_pairs(self.ranges, self.blocks[i], causal) for i in range(self.n_ranks ** 2))


def _nvtx(name: str):
    """An NVTX range (visible in an Nsight Systems timeline) around one host
    step of a schedule: each ring step's launch and each merge."""
    return torch.cuda.nvtx.range(name)


def partial_buffers(q_rows: int, n_h: int, d: int, n_parts: int, device="cuda", dtype=torch.float32):
    o = torch.empty((n_parts * q_rows, n_h, d), dtype=dtype, device=device)
    lse = torch.empty((n_parts * q_rows, n_h), dtype=torch.float32, device=device)
    return o, lse


def run_ring(sched: RingSchedule, q, k, v, n_h: int, n_kv: int, out, lse_out=None, causal: bool = True,
             scale: float | None = None, o_parts=None, lse_parts=None, workspace=None,
             merge: str = "final", stream=None):
    """Attention of q against k/v through the ring schedule, into `out`.

    merge="final": N partial buffers, one N-way merge at the end.
    merge="running": two partial buffers; after every step the step's partial
    is merged into the running one (less memory, N-1 extra merge passes).
    merge="fused": one buffer; every step's kernel merges its rows into the
    running (O, LSE) in its epilogue and the last step writes `out` directly
    (cp_attn_partial_fused; no merge pass). lse_out, if given, is the running
    LSE buffer.
    merge="final_bf16": as "final" with bf16 partial O buffers
    (cp_attn_partial_bf16_parts, then cp_attn_merge_bf16_parts): half the
    partial bytes written and read.
    """
    q_rows, d = int(q.shape[0]), int(q.shape[-1])
    n = sched.n_ranks
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    n_bufs = n if merge in ("final", "final_bf16") else (1 if merge == "fused" else 2)
    if o_parts is None:
        o_parts, lse_parts = partial_buffers(q_rows, n_h, d, n_bufs, q.device,
                                             torch.bfloat16 if merge == "final_bf16" else torch.float32)
    if workspace is None:
        workspace = torch.zeros(B.cp_workspace_size(B.CP_OP_PARTIAL, 0, n_h, d, 1), dtype=torch.uint8,
                                device=q.device)
    if merge not in ("fused", "final", "running", "final_bf16"):
        raise ValueError(merge)
    if merge == "final_bf16":
        for t in range(n):
            blocks = sched.step_blocks(t, q_rows)
            with _nvtx(f"ring step {t} (bf16 partials)"):
                B.cp_attn_partial_bf16_parts(q, k, v, n_h, n_kv, scale, causal, sched.ranges, sched.n_ranges, blocks,
                                             n, o_parts, lse_parts, workspace, stream)
        with _nvtx(f"merge {n}-way (bf16 partials)"):
            B.cp_attn_merge(o_parts, lse_parts, n, q_rows, q_rows, n_h, d, out, lse_out, stream)
        return out
    if merge == "fused":
        lse_acc = lse_out if lse_out is not None else lse_parts
        for t in range(n):
            blocks = sched.step_blocks(t, q_rows, part_of=lambda _p: 0)
            with _nvtx(f"ring step {t} (fused merge)"):
                B.cp_attn_partial_fused(q, k, v, n_h, n_kv, scale, causal, sched.ranges, sched.n_ranges, blocks, n,
                                        o_parts, lse_acc, t > 0, out if t == n - 1 else None, workspace, stream)
        return out
    if merge == "final":
        for t in range(n):
            blocks = sched.step_blocks(t, q_rows)
            with _nvtx(f"ring step {t}"):
                B.cp_attn_partial(q, k, v, n_h, n_kv, scale, causal, sched.ranges, sched.n_ranges, blocks, n,
                                  o_parts, lse_parts, workspace, stream)
        with _nvtx(f"merge {n}-way"):
            B.cp_attn_merge(o_parts, lse_parts, n, q_rows, q_rows, n_h, d, out, lse_out, stream)
    else:
        for t in range(n):
            target = 0 if t == 0 else 1
            blocks = sched.step_blocks(t, q_rows, part_of=lambda _p, _t=target: _t)
            with _nvtx(f"ring step {t}"):
                B.cp_attn_partial(q, k, v, n_h, n_kv, scale, causal, sched.ranges, sched.n_ranges, blocks, n,
                                  o_parts, lse_parts, workspace, stream)
            if t == 0 and n > 1:
                continue
            with _nvtx("merge running"):
                if t == n - 1:
                    B.cp_attn_merge(o_parts, lse_parts, 2 if n > 1 else 1, q_rows, q_rows, n_h, d, out, lse_out,
                                    stream)
                else:
                    B.cp_attn_merge(o_parts, lse_parts, 2, q_rows, q_rows, n_h, d, o_parts, lse_parts, stream)
    return out


class DecodeCP:
    """Context-parallel decode over N virtual ranks.

    "Context Parallelism for Scalable Million-Token Inference", section 3:
    in decode each CP rank holds a shard of every request's KV cache (the
    shards the prefill's plan gave it) and the queries travel the ring
    (pass-Q); after N steps every rank has decoded every query against its own
    shard, an all-to-all returns the partials (O, LSE) to the queries' owners
    and they are merged. On one GPU the N^2 (rank, query shard) visits of the
    ring are one batched cp_decode_partial launch over "virtual requests"
    (rank r, request b) in rank-major order, so the partial of rank r for
    request b lands at row r*B + b: the all-to-all is that index, and
    cp_attn_merge over the N parts finishes the decode. The shards are
    gathered once at construction (each rank's own cache in a real
    deployment); the arithmetic runs in the library's kernels.
    """

    def __init__(self, k, v, offsets_host, n_ranks: int, mode: int = B.CP_SHARD_LOAD_BALANCED):
        offsets_host = [int(x) for x in offsets_host]
        n_req = len(offsets_host) - 1
        self.n_ranks, self.n_req = n_ranks, n_req
        segs = B.segments([(offsets_host[b + 1] - offsets_host[b], offsets_host[b], 0, b) for b in range(n_req)])
        idx, offs = [], [0]
        for r in range(n_ranks):
            per_req = [[] for _ in range(n_req)]
            for g in B.cp_rank_ranges(segs, n_req, n_ranks, mode, r):
                per_req[g.seq].append(g)
            for b in range(n_req):
                n = 0
                for g in per_req[b]:
                    if g.len > 0:
                        idx.append(torch.arange(g.row0, g.row0 + g.len, dtype=torch.int64))
                        n += g.len
                offs.append(offs[-1] + n)
        rows = torch.cat(idx) if idx else torch.zeros(0, dtype=torch.int64)
        if rows.numel() == 0:   # no keys anywhere: one unused row keeps the buffers non-empty
            rows = torch.zeros(1, dtype=torch.int64)
        rows = rows.to(k.device)
        self.k = k.index_select(0, rows)
        self.v = v.index_select(0, rows)
        self.offsets = torch.tensor(offs, dtype=torch.int64, device=k.device)
        self.kv_bytes = 2 * (offs[-1] * int(k.shape[1]) * int(k.shape[2]) * k.element_size())

    def buffers(self, q, n_splits: int):
        """Partial buffers, the per-rank query copies and a decode workspace."""
        n, n_req = self.n_ranks, self.n_req
        n_h, d = int(q.shape[1]), int(q.shape[2])
        o_parts = torch.empty((n * n_req, n_h, d), dtype=torch.float32, device=q.device)
        lse_parts = torch.empty((n * n_req, n_h), dtype=torch.float32, device=q.device)
        ws = torch.zeros(B.cp_workspace_size(B.CP_OP_DECODE, n * n_req, n_h, d, n_splits), dtype=torch.uint8,
                         device=q.device)
        return o_parts, lse_parts, ws

    def run(self, q_ranks, n_kv: int, n_splits: int, softmax_scale: float, out, lse_out, o_parts, lse_parts,
            workspace, stream=None):
        """q_ranks: the queries as every rank holds them, [N*B, n_h, d] (q repeated
        N times, rank-major). out [B, n_h, d] bf16, lse_out [B, n_h] fp32."""
        n_h, d = int(q_ranks.shape[1]), int(q_ranks.shape[2])
        with _nvtx("cp decode: rank partials"):
            B.cp_decode_partial(q_ranks, self.k, self.v, self.offsets, n_h, n_kv, n_splits, softmax_scale,
                                o_parts, lse_parts, workspace, stream)
        with _nvtx("cp decode: merge"):
            B.cp_attn_merge(o_parts, lse_parts, self.n_ranks, self.n_req, self.n_req, n_h, d, out, lse_out, stream)
