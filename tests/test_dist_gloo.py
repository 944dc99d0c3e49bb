"""The multi-process ring (context_ring_attn_b200.dist) on gloo ranks on CPU.

Each rank runs the real exchange logic (ring sends of KV or Q shards into a
second buffer, the pass-Q all-to-all) with the library's attention and merge
replaced by the oracle on CPU tensors; every rank's output rows must equal the
unsharded attention of those rows. World sizes 2 and 4, both ring variants,
both shard modes, varlen segments and a persistent-KV prefill.
"""
import multiprocessing as mp
import os
import socket
import tempfile
import traceback
from datetime import timedelta

import numpy as np
import pytest

CASES = [
    # (name, world, variant, mode, KV-head groups)
    ("prefill", 2, "kv", "lb", 1),
    ("prefill", 4, "kv", "lb", 1),
    ("prefill", 4, "q", "lb", 1),
    ("prefill", 2, "q", "contig", 1),
    ("varlen", 4, "kv", "contig", 1),
    ("persistent", 4, "q", "lb", 1),
    ("persistent", 2, "kv", "lb", 1),
    # one CP ring per KV head: world 4 = 2 KV heads x a ring of 2
    ("prefill", 4, "kv", "lb", 2),
    ("prefill", 4, "q", "lb", 2),
    ("persistent", 4, "q", "lb", 2),
    ("varlen", 4, "kv", "lb", 2),
]


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _oracle_partial(q, k, v, n_h, n_kv, scale, causal, ranges, n_ranges, blocks, n_blocks, o_parts, lse_parts, ws):
    """Test stand-in for cp_attn_partial: block b writes rows out_row0 + q_row."""
    from oracle import attention as OA
    import torch
    for bi in range(n_blocks):
        b = blocks[bi]
        qr = [ranges[b.q_begin + j] for j in range(b.q_count)]
        kr = [ranges[b.kv_begin + j] for j in range(b.kv_count)]
        q_rows = np.concatenate([np.arange(g.row0, g.row0 + g.len) for g in qr]).astype(np.int64)
        q_pos = np.concatenate([np.arange(g.pos0, g.pos0 + g.len) for g in qr])
        q_seq = np.concatenate([np.full(g.len, g.seq) for g in qr])
        k_rows = np.concatenate([np.arange(g.row0, g.row0 + g.len) for g in kr] + [np.zeros(0)]).astype(np.int64)
        k_pos = np.concatenate([np.arange(g.pos0, g.pos0 + g.len) for g in kr] + [np.zeros(0)])
        k_seq = np.concatenate([np.full(g.len, g.seq) for g in kr] + [np.zeros(0)])
        o, lse = OA.attention(q.numpy()[q_rows], k.numpy()[k_rows], v.numpy()[k_rows], q_pos, k_pos, q_seq, k_seq,
                              scale, causal)
        o_parts[b.out_row0 + q_rows] = torch.from_numpy(o).to(o_parts.dtype)
        lse_parts[b.out_row0 + q_rows] = torch.from_numpy(lse).to(lse_parts.dtype)


def _oracle_merge(o_parts, lse_parts, n_parts, stride, rows, n_h, d, out, lse_out):
    from oracle import attention as OA
    import torch
    o, lse = OA.merge([o_parts.numpy()[j * stride:j * stride + rows] for j in range(n_parts)],
                      [lse_parts.numpy()[j * stride:j * stride + rows] for j in range(n_parts)])
    out.copy_(torch.from_numpy(o).to(out.dtype))
    lse_out.copy_(torch.from_numpy(lse).to(lse_out.dtype))


def _problem(name):
    """Global rows, positions and sequences of Q and KV, plus the segments."""
    from context_ring_attn_b200.dist import Segment
    if name == "prefill":
        t = 96
        q_segs = kv_segs = [Segment(t, 0, 0, 0)]
        q_pos = k_pos = np.arange(t)
        q_seq = k_seq = np.zeros(t, dtype=np.int64)
        tq, tk = t, t
    elif name == "varlen":
        lens = [40, 56]
        q_segs = kv_segs = [Segment(40, 0, 0, 0), Segment(56, 40, 0, 1)]
        q_pos = k_pos = np.concatenate([np.arange(40), np.arange(56)])
        q_seq = k_seq = np.concatenate([np.zeros(40), np.ones(56)]).astype(np.int64)
        tq = tk = sum(lens)
    else:   # persistent KV: 24 new tokens over a cache of 72
        t, p = 24, 72
        q_segs = [Segment(t, 0, p, 0)]
        kv_segs = [Segment(p, 0, 0, 0), Segment(t, p, p, 0)]
        q_pos = np.arange(p, p + t)
        k_pos = np.arange(p + t)
        q_seq = np.zeros(t, dtype=np.int64)
        k_seq = np.zeros(p + t, dtype=np.int64)
        tq, tk = t, p + t
    return q_segs, kv_segs, q_pos, k_pos, q_seq, k_seq, tq, tk


def _worker(rank, world, port, name, variant, mode, groups, out_dir):
    try:
        import torch
        import torch.distributed as dist
        from context_ring_attn_b200 import binding as B
        from context_ring_attn_b200.dist import RingAttention, head_slices, kv_head_groups
        from oracle import attention as OA

        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                                timeout=timedelta(seconds=60))
        n_h, n_kv, d = 4, 2, 16
        q_segs, kv_segs, q_pos, k_pos, q_seq, k_seq, tq, tk = _problem(name)
        rng = np.random.default_rng(7)
        q = rng.standard_normal((tq, n_h, d))
        k = rng.standard_normal((tk, n_kv, d))
        v = rng.standard_normal((tk, n_kv, d))
        scale = 1.0 / np.sqrt(d)
        group, gi = (None, 0) if groups == 1 else kv_head_groups(groups)
        hq, hk = head_slices(n_h, n_kv, groups, gi)
        q, k, v = q[:, hq], k[:, hk], v[:, hk]   # this ring's heads
        ra = RingAttention(q_segs, kv_segs, n_h // groups, n_kv // groups, d,
                           B.CP_PASS_KV if variant == "kv" else B.CP_PASS_Q,
                           B.CP_SHARD_LOAD_BALANCED if mode == "lb" else B.CP_SHARD_CONTIGUOUS, group=group,
                           partial_fn=_oracle_partial, merge_fn=_oracle_merge)
        assert ra.n == world // groups
        qi, ki = ra.q_shard_rows().numpy(), ra.kv_shard_rows().numpy()
        out, lse = ra.forward(torch.from_numpy(q[qi]), torch.from_numpy(k[ki]), torch.from_numpy(v[ki]), scale)
        # the unsharded attention of these rows, restricted to this ring's heads
        o_ref, l_ref = OA.attention(q[qi], k, v, q_pos[qi], k_pos, q_seq[qi], k_seq, scale)
        err = float(np.abs(out.numpy() - o_ref).max(initial=0.0))
        fin = np.isfinite(l_ref)
        lerr = float(np.abs(lse.numpy()[fin] - l_ref[fin]).max(initial=0.0))
        same_inf = bool(np.array_equal(np.isfinite(lse.numpy()), fin))
        # every row of Q is owned by exactly one rank
        owned = torch.zeros(tq, dtype=torch.int64)
        owned[torch.from_numpy(qi)] += 1
        dist.all_reduce(owned, group=group)
        dist.destroy_process_group()
        with open(os.path.join(out_dir, f"r{rank}"), "w") as f:
            f.write(f"{err} {lerr} {int(same_inf)} {int(bool((owned == 1).all()))}\n")
    except Exception:
        with open(os.path.join(out_dir, f"r{rank}"), "w") as f:
            f.write("EXC " + traceback.format_exc().replace("\n", " | "))


@pytest.mark.parametrize("name,world,variant,mode,groups", CASES)
def test_ring_over_gloo_matches_unsharded_attention(name, world, variant, mode, groups):
    ctx = mp.get_context("spawn")
    port = _free_port()
    with tempfile.TemporaryDirectory() as tmp:
        procs = [ctx.Process(target=_worker, args=(r, world, port, name, variant, mode, groups, tmp)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=180)
        for p in procs:
            if p.is_alive():
                p.kill()
                p.join()
        for r in range(world):
            path = os.path.join(tmp, f"r{r}")
            assert os.path.exists(path), f"rank {r} wrote no result"
            text = open(path).read()
            assert not text.startswith("EXC"), text
            err, lerr, same_inf, owned = text.split()
            # the partials are fp32 buffers, as the kernels write them: fp32 rounding
            assert float(err) < 2e-6 and float(lerr) < 2e-6, (r, err, lerr)
            assert same_inf == "1" and owned == "1"
