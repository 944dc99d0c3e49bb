"""The C planner against the independent reference planner, bit for bit."""
import itertools

import numpy as np
import pytest

from context_ring_attn_b200 import binding as B
from context_ring_attn_b200 import build as BUILD
from context_ring_attn_b200 import synth
from oracle import comm as OC
from oracle import plan as OP


@pytest.fixture(scope="module", autouse=True)
def _lib():
    BUILD.build()
    B.lib()


def _segs(lens, pos0=None, seqs=None, row_base=0):
    out, row = [], row_base
    for i, ln in enumerate(lens):
        out.append(OP.Segment(ln, row, 0 if pos0 is None else pos0[i], i if seqs is None else seqs[i]))
        row += ln
    return out


def _c_segs(segs):
    return B.segments([(s.length, s.row0, s.pos0, s.seq) for s in segs])


def _ranges_equal(c_list, o_list):
    assert len(c_list) == len(o_list)
    for c, o in zip(c_list, o_list):
        assert (c.row0, c.pos0, c.len, c.seq) == (o.row0, o.pos0, o.length, o.seq)


CASES = [
    ([256], 4), ([131072], 8), ([7], 4), ([1], 3), ([100, 37, 2], 3), ([5, 0, 9], 2),
    (synth.varlen_lengths(1005), 8), ([126976], 8), ([4096], 8), ([1000], 1),
]


@pytest.mark.parametrize("lens,n", CASES)
@pytest.mark.parametrize("mode", [OP.LOAD_BALANCED, OP.CONTIGUOUS])
def test_shard_plan_bit_exact(lens, n, mode):
    segs = _segs(lens)
    cb, rr, ti = B.cp_shard_plan(_c_segs(segs), len(segs), n, mode)
    ob, orr, oti = OP.shard_plan(segs, n, mode)
    # the sizes query (NULL arrays) gives the reference plan's array lengths
    assert B.cp_shard_plan_sizes(_c_segs(segs), len(segs), n, mode) == (sum(len(b) for b in ob), len(orr), len(oti))
    assert np.array_equal(cb, np.array(ob, dtype=np.int64).reshape(len(segs), 2 * n + 1))
    assert list(rr) == orr
    if len(oti) < 2_000_000:
        assert np.array_equal(ti, np.array(oti, dtype=np.int64))
    for r in range(n):
        _ranges_equal(B.cp_rank_ranges(_c_segs(segs), len(segs), n, mode, r), OP.rank_ranges(segs, n, mode, r))


def _schedule_case(kind):
    if kind == "tiny":
        s = _segs([256])
        return s, s, 4
    if kind == "prefill_128k":
        s = _segs([131072])
        return s, s, 8
    if kind == "persistent_kv":
        p, t = 126976, 4096
        return [OP.Segment(t, 0, p, 0)], [OP.Segment(p, 0, 0, 0), OP.Segment(t, p, p, 0)], 8
    if kind == "varlen":
        s = _segs(synth.varlen_lengths(1005))
        return s, s, 8
    if kind == "ragged":
        s = _segs([37, 5, 64], seqs=[0, 1, 2])
        return s, s, 3


@pytest.mark.parametrize("kind", ["tiny", "prefill_128k", "persistent_kv", "varlen", "ragged"])
@pytest.mark.parametrize("mode", [OP.LOAD_BALANCED, OP.CONTIGUOUS])
@pytest.mark.parametrize("variant", [OP.PASS_KV, OP.PASS_Q])
def test_ring_schedule_bit_exact(kind, mode, variant):
    q_segs, kv_segs, n = _schedule_case(kind)
    ranges, n_ranges, blocks, parts = B.cp_ring_schedule(_c_segs(q_segs), len(q_segs), _c_segs(kv_segs),
                                                         len(kv_segs), n, mode, variant)
    o_ranges, o_blocks, o_parts = OP.ring_schedule(q_segs, kv_segs, n, mode, variant)
    _ranges_equal([ranges[i] for i in range(n_ranges)], o_ranges)
    assert parts == o_parts
    for i, ob in enumerate(o_blocks):
        cb = blocks[i]
        assert (cb.q_begin, cb.q_count, cb.kv_begin, cb.kv_count, cb.out_row0) == \
            (ob.q_begin, ob.q_count, ob.kv_begin, ob.kv_count, ob.out_row0)
    # mask classes of every chunk pair, and the pair counts per block
    for ob in o_blocks:
        for a in range(ob.q_begin, ob.q_begin + ob.q_count):
            for b in range(ob.kv_begin, ob.kv_begin + ob.kv_count):
                assert B.cp_classify_pair(ranges[a], ranges[b], True) == OP.pair_class(o_ranges[a], o_ranges[b], True)
                assert B.cp_classify_pair(ranges[a], ranges[b], False) == OP.pair_class(o_ranges[a], o_ranges[b], False)
    if kind in ("tiny", "ragged"):
        for i, ob in enumerate(o_blocks):
            assert B.cp_block_pairs(ranges, blocks[i], True) == OP.block_pairs(o_ranges, ob, True)
            assert B.cp_block_pairs(ranges, blocks[i], False) == OP.block_pairs(o_ranges, ob, False)
    hops, total, a2a = B.cp_ring_comm_volume(ranges, blocks, n, variant, 128, 8, 128)
    ref = OC.schedule_volume(o_ranges, o_blocks, n, variant, 128, 8, 128)
    assert hops.tolist() == ref["hops"] and total == ref["total"] and a2a == ref["all_to_all"]


def test_pair_counts_closed_form_prefill_128k():
    """All blocks of the 128K schedule: C^2 + C(C+1) on the diagonal, 2C^2 elsewhere."""
    n, c = 8, 8192
    segs = _c_segs(_segs([2 * n * c]))
    ranges, _, blocks, _ = B.cp_ring_schedule(segs, 1, segs, 1, n, B.CP_SHARD_LOAD_BALANCED, B.CP_PASS_KV)
    total = 0
    for t, i in itertools.product(range(n), range(n)):
        want = c * c + c * (c + 1) if t == 0 else 2 * c * c
        got = B.cp_block_pairs(ranges, blocks[t * n + i], True)
        assert got == want
        total += got
    assert total == (2 * n * c) * (2 * n * c + 1) // 2


def test_random_pairs_against_reference():
    rng = np.random.default_rng(0)
    for _ in range(500):
        q = B.cp_range(0, int(rng.integers(0, 50)), int(rng.integers(0, 30)), int(rng.integers(0, 2)), 0)
        k = B.cp_range(0, int(rng.integers(0, 50)), int(rng.integers(0, 30)), int(rng.integers(0, 2)), 0)
        oq = OP.Range(0, q.pos0, q.len, q.seq)
        ok = OP.Range(0, k.pos0, k.len, k.seq)
        ranges = (B.cp_range * 2)(q, k)
        blk = B.cp_block(0, 1, 1, 1, 0)
        for causal in (True, False):
            assert B.cp_classify_pair(q, k, causal) == OP.pair_class(oq, ok, causal)
            assert B.cp_block_pairs(ranges, blk, causal) == OP.visible_pairs(oq, ok, causal)


@pytest.mark.parametrize("n_ranks,mode", [(2, B.CP_SHARD_LOAD_BALANCED), (8, B.CP_SHARD_LOAD_BALANCED),
                                          (3, B.CP_SHARD_CONTIGUOUS)])
def test_decode_shards_partition_every_request(n_ranks, mode):
    """The per-rank decode shards hold every key of every request exactly once,
    in request order within each rank, with CSR offsets per (rank, request)."""
    import torch
    from context_ring_attn_b200 import ring
    lens = [0, 5, 100, 31, 256, 1000]
    offsets = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    total = int(offsets[-1])
    k = torch.arange(total, dtype=torch.float32).reshape(total, 1, 1)   # row id as the value
    cp = ring.DecodeCP(k, k, offsets, n_ranks, mode)
    offs = cp.offsets.numpy()
    assert offs.shape == (n_ranks * len(lens) + 1,) and offs[0] == 0
    assert np.all(np.diff(offs) >= 0)
    seen = np.zeros(total, dtype=np.int64)
    for r in range(n_ranks):
        for b in range(len(lens)):
            i = r * len(lens) + b
            rows = cp.k[offs[i]:offs[i + 1], 0, 0].numpy().astype(np.int64)
            assert np.all((rows >= offsets[b]) & (rows < offsets[b + 1]))
            seen[rows] += 1
    assert np.all(seen == 1)


def test_select_ring_variant_matches_oracle():
    """The library's Algorithm 1 equals the oracle's on a grid of miss rates,
    head counts, rank counts, link speeds and step times."""
    total = 128000
    for n_h, n_kv in ((128, 8), (16, 1), (32, 8)):
        for n in (2, 8):
            for link in (12.5e9, 50e9, 770e9):
                for step in (0.0, 1e-4, 1e-3, 1e-2):
                    for t in (1, 1280, 6400, 16000, 16001, 40000, 127999):
                        want = OC.select_variant_alg1(t, total - t, n_h, n_kv, 128, n, 2, link, step)
                        got = B.cp_select_ring_variant(t, total - t, n_h, n_kv, 128, n, 2, link, step)
                        assert got == want, (n_h, n_kv, n, link, step, t)
    with pytest.raises(B.CpError):
        B.cp_select_ring_variant(0, 0, 128, 8, 128, 8, 2, 50e9, 0.0)
    with pytest.raises(B.CpError):
        B.cp_select_ring_variant(10, 10, 128, 8, 128, 8, 2, 0.0, 0.0)


@pytest.mark.parametrize("k", [1000, 1024])
def test_library_contiguous_layout_matches_page(golden, k):
    """cp_rank_ranges in contiguous mode gives GPU r the tokens the CP/EP page
    prints for 128K tokens on 8 GPUs: 16K*r .. 16K*(r+1)."""
    seq_k, n = (int(x) for x in golden["cp_layout_sequence_k_and_ranks"])
    first = [int(x) * k for x in golden["cp_layout_rank_first_token_k"]]
    segs = B.segments([(seq_k * k, 0, 0, 0)])
    for r in range(n):
        got = B.cp_rank_ranges(segs, 1, n, B.CP_SHARD_CONTIGUOUS, r)
        rows = [t for g in got for t in range(g.row0, g.row0 + g.len)]
        assert rows == list(range(first[r], first[r + 1]))
