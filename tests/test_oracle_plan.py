"""Pins for the reference shard planner: partitions, the load-balance closed
forms and the ring structure."""
import itertools

import numpy as np
import pytest

from oracle import plan as P


@pytest.mark.parametrize("length,n", [(256, 4), (131072, 8), (7, 4), (1, 2), (100, 3), (0, 2)])
def test_chunks_partition(length, n):
    b = P.chunk_bounds(length, n)
    assert b[0] == 0 and b[-1] == length and len(b) == 2 * n + 1
    sizes = np.diff(b)
    assert sizes.min() >= 0 and sizes.max() - sizes.min() <= 1


@pytest.mark.parametrize("mode", [P.LOAD_BALANCED, P.CONTIGUOUS])
@pytest.mark.parametrize("lens,n", [([256], 4), ([13, 40, 2], 3), ([5], 4)])
def test_token_index_is_permutation(mode, lens, n):
    segs, r0 = [], 0
    for s, ln in enumerate(lens):
        segs.append(P.Segment(ln, r0, 0, s))
        r0 += ln
    _, rank_rows, tok = P.shard_plan(segs, n, mode)
    assert sorted(tok) == list(range(r0))
    assert rank_rows[0] == 0 and rank_rows[-1] == r0
    assert all(a <= b for a, b in zip(rank_rows, rank_rows[1:]))


def _rank_total_pairs(length, n, mode, rank):
    seg = [P.Segment(length, 0, 0, 0)]
    mine = P.rank_ranges(seg, n, mode, rank)
    everything = P.Range(0, 0, length, 0)
    return sum(P.visible_pairs(r, everything) for r in mine)


@pytest.mark.parametrize("n,c", [(2, 3), (4, 32), (8, 5)])
def test_load_balanced_closed_form(n, c):
    """Every rank's causal work is C^2 (2N-1) + C (C+1): the balance claim."""
    length = 2 * n * c
    for r in range(n):
        assert _rank_total_pairs(length, n, P.LOAD_BALANCED, r) == c * c * (2 * n - 1) + c * (c + 1)


@pytest.mark.parametrize("n,cc", [(2, 6), (4, 64), (8, 3)])
def test_contiguous_closed_form(n, cc):
    """Contiguous shards are unbalanced: rank k holds C'^2 k + C'(C'+1)/2 pairs."""
    length = n * cc
    for r in range(n):
        assert _rank_total_pairs(length, n, P.CONTIGUOUS, r) == cc * cc * r + cc * (cc + 1) // 2


@pytest.mark.parametrize("n,c", [(4, 32), (3, 7), (8, 4)])
@pytest.mark.parametrize("variant", [P.PASS_KV, P.PASS_Q])
def test_block_pairs_closed_form(n, c, variant):
    segs = [P.Segment(2 * n * c, 0, 0, 0)]
    ranges, blocks, _ = P.ring_schedule(segs, segs, n, P.LOAD_BALANCED, variant)
    for t in range(n):
        for i in range(n):
            b = blocks[t * n + i]
            same = b.q_begin == b.kv_begin - len(ranges) // 2
            want = c * c + c * (c + 1) if same else 2 * c * c
            assert P.block_pairs(ranges, b) == want


def test_visible_pairs_bruteforce():
    rng = np.random.default_rng(0)
    for _ in range(200):
        q = P.Range(0, int(rng.integers(0, 20)), int(rng.integers(0, 9)), 0)
        k = P.Range(0, int(rng.integers(0, 20)), int(rng.integers(0, 9)), int(rng.integers(0, 2)))
        brute = sum(1 for a in range(q.pos0, q.pos0 + q.length)
                    for b in range(k.pos0, k.pos0 + k.length) if b <= a and k.seq == q.seq)
        assert P.visible_pairs(q, k) == brute
        cls = P.pair_class(q, k)
        if brute == 0:
            assert cls == P.SKIP
        elif brute == q.length * k.length:
            assert cls == P.FULL
        else:
            assert cls == P.PARTIAL


@pytest.mark.parametrize("n", [1, 2, 5, 8])
@pytest.mark.parametrize("variant", [P.PASS_KV, P.PASS_Q])
def test_ring_covers_every_pair_once(n, variant):
    segs = [P.Segment(4 * n, 0, 0, 0)]
    ranges, blocks, parts = P.ring_schedule(segs, segs, n, P.LOAD_BALANCED, variant)
    n_q = len(ranges) // 2
    seen = set()
    per_q_parts = {}
    for idx, (b, part) in enumerate(zip(blocks, parts)):
        qr = [j for j in range(n) if b.q_begin == 2 * j]
        kr = [j for j in range(n) if b.kv_begin == n_q + 2 * j]
        assert len(qr) == 1 and len(kr) == 1
        seen.add((qr[0], kr[0]))
        per_q_parts.setdefault(qr[0], []).append(part)
        t, i = divmod(idx, n)
        if variant == P.PASS_KV:
            assert qr[0] == i and kr[0] == (i - t) % n
        else:
            assert kr[0] == i and qr[0] == (i - t) % n
    assert seen == set(itertools.product(range(n), range(n)))
    assert all(sorted(v) == list(range(n)) for v in per_q_parts.values())


@pytest.mark.parametrize("k", [1000, 1024])
def test_contiguous_layout_matches_page(golden, k):
    """The contiguous shard mode is the layout the CP/EP page prints for 128K
    tokens on 8 GPUs (GPU r holds tokens 16K*r .. 16K*(r+1)); K is read as
    1000 and as 1024 tokens, and the layout holds for both."""
    seq_k, n = (int(x) for x in golden["cp_layout_sequence_k_and_ranks"])
    first = [int(x) * k for x in golden["cp_layout_rank_first_token_k"]]
    segs = [P.Segment(seq_k * k, 0, 0, 0)]
    for r in range(n):
        rows = [t for g in P.rank_ranges(segs, n, P.CONTIGUOUS, r) for t in range(g.row0, g.row0 + g.length)]
        assert rows == list(range(first[r], first[r + 1]))
