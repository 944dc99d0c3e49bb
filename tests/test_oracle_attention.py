"""Pins for the fp64 attention reference: library special cases, brute force,
invariants. None of these re-types the reference's own formula."""
import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import plan as P

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _sdpa(q, k, v, q_pos, k_pos, causal, scale):
    """torch SDPA in fp64 on CPU, with GQA expanded by repeat_interleave and an
    explicit boolean keep-mask for the positions."""
    n_h, n_kv = q.shape[1], k.shape[1]
    g = n_h // n_kv
    qt = torch.tensor(q).permute(1, 0, 2)                       # [H, Tq, D]
    kt = torch.tensor(k).repeat_interleave(g, dim=1).permute(1, 0, 2)
    vt = torch.tensor(v).repeat_interleave(g, dim=1).permute(1, 0, 2)
    keep = torch.ones(q.shape[0], k.shape[0], dtype=torch.bool)
    if causal:
        keep = torch.tensor(k_pos)[None, :] <= torch.tensor(q_pos)[:, None]
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=keep, scale=scale)
    return out.permute(1, 0, 2).numpy()


@pytest.mark.parametrize("tq,p,n_h,n_kv,d,causal", [
    (16, 0, 4, 1, 8, True), (33, 0, 4, 2, 16, True), (64, 0, 2, 2, 32, True),
    (20, 13, 8, 2, 8, True), (17, 5, 4, 4, 8, False), (1, 40, 4, 1, 16, True),
])
def test_matches_torch_sdpa(tq, p, n_h, n_kv, d, causal):
    rng = np.random.default_rng(tq * 100 + p)
    q, k, v = _rand(rng, tq, n_h, d), _rand(rng, tq + p, n_kv, d), _rand(rng, tq + p, n_kv, d)
    q_pos, k_pos = np.arange(p, p + tq), np.arange(tq + p)
    scale = 1.0 / math.sqrt(d)
    o, lse = A.attention(q, k, v, q_pos, k_pos, causal=causal, scale=scale)
    ref = _sdpa(q, k, v, q_pos, k_pos, causal, scale)
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    assert np.all(np.isfinite(lse))


def test_bruteforce_tiny_two_sequences():
    """Pure-Python loops over every (row, head, key), with math.exp."""
    rng = np.random.default_rng(7)
    n_h, n_kv, d = 4, 2, 3
    q, k, v = _rand(rng, 6, n_h, d), _rand(rng, 6, n_kv, d), _rand(rng, 6, n_kv, d)
    pos = np.array([0, 1, 2, 0, 1, 2])
    seq = np.array([0, 0, 0, 1, 1, 1])
    scale = 0.7
    o, lse = A.attention(q, k, v, pos, pos, seq, seq, scale=scale)
    for i in range(6):
        for h in range(n_h):
            g = h // (n_h // n_kv)
            ws, num = [], [0.0] * d
            for j in range(6):
                if seq[j] == seq[i] and pos[j] <= pos[i]:
                    ws.append((j, math.exp(scale * sum(q[i, h, c] * k[j, g, c] for c in range(d)))))
            z = sum(w for _, w in ws)
            for j, w in ws:
                for c in range(d):
                    num[c] += w / z * v[j, g, c]
            assert abs(lse[i, h] - math.log(z)) < 1e-12
            assert max(abs(num[c] - o[i, h, c]) for c in range(d)) < 1e-12


def test_uniform_v_gives_that_row():
    rng = np.random.default_rng(1)
    q, k = _rand(rng, 40, 8, 16) * 3, _rand(rng, 40, 2, 16) * 3
    vrow = _rand(rng, 2, 16)
    v = np.broadcast_to(vrow, (40, 2, 16)).copy()
    o, _ = A.attention(q, k, v, np.arange(40), np.arange(40))
    for h in range(8):
        np.testing.assert_allclose(o[:, h, :], np.broadcast_to(vrow[h // 4], (40, 16)), atol=1e-12)


def test_zero_q_gives_mean_and_log_count():
    rng = np.random.default_rng(2)
    p, t = 9, 25
    k, v = _rand(rng, p + t, 1, 8), _rand(rng, p + t, 1, 8)
    q = np.zeros((t, 4, 8))
    o, lse = A.attention(q, k, v, np.arange(p, p + t), np.arange(p + t))
    for i in range(t):
        n_vis = p + i + 1
        np.testing.assert_allclose(lse[i], math.log(n_vis), atol=1e-12)
        np.testing.assert_allclose(o[i], np.broadcast_to(v[:n_vis, 0].mean(0), (4, 8)), atol=1e-12)


def test_first_row_sees_only_itself():
    rng = np.random.default_rng(3)
    q, k, v = _rand(rng, 10, 2, 8), _rand(rng, 10, 1, 8), _rand(rng, 10, 1, 8)
    o, lse = A.attention(q, k, v, np.arange(10), np.arange(10), scale=0.25)
    for h in range(2):
        np.testing.assert_allclose(o[0, h], v[0, 0], atol=1e-14)
        np.testing.assert_allclose(lse[0, h], 0.25 * q[0, h] @ k[0, 0], atol=1e-14)


def test_key_permutation_invariance():
    rng = np.random.default_rng(4)
    q, k, v = _rand(rng, 30, 4, 8), _rand(rng, 30, 2, 8), _rand(rng, 30, 2, 8)
    pos = np.arange(30)
    o1, l1 = A.attention(q, k, v, pos, pos)
    perm = rng.permutation(30)
    o2, l2 = A.attention(q, k[perm], v[perm], pos, pos[perm])
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(l1, l2, atol=1e-12)


def test_merge_with_itself_adds_log2():
    rng = np.random.default_rng(5)
    o, lse = _rand(rng, 7, 3, 4), _rand(rng, 7, 3)
    om, lm = A.merge([o, o], [lse, lse])
    np.testing.assert_allclose(om, o, atol=1e-14)
    np.testing.assert_allclose(lm, lse + math.log(2.0), atol=1e-14)


def test_merge_neg_inf_parts():
    o1 = np.ones((2, 1, 3))
    o2 = np.full((2, 1, 3), 5.0)
    l1 = np.array([[0.5], [-np.inf]])
    l2 = np.array([[-np.inf], [-np.inf]])
    om, lm = A.merge([o1, o2], [l1, l2])
    np.testing.assert_allclose(om[0], 1.0)
    assert lm[0, 0] == 0.5
    assert np.all(om[1] == 0.0) and lm[1, 0] == -np.inf


def test_varlen_equals_separate_sequences():
    rng = np.random.default_rng(6)
    lens = [5, 11, 3]
    tot = sum(lens)
    q, k, v = _rand(rng, tot, 4, 8), _rand(rng, tot, 2, 8), _rand(rng, tot, 2, 8)
    seq = np.repeat(np.arange(3), lens)
    pos = np.concatenate([np.arange(n) for n in lens])
    o, lse = A.attention(q, k, v, pos, pos, seq, seq)
    r0 = 0
    for n in lens:
        os_, ls_ = A.attention(q[r0:r0 + n], k[r0:r0 + n], v[r0:r0 + n], np.arange(n), np.arange(n))
        np.testing.assert_allclose(o[r0:r0 + n], os_, atol=1e-13)
        np.testing.assert_allclose(lse[r0:r0 + n], ls_, atol=1e-13)
        r0 += n


def test_gqa_head_grouping_matches_page(golden):
    """Head h reads KV head floor(h / (N_H/N_KV)): with V constant per KV head,
    each query head's output names the KV head it used."""
    want = [int(x) for x in golden["gqa_kv_head_of_query_head_32_4"]]
    rng = np.random.default_rng(8)
    n_h, n_kv, d, t = 32, 4, 4, 5
    q, k = _rand(rng, t, n_h, d), _rand(rng, t, n_kv, d)
    v = np.zeros((t, n_kv, d))
    for g in range(n_kv):
        v[:, g, :] = g
    o, _ = A.attention(q, k, v, np.arange(t), np.arange(t))
    got = [int(round(o[-1, h, 0])) for h in range(n_h)]
    assert got == want


@pytest.mark.parametrize("n_ranks", [1, 2, 3, 4])
@pytest.mark.parametrize("mode", [P.LOAD_BALANCED, P.CONTIGUOUS])
@pytest.mark.parametrize("variant", [P.PASS_KV, P.PASS_Q])
@pytest.mark.parametrize("group", [1, 2, 4])
def test_shard_and_merge_equals_unsharded(n_ranks, mode, variant, group):
    """The ring is lossless exact: any plan, ring variant and merge order gives
    the unsharded result (method page, section 2 and section 4), for GQA groups
    of 1, 2 and 4 query heads per KV head."""
    rng = np.random.default_rng(1000 * group + 100 * n_ranks + 10 * mode + variant)
    lens = [29, 16]
    tot = sum(lens)
    n_h, d = 4, 8
    n_kv = n_h // group
    q, k, v = _rand(rng, tot, n_h, d), _rand(rng, tot, n_kv, d), _rand(rng, tot, n_kv, d)
    seq = np.repeat(np.arange(len(lens)), lens)
    pos = np.concatenate([np.arange(n) for n in lens])
    segs, r0 = [], 0
    for s, n in enumerate(lens):
        segs.append(P.Segment(n, r0, 0, s))
        r0 += n
    o_ref, l_ref = A.attention(q, k, v, pos, pos, seq, seq)
    ranges, blocks, parts = P.ring_schedule(segs, segs, n_ranks, mode, variant)
    o_parts = [np.zeros_like(o_ref) for _ in range(n_ranks)]
    l_parts = [np.full_like(l_ref, -np.inf) for _ in range(n_ranks)]
    for b, part in zip(blocks, parts):
        q_rows = np.concatenate([np.arange(ranges[j].row0, ranges[j].row0 + ranges[j].length)
                                 for j in range(b.q_begin, b.q_begin + b.q_count)] or [np.zeros(0, int)])
        kv_rows = np.concatenate([np.arange(ranges[j].row0, ranges[j].row0 + ranges[j].length)
                                  for j in range(b.kv_begin, b.kv_begin + b.kv_count)] or [np.zeros(0, int)])
        if q_rows.size == 0:
            continue
        ob, lb = A.block_partial(q[q_rows], k, v, pos[q_rows], pos, kv_rows, seq[q_rows], seq)
        o_parts[part][q_rows] = ob
        l_parts[part][q_rows] = lb
    order = rng.permutation(n_ranks)
    om, lm = A.merge([o_parts[i] for i in order], [l_parts[i] for i in order])
    np.testing.assert_allclose(om, o_ref, atol=1e-12)
    np.testing.assert_allclose(lm, l_ref, atol=1e-12)


def test_row_without_visible_keys():
    rng = np.random.default_rng(9)
    q, k, v = _rand(rng, 3, 2, 4), _rand(rng, 5, 1, 4), _rand(rng, 5, 1, 4)
    o, lse = A.attention(q, k, v, np.array([0, 1, 9]), np.arange(2, 7))
    assert np.all(o[:2] == 0) and np.all(lse[:2] == -np.inf)
    assert np.all(np.isfinite(lse[2]))
