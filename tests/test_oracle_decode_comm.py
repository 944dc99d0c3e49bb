"""Pins for the decode reference and the communication accounting."""
import math

import numpy as np
import pytest

from oracle import attention as A
from oracle import comm as C
from oracle import decode as D
from oracle import plan as P


def _decode_case(rng, lens, n_h=4, n_kv=1, d=8):
    offsets = np.concatenate([[0], np.cumsum(lens)])
    q = rng.standard_normal((len(lens), n_h, d))
    k = rng.standard_normal((offsets[-1], n_kv, d))
    v = rng.standard_normal((offsets[-1], n_kv, d))
    return q, k, v, offsets


def test_split_decode_equals_whole():
    rng = np.random.default_rng(0)
    q, k, v, off = _decode_case(rng, [37, 5, 300], n_h=8, n_kv=2)
    o1, l1 = D.decode(q, k, v, off)
    for n_splits in (1, 4, 16, 256):
        o2, l2 = D.decode_split(q, k, v, off, n_splits)
        np.testing.assert_allclose(o2, o1, atol=1e-12)
        np.testing.assert_allclose(l2, l1, atol=1e-12)


def test_decode_zero_q_log_length():
    rng = np.random.default_rng(1)
    q, k, v, off = _decode_case(rng, [9, 130])
    q[:] = 0
    o, lse = D.decode(q, k, v, off)
    np.testing.assert_allclose(lse[0], math.log(9), atol=1e-13)
    np.testing.assert_allclose(lse[1], math.log(130), atol=1e-13)
    np.testing.assert_allclose(o[1, 0], v[9:139, 0].mean(0), atol=1e-13)


def test_decode_is_last_prefill_row():
    """Decoding token L-1 over L cached keys equals the last row of a causal prefill."""
    rng = np.random.default_rng(2)
    q, k, v, off = _decode_case(rng, [50], n_h=4, n_kv=2)
    qp = rng.standard_normal((50, 4, 8))
    qp[-1] = q[0]
    o_pf, l_pf = A.attention(qp, k, v, np.arange(50), np.arange(50))
    o_dc, l_dc = D.decode(q, k, v, off)
    np.testing.assert_allclose(o_dc[0], o_pf[-1], atol=1e-12)
    np.testing.assert_allclose(l_dc[0], l_pf[-1], atol=1e-12)


def test_page_ratio_and_threshold(golden):
    n_h, n_kv = (int(x) for x in golden["llama3_405b_heads"])
    assert C.cp_over_tp_ratio(n_h, n_kv) == float(golden["cp_over_tp_message_ratio_128_8"][0])
    assert C.miss_rate_threshold(n_h, n_kv) == float(golden["miss_rate_threshold_128_8"][0])


def test_variant_selection_crosses_at_threshold():
    n_h, n_kv = 128, 8
    total = 128000
    for t in range(100, total, 700):
        miss = t / total
        want = P.PASS_KV if miss > 0.125 else P.PASS_Q
        assert C.select_variant(t, total - t, n_h, n_kv) == want
    t_sw, p_sw = 6400, 121600
    assert C.select_variant(t_sw, p_sw, n_h, n_kv) == P.PASS_Q    # 5% < 12.5%


def test_volume_crossover_is_the_threshold():
    """Per hop, pass-Q's Q bytes equal pass-KV's K+V bytes exactly at T/(T+P) = 2 N_KV/N_H."""
    n_h, n_kv, d = 128, 8, 128
    t, p = 1600, 11200          # miss = 1/8
    n = 4
    q_segs = [P.Segment(t, 0, p, 0)]
    kv_segs = [P.Segment(p, 0, 0, 0), P.Segment(t, p, p, 0)]
    r1, b1, _ = P.ring_schedule(q_segs, kv_segs, n, P.LOAD_BALANCED, P.PASS_KV)
    r2, b2, _ = P.ring_schedule(q_segs, kv_segs, n, P.LOAD_BALANCED, P.PASS_Q)
    kv = C.schedule_volume(r1, b1, n, P.PASS_KV, n_h, n_kv, d)["total"]
    qv = C.schedule_volume(r2, b2, n, P.PASS_Q, n_h, n_kv, d)["total"]
    assert qv == 2 * kv


@pytest.mark.parametrize("t,n", [(131072, 8), (256, 4), (96, 3)])
def test_pass_kv_volume_closed_form(t, n):
    n_kv, d = 1, 128
    segs = [P.Segment(t, 0, 0, 0)]
    ranges, blocks, _ = P.ring_schedule(segs, segs, n, P.LOAD_BALANCED, P.PASS_KV)
    vol = C.schedule_volume(ranges, blocks, n, P.PASS_KV, 16, n_kv, d)
    for hop in vol["hops"]:
        assert hop == [C.cp_block_elems(t // n, n_kv, d)] * n      # T_shard * N_KV * D_H
    assert vol["total"] == (n - 1) * C.cp_block_elems(t, n_kv, d)   # (N-1) * T * N_KV * D_H


def test_pass_q_volume():
    t, n, n_h, d = 4096, 8, 128, 128
    q_segs = [P.Segment(t, 0, 126976, 0)]
    kv_segs = [P.Segment(126976, 0, 0, 0), P.Segment(t, 126976, 126976, 0)]
    ranges, blocks, _ = P.ring_schedule(q_segs, kv_segs, n, P.LOAD_BALANCED, P.PASS_Q)
    vol = C.schedule_volume(ranges, blocks, n, P.PASS_Q, n_h, 8, d)
    assert vol["total"] == (n - 1) * t * n_h * d
    assert vol["all_to_all"] == (n - 1) * t * n_h * (d + 1)


def test_algorithm1_second_condition():
    """Condition 2 of Algorithm 1: below the miss-rate threshold pass-KV is
    still chosen when one KV hop hides under one ring step of attention. Pins:
    the hop time of the page's switch point (T=6400, P=121600, 8 KV heads of
    128, 8 ranks, bf16) is 16000 tokens x 8 x 128 x 2 tensors x 2 bytes =
    65,536,000 bytes over the link; the conditions apply in order."""
    n_h, n_kv, d, n, eb = 128, 8, 128, 8, 2
    t, p = 6400, 121600
    link = 50e9   # 400 Gb/s per GPU, the page's RDMA network
    hop = C.kv_hop_seconds(t, p, n_kv, d, n, eb, link)
    assert hop == 65_536_000 / link
    assert C.select_variant_alg1(t, p, n_h, n_kv, d, n, eb, link, hop) == (P.PASS_KV, 2)          # hides exactly
    assert C.select_variant_alg1(t, p, n_h, n_kv, d, n, eb, link, hop * 0.999) == (P.PASS_Q, 0)   # does not
    # condition 1 wins regardless of timing
    assert C.select_variant_alg1(64000, 64000, n_h, n_kv, d, n, eb, link, 0.0) == (P.PASS_KV, 1)
    # at exactly the threshold condition 1 does not fire (strict), condition 2 decides
    assert C.select_variant_alg1(16000, 112000, n_h, n_kv, d, n, eb, link, 0.0) == (P.PASS_Q, 0)
    # a faster link turns the same workload to pass-KV
    assert C.select_variant_alg1(t, p, n_h, n_kv, d, n, eb, 770e9, hop / 10)[0] == P.PASS_KV
    # with condition 2 unsatisfiable, the choice is condition 1 alone
    for tt in range(100, 128000, 3100):
        assert C.select_variant_alg1(tt, 128000 - tt, n_h, n_kv, d, n, eb, link, 0.0)[0] == \
            C.select_variant(tt, 128000 - tt, n_h, n_kv)
