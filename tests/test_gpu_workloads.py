"""GPU parity at the full workload sizes, in the launch configuration the
bench times, on sampled rows the fp64 reference computes one by one.

Each prefill workload's own launch configuration is checked on N_SAMPLE =
2048 query tokens (all heads of each), which always include the first and
last row of every chunk of the load-balanced plan and of every sequence, plus
seeded random rows. Its other variants (the fused or bf16-partial merge, the
running merge, and Q scaled by 8, "peaked": the softmax concentrates on a few
keys, so |O| is of order 0.5 rather than 0.5/sqrt(keys) and the absolute
bounds bite) are checked on N_SAMPLE_VARIANT = 512 tokens with the same forced
rows. Scaling bf16 values by a power of two is exact, so the reference sees
the same Q the GPU does."""
import math

import numpy as np
import pytest
import torch

from context_ring_attn_b200 import binding as B
from context_ring_attn_b200 import ring, synth
from oracle import attention as OA
from oracle import decode as OD
from oracle import plan as OP

from gpu_util import check, oracle_rows, sample_rows

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

N_SAMPLE = 2048
N_SAMPLE_VARIANT = 512


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    B.lib()


def _host_kv(w, n_rows):
    """K and V as stored (bf16 values), widened to float64 once for the reference."""
    k = synth.stored_values(synth.normal_rows(w["seed"], synth.TENSOR_K, n_rows, (w["n_kv"], w["d"]), w["std"]),
                            "bf16")[0]
    v = synth.stored_values(synth.normal_rows(w["seed"], synth.TENSOR_V, n_rows, (w["n_kv"], w["d"]), w["std"]),
                            "bf16")[0]
    return k.astype(np.float64), v.astype(np.float64)


def _host_q(w, n_rows, rows, q_mult):
    qs = synth.stored_values(synth.normal_rows(w["seed"], synth.TENSOR_Q, n_rows, (w["n_h"], w["d"]), w["std"], rows),
                             "bf16")[0]
    return qs.astype(np.float64) * q_mult


def _dev(w, tid, n_rows, heads):
    return synth.device_rows(w["seed"], tid, n_rows, (heads, w["d"]), w["std"], "bf16")


def _chunk_edges(lengths, starts, n_ranks):
    must = []
    for ln, s in zip(lengths, starts):
        b = OP.chunk_bounds(ln, n_ranks)
        for c in range(2 * n_ranks):
            if b[c + 1] > b[c]:
                must += [s + b[c], s + b[c + 1] - 1]
    return must


def _gather(out, lse, rows):
    sel = torch.from_numpy(rows).cuda()
    return out[sel].float().cpu().numpy(), lse[sel].cpu().numpy()


@pytest.mark.parametrize("merge,q_mult", [("final", 1.0), ("fused", 1.0), ("final_bf16", 1.0), ("final", 8.0)])
def test_prefill_128k_pass_kv(merge, q_mult):
    """The headline step (separate 8-way merge), its fused-merge and bf16-
    partial variants, and the headline step on peaked queries."""
    w = synth.WORKLOADS["prefill_128k"]
    t, n_h, n_kv, d, n = w["t"], w["n_h"], w["n_kv"], w["d"], w["n_ranks"]
    q, k, v = _dev(w, synth.TENSOR_Q, t, n_h), _dev(w, synth.TENSOR_K, t, n_kv), _dev(w, synth.TENSOR_V, t, n_kv)
    if q_mult != 1.0:
        q.mul_(q_mult)
    segs = [ring.Segment(t, 0, 0, 0)]
    sched = ring.RingSchedule(segs, segs, n, B.CP_PASS_KV)
    out = torch.empty((t, n_h, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((t, n_h), dtype=torch.float32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    ring.run_ring(sched, q, k, v, n_h, n_kv, out, lse, workspace=ws, merge=merge)
    B.cp_check_status(ws)
    n_sample = N_SAMPLE if (merge, q_mult) == ("final", 1.0) else N_SAMPLE_VARIANT
    rows = sample_rows(np.random.default_rng(2 + int(q_mult)), t, n_sample, _chunk_edges([t], [0], n))
    assert rows.size >= n_sample
    o_gpu, l_gpu = _gather(out, lse, rows)
    del q, k, v, out, lse
    torch.cuda.empty_cache()
    kh, vh = _host_kv(w, t)
    qs = _host_q(w, t, rows, q_mult)
    o_ref, l_ref = oracle_rows(lambda a, b: OA.attention(qs[a:b], kh, vh, rows[a:b], np.arange(t)), rows.size)
    check(o_gpu, l_gpu, o_ref, l_ref, "bf16", f"prefill_128k merge={merge} q*{q_mult}")


def test_persistent_kv_pass_q_and_pass_kv():
    """Both ring variants on the persistent-KV workload: each against the
    reference on the sampled rows, and the two against each other on every row."""
    w = synth.WORKLOADS["persistent_kv"]
    t, p, n_h, n_kv, d, n = w["t"], w["p"], w["n_h"], w["n_kv"], w["d"], w["n_ranks"]
    q = _dev(w, synth.TENSOR_Q, t, n_h)
    k, v = _dev(w, synth.TENSOR_K, p + t, n_kv), _dev(w, synth.TENSOR_V, p + t, n_kv)
    q_segs = [ring.Segment(t, 0, p, 0)]
    kv_segs = [ring.Segment(p, 0, 0, 0), ring.Segment(t, p, p, 0)]
    # query rows at positions P and P+T-1 and the chunk edges of the new tokens' plan
    must = [0, t - 1] + _chunk_edges([t], [0], n)
    rows = sample_rows(np.random.default_rng(3), t, N_SAMPLE, must)
    assert rows.size >= N_SAMPLE
    outs, got = {}, {}
    for variant in (B.CP_PASS_Q, B.CP_PASS_KV):
        sched = ring.RingSchedule(q_segs, kv_segs, n, variant)
        out = torch.empty((t, n_h, d), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((t, n_h), dtype=torch.float32, device="cuda")
        ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
        ring.run_ring(sched, q, k, v, n_h, n_kv, out, lse, workspace=ws)
        B.cp_check_status(ws)
        outs[variant] = (out, lse)
        got[variant] = _gather(out, lse, rows)
    diff = (outs[B.CP_PASS_Q][0].float() - outs[B.CP_PASS_KV][0].float()).abs().max().item()
    ldiff = (outs[B.CP_PASS_Q][1] - outs[B.CP_PASS_KV][1]).abs().max().item()
    assert diff <= 2e-2 and ldiff <= 1e-3, (diff, ldiff)
    del outs, q, k, v
    torch.cuda.empty_cache()
    kh, vh = _host_kv(w, p + t)
    qs = _host_q(w, t, rows, 1.0)
    o_ref, l_ref = oracle_rows(lambda a, b: OA.attention(qs[a:b], kh, vh, p + rows[a:b], np.arange(p + t)),
                               rows.size, chunk=64)
    for variant, name in ((B.CP_PASS_Q, "pass-Q"), (B.CP_PASS_KV, "pass-KV")):
        check(*got[variant], o_ref, l_ref, "bf16", f"persistent_kv {name}")


def test_decode_split_full():
    w = synth.WORKLOADS["decode_split"]
    lens = synth.decode_lengths(w["seed"], w["batch"], w["lo"], w["hi"])
    dc = synth.make_decode(w["batch"], w["n_h"], w["n_kv"], w["d"], lens, w["seed"], w["std"])
    to = lambda raw: torch.from_numpy(raw.view(np.int16)).view(torch.bfloat16).cuda()  # noqa: E731
    out = torch.empty((w["batch"], w["n_h"], w["d"]), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w["batch"], w["n_h"]), dtype=torch.float32, device="cuda")
    ws = torch.zeros(B.cp_workspace_size(B.CP_OP_DECODE, w["batch"], w["n_h"], w["d"], w["n_splits"]),
                     dtype=torch.uint8, device="cuda")
    B.cp_decode(to(dc.q_raw), to(dc.k_raw), to(dc.v_raw), torch.from_numpy(dc.offsets).cuda(), w["n_h"], w["n_kv"],
                w["n_splits"], 1 / math.sqrt(w["d"]), out, lse, ws)
    B.cp_check_status(ws)
    o_ref, l_ref = OD.decode(dc.q, dc.k, dc.v, dc.offsets)
    check(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, "bf16", "decode_split")


@pytest.mark.parametrize("merge,q_mult", [("final_bf16", 1.0), ("fused", 1.0), ("running", 1.0),
                                          ("final_bf16", 8.0)])
def test_varlen_prefill_pass_kv(merge, q_mult):
    """The full varlen workload in the merge modes the bench times (bf16
    partial buffers and one 8-way merge is the workload's default), and the
    default on peaked queries."""
    w = synth.WORKLOADS["varlen_prefill"]
    lens = synth.varlen_lengths(w["seed"], w["n_seq"], w["total"])
    total, n_h, n_kv, d, n = w["total"], w["n_h"], w["n_kv"], w["d"], w["n_ranks"]
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)
    segs = [ring.Segment(int(ln), int(s), 0, i) for i, (ln, s) in enumerate(zip(lens, starts))]
    q = _dev(w, synth.TENSOR_Q, total, n_h)
    if q_mult != 1.0:
        q.mul_(q_mult)
    k, v = _dev(w, synth.TENSOR_K, total, n_kv), _dev(w, synth.TENSOR_V, total, n_kv)
    sched = ring.RingSchedule(segs, segs, n, B.CP_PASS_KV)
    out = torch.empty((total, n_h, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((total, n_h), dtype=torch.float32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    ring.run_ring(sched, q, k, v, n_h, n_kv, out, lse, workspace=ws, merge=merge)
    B.cp_check_status(ws)
    must = [int(s) for s in starts] + [int(s + ln - 1) for s, ln in zip(starts, lens)]
    must += _chunk_edges([int(x) for x in lens], [int(s) for s in starts], n)
    n_sample = N_SAMPLE if (merge, q_mult) == ("final_bf16", 1.0) else N_SAMPLE_VARIANT
    rows = sample_rows(np.random.default_rng(5 + int(q_mult)), total, n_sample, must)
    assert rows.size >= n_sample
    o_gpu, l_gpu = _gather(out, lse, rows)
    del q, out, lse, k, v
    torch.cuda.empty_cache()
    kh, vh = _host_kv(w, total)
    qs = _host_q(w, total, rows, q_mult)
    # keys of other sequences are never visible: each sequence is checked against its own keys
    o_ref = np.zeros((rows.size, n_h, d))
    l_ref = np.zeros((rows.size, n_h))
    for s0, ln in zip(starts, lens):
        idx = np.nonzero((rows >= s0) & (rows < s0 + ln))[0]
        if idx.size == 0:
            continue
        ks, vs = kh[s0:s0 + ln], vh[s0:s0 + ln]
        qi, pos = qs[idx], rows[idx] - s0
        o_ref[idx], l_ref[idx] = oracle_rows(lambda a, b: OA.attention(qi[a:b], ks, vs, pos[a:b], np.arange(ln)),
                                             idx.size, chunk=64)
    check(o_gpu, l_gpu, o_ref, l_ref, "bf16", f"varlen_prefill merge={merge} q*{q_mult}")
