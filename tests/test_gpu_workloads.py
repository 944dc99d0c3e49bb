"""GPU parity at the full workload sizes, in the launch configuration the
bench times, on sampled rows the fp64 reference computes one by one.

Samples always include the first and last row of every chunk (and every
sequence), plus seeded random rows."""
import math

import numpy as np
import pytest
import torch

from context_ring_attn_b200 import binding as B
from context_ring_attn_b200 import ring, synth
from oracle import attention as OA
from oracle import decode as OD
from oracle import plan as OP

from gpu_util import check, sample_rows

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    B.lib()


def _host_kv(w, n_rows):
    k = synth.stored_values(synth.normal_rows(w["seed"], synth.TENSOR_K, n_rows, (w["n_kv"], w["d"]), w["std"]),
                            "bf16")[0]
    v = synth.stored_values(synth.normal_rows(w["seed"], synth.TENSOR_V, n_rows, (w["n_kv"], w["d"]), w["std"]),
                            "bf16")[0]
    return k, v


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


@pytest.mark.parametrize("merge", ["final", "fused"])
def test_prefill_128k_pass_kv(merge):
    """The headline step (separate 8-way merge) and its fused-merge variant."""
    w = synth.WORKLOADS["prefill_128k"]
    t, n_h, n_kv, d, n = w["t"], w["n_h"], w["n_kv"], w["d"], w["n_ranks"]
    q, k, v = _dev(w, synth.TENSOR_Q, t, n_h), _dev(w, synth.TENSOR_K, t, n_kv), _dev(w, synth.TENSOR_V, t, n_kv)
    segs = [ring.Segment(t, 0, 0, 0)]
    sched = ring.RingSchedule(segs, segs, n, B.CP_PASS_KV)
    out = torch.empty((t, n_h, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((t, n_h), dtype=torch.float32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    ring.run_ring(sched, q, k, v, n_h, n_kv, out, lse, workspace=ws, merge=merge)
    B.cp_check_status(ws)
    rows = sample_rows(np.random.default_rng(2), t, 1024, _chunk_edges([t], [0], n))
    o_gpu = out[torch.from_numpy(rows).cuda()].float().cpu().numpy()
    l_gpu = lse[torch.from_numpy(rows).cuda()].cpu().numpy()
    del q, out, lse
    kh, vh = _host_kv(w, t)
    qs = synth.stored_values(synth.normal_rows(w["seed"], synth.TENSOR_Q, t, (n_h, d), w["std"], rows), "bf16")[0]
    o_ref, l_ref = OA.attention(qs, kh, vh, rows, np.arange(t))
    check(o_gpu, l_gpu, o_ref, l_ref, "bf16", "prefill_128k")


def test_persistent_kv_pass_q_and_pass_kv_agree():
    w = synth.WORKLOADS["persistent_kv"]
    t, p, n_h, n_kv, d, n = w["t"], w["p"], w["n_h"], w["n_kv"], w["d"], w["n_ranks"]
    q = _dev(w, synth.TENSOR_Q, t, n_h)
    k, v = _dev(w, synth.TENSOR_K, p + t, n_kv), _dev(w, synth.TENSOR_V, p + t, n_kv)
    q_segs = [ring.Segment(t, 0, p, 0)]
    kv_segs = [ring.Segment(p, 0, 0, 0), ring.Segment(t, p, p, 0)]
    outs = {}
    for variant in (B.CP_PASS_Q, B.CP_PASS_KV):
        sched = ring.RingSchedule(q_segs, kv_segs, n, variant)
        out = torch.empty((t, n_h, d), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((t, n_h), dtype=torch.float32, device="cuda")
        ring.run_ring(sched, q, k, v, n_h, n_kv, out, lse)
        outs[variant] = (out, lse)
    torch.cuda.synchronize()
    # the two ring variants agree on every row
    diff = (outs[B.CP_PASS_Q][0].float() - outs[B.CP_PASS_KV][0].float()).abs().max().item()
    ldiff = (outs[B.CP_PASS_Q][1] - outs[B.CP_PASS_KV][1]).abs().max().item()
    assert diff <= 2e-2 and ldiff <= 1e-3, (diff, ldiff)
    must = [0, t - 1] + _chunk_edges([t], [0], n)
    rows = sample_rows(np.random.default_rng(3), t, 64, must)
    sel = torch.from_numpy(rows).cuda()
    o_gpu = outs[B.CP_PASS_Q][0][sel].float().cpu().numpy()
    l_gpu = outs[B.CP_PASS_Q][1][sel].cpu().numpy()
    del outs, q, k, v
    kh, vh = _host_kv(w, p + t)
    qs = synth.stored_values(synth.normal_rows(w["seed"], synth.TENSOR_Q, t, (n_h, d), w["std"], rows), "bf16")[0]
    o_ref, l_ref = OA.attention(qs, kh, vh, p + rows, np.arange(p + t))
    check(o_gpu, l_gpu, o_ref, l_ref, "bf16", "persistent_kv")


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


@pytest.mark.parametrize("merge", ["fused", "running"])
def test_varlen_prefill_pass_kv(merge):
    """The full varlen workload in both merge modes the bench times (fused is
    the workload's default)."""
    w = synth.WORKLOADS["varlen_prefill"]
    lens = synth.varlen_lengths(w["seed"], w["n_seq"], w["total"])
    total, n_h, n_kv, d, n = w["total"], w["n_h"], w["n_kv"], w["d"], w["n_ranks"]
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)
    segs = [ring.Segment(int(ln), int(s), 0, i) for i, (ln, s) in enumerate(zip(lens, starts))]
    q = _dev(w, synth.TENSOR_Q, total, n_h)
    k, v = _dev(w, synth.TENSOR_K, total, n_kv), _dev(w, synth.TENSOR_V, total, n_kv)
    sched = ring.RingSchedule(segs, segs, n, B.CP_PASS_KV)
    out = torch.empty((total, n_h, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((total, n_h), dtype=torch.float32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    ring.run_ring(sched, q, k, v, n_h, n_kv, out, lse, workspace=ws, merge=merge)
    B.cp_check_status(ws)
    must = [int(s) for s in starts] + [int(s + ln - 1) for s, ln in zip(starts, lens)]
    must += _chunk_edges([lens[0]], [0], n)
    rows = sample_rows(np.random.default_rng(5), total, 128, must)
    sel = torch.from_numpy(rows).cuda()
    o_gpu = out[sel].float().cpu().numpy()
    l_gpu = lse[sel].cpu().numpy()
    del q, out, lse, k, v
    torch.cuda.empty_cache()
    kh, vh = _host_kv(w, total)
    qs = synth.stored_values(synth.normal_rows(w["seed"], synth.TENSOR_Q, total, (n_h, d), w["std"], rows), "bf16")[0]
    # keys of other sequences are never visible: each sequence is checked against its own keys
    o_ref = np.zeros((rows.size, n_h, d))
    l_ref = np.zeros((rows.size, n_h))
    for s0, ln in zip(starts, lens):
        sel_rows = np.nonzero((rows >= s0) & (rows < s0 + ln))[0]
        if sel_rows.size == 0:
            continue
        o_ref[sel_rows], l_ref[sel_rows] = OA.attention(qs[sel_rows], kh[s0:s0 + ln], vh[s0:s0 + ln],
                                                        rows[sel_rows] - s0, np.arange(ln))
    check(o_gpu, l_gpu, o_ref, l_ref, "bf16", "varlen_prefill")
