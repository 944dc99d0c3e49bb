"""GPU parity of each kernel against the fp64 reference on small seeded
inputs that still span several tiles and a ragged tail."""
import math

import numpy as np
import pytest
import torch

from context_ring_attn_b200 import binding as B
from context_ring_attn_b200 import ring, synth
from oracle import attention as OA
from oracle import decode as OD
from oracle import plan as OP

from gpu_util import check, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    B.lib()


def _ws():
    return torch.zeros(256, dtype=torch.uint8, device="cuda")


def _run_prefill(pr, n_ranks, variant, mode, merge="final", q_scale=1.0, segs=None):
    """Ring attention through the library vs the unsharded reference."""
    t, p = pr.t, pr.p
    q_np = pr.q * q_scale
    q_raw = synth.bf16_bits(q_np) if pr.dtype == "bf16" else q_np.astype(np.float32)
    q = dev(q_raw, pr.dtype)
    k, v = dev(pr.k_raw, pr.dtype), dev(pr.v_raw, pr.dtype)
    if segs is None:
        q_segs = [ring.Segment(t, 0, p, 0)]
        kv_segs = [ring.Segment(p, 0, 0, 0), ring.Segment(t, p, p, 0)] if p else [ring.Segment(t, 0, 0, 0)]
        q_pos, k_pos = np.arange(p, p + t), np.arange(p + t)
        q_seq = k_seq = None
    else:
        q_segs = kv_segs = segs
        q_pos = k_pos = np.concatenate([np.arange(s.pos0, s.pos0 + s.length) for s in segs])
        q_seq = k_seq = np.concatenate([np.full(s.length, s.seq) for s in segs])
    sched = ring.RingSchedule(q_segs, kv_segs, n_ranks, variant, mode)
    out_dt = torch.bfloat16 if pr.dtype == "bf16" else torch.float32
    out = torch.empty((t, pr.n_h, pr.d), dtype=out_dt, device="cuda")
    lse = torch.empty((t, pr.n_h), dtype=torch.float32, device="cuda")
    ring.run_ring(sched, q, k, v, pr.n_h, pr.n_kv, out, lse, merge=merge, workspace=_ws())
    torch.cuda.synchronize()
    q_vals = synth.bf16_bits_to_f32(q_raw) if pr.dtype == "bf16" else q_raw
    o_ref, l_ref = OA.attention(q_vals, pr.k, pr.v, q_pos, k_pos, q_seq, k_seq)
    return check(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, pr.dtype,
                 f"{pr.dtype} T={t} P={p} N={n_ranks} var={variant} mode={mode}")


# ---------------------------------------------------------------------------- fp32 exact path
@pytest.mark.parametrize("variant", [B.CP_PASS_KV, B.CP_PASS_Q])
@pytest.mark.parametrize("mode", [B.CP_SHARD_LOAD_BALANCED, B.CP_SHARD_CONTIGUOUS])
def test_tiny_exact_fp32(variant, mode):
    w = synth.WORKLOADS["tiny_exact"]
    pr = synth.make_prefill(w["t"], w["n_h"], w["n_kv"], w["d"], "f32", w["seed"], w["std"])
    _run_prefill(pr, w["n_ranks"], variant, mode)


@pytest.mark.parametrize("merge", ["final", "running"])
def test_fp32_gqa_ragged(merge):
    pr = synth.make_prefill(301, 8, 2, 128, "f32", 11, 1.0, p=77)
    _run_prefill(pr, 3, B.CP_PASS_Q, B.CP_SHARD_LOAD_BALANCED, merge=merge)


def test_fp32_partial_empty_rows_and_noncausal():
    """A block whose queries sit before part of the KV range: some rows see
    nothing (O = 0, LSE = -inf); the non-causal block sees everything."""
    rng = np.random.default_rng(3)
    n_h, n_kv, d = 4, 2, 64
    q = rng.standard_normal((50, n_h, d)).astype(np.float32)
    k = rng.standard_normal((300, n_kv, d)).astype(np.float32)
    v = rng.standard_normal((300, n_kv, d)).astype(np.float32)
    ranges = (B.cp_range * 3)(B.cp_range(0, 100, 50, 0, 0), B.cp_range(20, 120, 200, 0, 0),
                              B.cp_range(0, 100, 20, 0, 0))
    for causal, blk in ((True, B.cp_block(0, 1, 1, 1, 0)), (False, B.cp_block(0, 1, 1, 2, 0))):
        blocks = (B.cp_block * 1)(blk)
        o = torch.full((50, n_h, d), float("nan"), device="cuda")
        lse = torch.full((50, n_h), float("nan"), device="cuda")
        B.cp_attn_partial(dev(q, "f32"), dev(k, "f32"), dev(v, "f32"), n_h, n_kv, 1 / 8, causal, ranges, 3,
                          blocks, 1, o, lse, _ws())
        torch.cuda.synchronize()
        kv_rows = np.arange(20, 220) if causal else np.concatenate([np.arange(20, 220), np.arange(0, 20)])
        k_pos = np.concatenate([np.arange(120, 320), np.arange(100, 120)])[:len(kv_rows)]
        o_ref, l_ref = OA.attention(q, k[kv_rows], v[kv_rows], np.arange(100, 150), k_pos, scale=1 / 8,
                                    causal=causal)
        check(o.cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, "f32", f"causal={causal}")
        if causal:
            assert np.all(np.isinf(l_ref[:20]))


# ---------------------------------------------------------------------------- bf16 tensor-core path
@pytest.mark.parametrize("t,n_h,n_kv,n_ranks,variant,mode", [
    (1000, 16, 1, 3, B.CP_PASS_KV, B.CP_SHARD_LOAD_BALANCED),
    (777, 8, 2, 2, B.CP_PASS_Q, B.CP_SHARD_LOAD_BALANCED),
    (1024, 16, 1, 4, B.CP_PASS_KV, B.CP_SHARD_CONTIGUOUS),
    (513, 128, 8, 2, B.CP_PASS_KV, B.CP_SHARD_LOAD_BALANCED),
    (300, 1, 1, 1, B.CP_PASS_KV, B.CP_SHARD_LOAD_BALANCED),
])
def test_bf16_ring(t, n_h, n_kv, n_ranks, variant, mode):
    pr = synth.make_prefill(t, n_h, n_kv, 128, "bf16", 100 + t, 0.5)
    _run_prefill(pr, n_ranks, variant, mode)


@pytest.mark.parametrize("t,n_h,n_kv,n_ranks,variant,p,merge", [
    (1000, 16, 1, 3, B.CP_PASS_KV, 0, "final"),
    (777, 8, 2, 2, B.CP_PASS_Q, 0, "final"),
    (300, 32, 2, 4, B.CP_PASS_Q, 1500, "final"),
    (513, 128, 8, 2, B.CP_PASS_KV, 0, "fused"),
    (129, 64, 1, 1, B.CP_PASS_KV, 0, "running"),
])
def test_bf16_ring_head_dim_64(t, n_h, n_kv, n_ranks, variant, p, merge):
    """The tensor-core partial with D_H = 64 (its own instantiation: one
    128-byte swizzle column per row, N = 64 PV products)."""
    pr = synth.make_prefill(t, n_h, n_kv, 64, "bf16", 700 + t, 0.5, p=p)
    _run_prefill(pr, n_ranks, variant, B.CP_SHARD_LOAD_BALANCED, merge=merge)
    _run_prefill(pr, n_ranks, variant, B.CP_SHARD_LOAD_BALANCED, merge=merge, q_scale=8.0)


@pytest.mark.parametrize("q_scale", [1.0, 8.0])
def test_bf16_persistent_kv_pass_q(q_scale):
    """T new tokens over P cached + T keys, queries sharded and LSE-merged;
    q_scale 8 makes the softmax peaked (|O| ~ |v|)."""
    pr = synth.make_prefill(300, 32, 2, 128, "bf16", 7, 0.5, p=1500)
    _run_prefill(pr, 4, B.CP_PASS_Q, B.CP_SHARD_LOAD_BALANCED, q_scale=q_scale)


def test_bf16_varlen_running_merge():
    lens = [700, 129, 1000]
    segs, r0 = [], 0
    for i, n in enumerate(lens):
        segs.append(ring.Segment(n, r0, 0, i))
        r0 += n
    pr = synth.make_prefill(sum(lens), 16, 2, 128, "bf16", 5, 0.5)
    _run_prefill(pr, 3, B.CP_PASS_KV, B.CP_SHARD_LOAD_BALANCED, merge="running", segs=segs)


def test_bf16_partial_empty_rows():
    rng = np.random.default_rng(4)
    n_h, n_kv, d = 16, 1, 128
    pr_q = synth.bf16_bits(rng.standard_normal((200, n_h, d)).astype(np.float32) * 0.5)
    pr_k = synth.bf16_bits(rng.standard_normal((600, n_kv, d)).astype(np.float32) * 0.5)
    pr_v = synth.bf16_bits(rng.standard_normal((600, n_kv, d)).astype(np.float32) * 0.5)
    ranges = (B.cp_range * 2)(B.cp_range(3, 1000, 190, 0, 0), B.cp_range(7, 1050, 500, 0, 0))
    blocks = (B.cp_block * 1)(B.cp_block(0, 1, 1, 1, 5))
    o = torch.full((200, n_h, d), float("nan"), device="cuda")
    lse = torch.full((200, n_h), float("nan"), device="cuda")
    B.cp_attn_partial(dev(pr_q, "bf16"), dev(pr_k, "bf16"), dev(pr_v, "bf16"), n_h, n_kv, 1 / math.sqrt(d), True,
                      ranges, 2, blocks, 1, o, lse, _ws())
    torch.cuda.synchronize()
    qv, kv, vv = (synth.bf16_bits_to_f32(x) for x in (pr_q, pr_k, pr_v))
    o_ref, l_ref = OA.attention(qv[3:193], kv[7:507], vv[7:507], np.arange(1000, 1190), np.arange(1050, 1550))
    check(o.cpu().numpy()[8:198], lse.cpu().numpy()[8:198], o_ref, l_ref, "bf16", "partial")
    assert np.isnan(o.cpu().numpy()[:8]).all() and np.isnan(o.cpu().numpy()[198:]).all()   # untouched rows


# ---------------------------------------------------------------------------- merge
@pytest.mark.parametrize("n_parts,d,out_dtype,n_h", [(1, 128, "f32", 4), (3, 64, "f32", 4), (8, 128, "bf16", 4),
                                                      (40, 128, "f32", 4), (256, 128, "bf16", 4),
                                                      (2, 128, "f32", 3), (5, 128, "bf16", 3), (3, 128, "f32", 3)])
def test_merge(n_parts, d, out_dtype, n_h):
    """Part counts that take every grouping of (row, head) pairs per warp and
    parts per round, with row-head counts (148, 111) that leave ragged tails."""
    rng = np.random.default_rng(n_parts)
    rows = 37
    o = rng.standard_normal((n_parts, rows, n_h, d)).astype(np.float32)
    lse = (rng.standard_normal((n_parts, rows, n_h)) * 3).astype(np.float32)
    lse[rng.random(lse.shape) < 0.2] = -np.inf
    lse[:, 5, 1] = -np.inf      # a row-head with no part
    o[np.isinf(lse)] = 0.0
    o_ref, l_ref = OA.merge(list(o), list(lse))
    out = torch.empty((rows, n_h, d), dtype=torch.bfloat16 if out_dtype == "bf16" else torch.float32, device="cuda")
    lse_out = torch.empty((rows, n_h), dtype=torch.float32, device="cuda")
    B.cp_attn_merge(dev(o, "f32"), dev(lse, "f32"), n_parts, rows, rows, n_h, d, out, lse_out)
    torch.cuda.synchronize()
    check(out.float().cpu().numpy(), lse_out.cpu().numpy(), o_ref, l_ref, "bf16" if out_dtype == "bf16" else "f32")


def test_merge_in_place():
    rng = np.random.default_rng(9)
    rows, n_h, d = 64, 8, 128
    o = rng.standard_normal((2, rows, n_h, d)).astype(np.float32)
    lse = rng.standard_normal((2, rows, n_h)).astype(np.float32)
    o_ref, l_ref = OA.merge(list(o), list(lse))
    od, ld = dev(o, "f32"), dev(lse, "f32")
    B.cp_attn_merge(od, ld, 2, rows, rows, n_h, d, od, ld)
    torch.cuda.synchronize()
    check(od[0].cpu().numpy(), ld[0].cpu().numpy(), o_ref, l_ref, "f32")


@pytest.mark.parametrize("n_parts", [2, 3, 8])
def test_merge_ignores_rows_of_parts_at_minus_inf(n_parts):
    """A part whose LSE is -inf weighs 0, so whatever its O row holds (NaN
    here) must not reach the output."""
    rng = np.random.default_rng(100 + n_parts)
    rows, n_h, d = 29, 4, 128
    o = rng.standard_normal((n_parts, rows, n_h, d)).astype(np.float32)
    lse = rng.standard_normal((n_parts, rows, n_h)).astype(np.float32)
    lse[0, ::3] = -np.inf
    lse[:, 7, 2] = -np.inf          # every part empty: O = 0, LSE = -inf
    o_clean = np.where(np.isinf(lse)[..., None], 0.0, o).astype(np.float32)
    o_ref, l_ref = OA.merge(list(o_clean), list(lse))
    o_dirty = np.where(np.isinf(lse)[..., None], np.nan, o).astype(np.float32)
    out = torch.empty((rows, n_h, d), dtype=torch.float32, device="cuda")
    lse_out = torch.empty((rows, n_h), dtype=torch.float32, device="cuda")
    B.cp_attn_merge(dev(o_dirty, "f32"), dev(lse, "f32"), n_parts, rows, rows, n_h, d, out, lse_out)
    torch.cuda.synchronize()
    check(out.cpu().numpy(), lse_out.cpu().numpy(), o_ref, l_ref, "f32", "merge with NaN in -inf parts")


def test_fused_accumulate_ignores_earlier_rows_at_minus_inf():
    """cp_attn_partial_fused with accumulate: an earlier (O, LSE) at -inf weighs
    0, so a NaN O row there must not reach the merged row."""
    t, n_h, n_kv, d = 300, 16, 1, 128
    pr = synth.make_prefill(t, n_h, n_kv, d, "bf16", 321, 0.5)
    q, k, v = dev(pr.q_raw, "bf16"), dev(pr.k_raw, "bf16"), dev(pr.v_raw, "bf16")
    ranges = (B.cp_range * 2)(B.cp_range(0, 0, t, 0, 0), B.cp_range(0, 0, t, 0, 0))
    blocks = (B.cp_block * 1)(B.cp_block(0, 1, 1, 1, 0))
    o_acc = torch.full((t, n_h, d), float("nan"), dtype=torch.float32, device="cuda")
    lse_acc = torch.full((t, n_h), float("-inf"), dtype=torch.float32, device="cuda")
    out = torch.empty((t, n_h, d), dtype=torch.bfloat16, device="cuda")
    B.cp_attn_partial_fused(q, k, v, n_h, n_kv, 1 / math.sqrt(d), True, ranges, 2, blocks, 1, o_acc, lse_acc, True,
                            out, _ws())
    torch.cuda.synchronize()
    o_ref, l_ref = OA.attention(pr.q, pr.k, pr.v, np.arange(t), np.arange(t))
    check(out.float().cpu().numpy(), lse_acc.cpu().numpy(), o_ref, l_ref, "bf16", "fused accumulate over -inf rows")


# ---------------------------------------------------------------------------- decode
@pytest.mark.parametrize("n_h,n_kv,n_splits,d", [
    (16, 1, 256, 128), (16, 2, 16, 128), (16, 1, 1, 128), (64, 4, 256, 128),
    (12, 4, 32, 128),     # G = 3: rows past the group are zero
    (128, 1, 64, 128),    # MQA, G = 128: eight 16-head units per KV head
    (64, 2, 16, 128),     # G = 32 on two KV heads
    (16, 1, 256, 64), (8, 8, 16, 64), (128, 2, 64, 64),   # head dim 64
])
def test_decode(n_h, n_kv, n_splits, d):
    lens = [0, 5, 100, 255, 256, 1000, 3001, 64]
    dc = synth.make_decode(len(lens), n_h, n_kv, d, lens, 40 + n_splits + n_h + d, 0.5)
    q, k, v = dev(dc.q_raw, "bf16"), dev(dc.k_raw, "bf16"), dev(dc.v_raw, "bf16")
    off = torch.from_numpy(dc.offsets).cuda()
    out = torch.empty((len(lens), n_h, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((len(lens), n_h), dtype=torch.float32, device="cuda")
    ws = torch.zeros(B.cp_workspace_size(B.CP_OP_DECODE, len(lens), n_h, d, n_splits), dtype=torch.uint8,
                     device="cuda")
    B.cp_decode(q, k, v, off, n_h, n_kv, n_splits, 1 / math.sqrt(d), out, lse, ws)
    B.cp_check_status(ws)
    o_ref, l_ref = OD.decode(dc.q, dc.k, dc.v, dc.offsets)
    check(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, "bf16", "decode")


def test_decode_reports_decreasing_offsets():
    """Offsets that decrease are reported through the status word; every row
    read stays inside the K/V rows the call was given."""
    lens = [100, 60, 140]
    dc = synth.make_decode(len(lens), 16, 1, 128, lens, 77, 0.5)
    q, k, v = dev(dc.q_raw, "bf16"), dev(dc.k_raw, "bf16"), dev(dc.v_raw, "bf16")
    bad = torch.tensor([0, 100, 50, 300], dtype=torch.int64, device="cuda")   # request 1 ends before it starts
    out = torch.empty((3, 16, 128), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(B.cp_workspace_size(B.CP_OP_DECODE, 3, 16, 128, 16), dtype=torch.uint8, device="cuda")
    B.cp_decode(q, k, v, bad, 16, 1, 16, 1 / math.sqrt(128), out, None, ws)
    torch.cuda.synchronize()
    with pytest.raises(B.CpError) as e:
        B.cp_check_status(ws)
    assert e.value.code == B.CP_ERR_INTERNAL


# ---------------------------------------------------------------------------- decode partials, CP decode, graphs
def _decode_case(lens, n_h, n_kv, seed):
    dc = synth.make_decode(len(lens), n_h, n_kv, 128, lens, seed, 0.5)
    return dc, dev(dc.q_raw, "bf16"), dev(dc.k_raw, "bf16"), dev(dc.v_raw, "bf16"), torch.from_numpy(dc.offsets).cuda()


@pytest.mark.parametrize("n_h,n_kv,d", [(16, 2, 128), (32, 1, 64)])
def test_decode_partial_matches_oracle(n_h, n_kv, d):
    lens = [0, 7, 129, 2000, 64]
    dc = synth.make_decode(len(lens), n_h, n_kv, d, lens, 61 + d, 0.5)
    q, k, v = dev(dc.q_raw, "bf16"), dev(dc.k_raw, "bf16"), dev(dc.v_raw, "bf16")
    off = torch.from_numpy(dc.offsets).cuda()
    o = torch.empty((len(lens), n_h, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((len(lens), n_h), dtype=torch.float32, device="cuda")
    ws = torch.zeros(B.cp_workspace_size(B.CP_OP_DECODE, len(lens), n_h, d, 32), dtype=torch.uint8, device="cuda")
    B.cp_decode_partial(q, k, v, off, n_h, n_kv, 32, 1 / math.sqrt(d), o, lse, ws)
    B.cp_check_status(ws)
    o_ref, l_ref = OD.decode(dc.q, dc.k, dc.v, dc.offsets)
    check(o.cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, "bf16", "decode partial")


@pytest.mark.parametrize("n_ranks,mode", [(2, B.CP_SHARD_LOAD_BALANCED), (4, B.CP_SHARD_LOAD_BALANCED),
                                          (8, B.CP_SHARD_CONTIGUOUS), (8, B.CP_SHARD_LOAD_BALANCED)])
def test_decode_context_parallel(n_ranks, mode):
    """Every rank decodes every query against its shard of the cache; the merged
    partials equal the decode of the whole cache."""
    lens = [0, 5, 100, 255, 256, 1000, 3001, 64, 17]
    dc, q, k, v, off = _decode_case(lens, 16, 1, 70 + n_ranks)
    cp = ring.DecodeCP(k, v, dc.offsets, n_ranks, mode)
    o_parts, lse_parts, ws = cp.buffers(q, 16)
    q_ranks = q.repeat(n_ranks, 1, 1)
    out = torch.empty((len(lens), 16, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((len(lens), 16), dtype=torch.float32, device="cuda")
    cp.run(q_ranks, 1, 16, 1 / math.sqrt(128), out, lse, o_parts, lse_parts, ws)
    B.cp_check_status(ws)
    o_ref, l_ref = OD.decode(dc.q, dc.k, dc.v, dc.offsets)
    check(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, "bf16", "cp decode")


def test_decode_replays_from_a_cuda_graph():
    """cp_decode captured once (after one eager call) and replayed on new
    inputs copied into the captured buffers gives the eager results."""
    lens = [300, 4096, 77, 1500]
    dc, q, k, v, off = _decode_case(lens, 16, 1, 81)
    dc2, q2, k2, v2, _ = _decode_case(lens, 16, 1, 82)
    out = torch.empty((4, 16, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((4, 16), dtype=torch.float32, device="cuda")
    ws = torch.zeros(B.cp_workspace_size(B.CP_OP_DECODE, 4, 16, 128, 64), dtype=torch.uint8, device="cuda")
    scale = 1 / math.sqrt(128)
    B.cp_decode(q, k, v, off, 16, 1, 64, scale, out, lse, ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        B.cp_decode(q, k, v, off, 16, 1, 64, scale, out, lse, ws)
    g.replay()
    torch.cuda.synchronize()
    o_ref, l_ref = OD.decode(dc.q, dc.k, dc.v, dc.offsets)
    check(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, "bf16", "graph replay")
    q.copy_(q2), k.copy_(k2), v.copy_(v2)
    g.replay()
    torch.cuda.synchronize()
    B.cp_check_status(ws)
    o_ref2, l_ref2 = OD.decode(dc2.q, dc2.k, dc2.v, dc2.offsets)
    check(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref2, l_ref2, "bf16", "graph replay, new inputs")


# ---------------------------------------------------------------------------- merge fused into the partial epilogue
@pytest.mark.parametrize("t,n_h,n_kv,n_ranks,variant,p", [
    (1000, 16, 1, 3, B.CP_PASS_KV, 0),
    (777, 8, 2, 4, B.CP_PASS_Q, 0),
    (300, 32, 2, 4, B.CP_PASS_Q, 1500),
    (300, 16, 1, 1, B.CP_PASS_KV, 0),
])
def test_bf16_ring_fused_merge(t, n_h, n_kv, n_ranks, variant, p):
    """The ring with the LSE merge in the partial kernel's epilogue (one running
    buffer, the last step writes bf16 out) equals unsharded attention."""
    pr = synth.make_prefill(t, n_h, n_kv, 128, "bf16", 200 + t, 0.5, p=p)
    _run_prefill(pr, n_ranks, variant, B.CP_SHARD_LOAD_BALANCED, merge="fused")


@pytest.mark.parametrize("t,n_h,n_kv,n_ranks,variant,p,d", [
    (1000, 16, 1, 3, B.CP_PASS_KV, 0, 128),
    (300, 32, 2, 4, B.CP_PASS_Q, 1500, 128),
    (777, 8, 2, 2, B.CP_PASS_KV, 0, 64),
])
def test_bf16_ring_bf16_partials(t, n_h, n_kv, n_ranks, variant, p, d):
    """The ring with bf16 partial O buffers (cp_attn_partial_bf16_parts, then
    cp_attn_merge_bf16_parts) equals unsharded attention within the bf16
    tolerances, on diffuse and on peaked queries."""
    pr = synth.make_prefill(t, n_h, n_kv, d, "bf16", 250 + t, 0.5, p=p)
    _run_prefill(pr, n_ranks, variant, B.CP_SHARD_LOAD_BALANCED, merge="final_bf16")
    _run_prefill(pr, n_ranks, variant, B.CP_SHARD_LOAD_BALANCED, merge="final_bf16", q_scale=8.0)


@pytest.mark.parametrize("n_parts,out_dtype", [(2, "bf16"), (8, "f32"), (5, "bf16")])
def test_merge_bf16_parts(n_parts, out_dtype):
    """cp_attn_merge_bf16_parts on bf16 partials against the reference merge of
    the same (rounded) values; -inf parts hold NaN and must not leak."""
    rng = np.random.default_rng(200 + n_parts)
    rows, n_h, d = 41, 4, 128
    o = rng.standard_normal((n_parts, rows, n_h, d)).astype(np.float32)
    lse = (rng.standard_normal((n_parts, rows, n_h)) * 3).astype(np.float32)
    lse[rng.random(lse.shape) < 0.2] = -np.inf
    o_bits = synth.bf16_bits(o)
    o_vals = synth.bf16_bits_to_f32(o_bits)
    o_ref, l_ref = OA.merge(list(np.where(np.isinf(lse)[..., None], 0.0, o_vals)), list(lse))
    o_bits = np.where(np.isinf(lse)[..., None], np.uint16(0x7FC0), o_bits).astype(np.uint16)   # NaN in -inf parts
    out = torch.empty((rows, n_h, d), dtype=torch.bfloat16 if out_dtype == "bf16" else torch.float32, device="cuda")
    lse_out = torch.empty((rows, n_h), dtype=torch.float32, device="cuda")
    B.cp_attn_merge(dev(o_bits, "bf16"), dev(lse, "f32"), n_parts, rows, rows, n_h, d, out, lse_out)
    torch.cuda.synchronize()
    check(out.float().cpu().numpy(), lse_out.cpu().numpy(), o_ref, l_ref, out_dtype, "merge of bf16 parts")


def test_bf16_varlen_fused_merge():
    lens = [700, 129, 1000]
    segs, r0 = [], 0
    for i, n in enumerate(lens):
        segs.append(ring.Segment(n, r0, 0, i))
        r0 += n
    pr = synth.make_prefill(sum(lens), 16, 2, 128, "bf16", 6, 0.5)
    _run_prefill(pr, 3, B.CP_PASS_KV, B.CP_SHARD_LOAD_BALANCED, merge="fused", segs=segs)


def test_fused_rejects_overlapping_rows_and_fp32():
    rng = np.random.default_rng(8)
    q = dev(synth.bf16_bits(rng.standard_normal((64, 16, 128)).astype(np.float32)), "bf16")
    k = dev(synth.bf16_bits(rng.standard_normal((64, 1, 128)).astype(np.float32)), "bf16")
    o = torch.zeros((64, 16, 128), device="cuda")
    lse = torch.zeros((64, 16), device="cuda")
    ranges = (B.cp_range * 2)(B.cp_range(0, 0, 64, 0, 0), B.cp_range(0, 0, 64, 0, 0))
    blocks = (B.cp_block * 2)(B.cp_block(0, 1, 1, 1, 0), B.cp_block(0, 1, 1, 1, 0))   # same rows twice
    with pytest.raises(B.CpError) as e:
        B.cp_attn_partial_fused(q, k, k, 16, 1, 0.1, True, ranges, 2, blocks, 2, o, lse, True, None, _ws())
    assert e.value.code == B.CP_ERR_INVALID_ARG
    qf = torch.zeros((64, 16, 64), device="cuda")
    kf = torch.zeros((64, 1, 64), device="cuda")
    with pytest.raises(B.CpError) as e:
        B.cp_attn_partial_fused(qf, kf, kf, 16, 1, 0.1, True, ranges, 2, blocks, 1, o, lse, True, None, _ws())
    assert e.value.code == B.CP_ERR_UNSUPPORTED


# ---------------------------------------------------------------------------- degenerate shapes
@pytest.mark.parametrize("t,n_ranks,variant,merge", [
    (5, 4, B.CP_PASS_KV, "final"),     # 8 chunks for 5 tokens: most shards empty
    (1, 2, B.CP_PASS_Q, "final"),      # one token
    (3, 8, B.CP_PASS_KV, "fused"),
    (7, 3, B.CP_PASS_Q, "running"),
])
def test_bf16_ring_fewer_tokens_than_chunks(t, n_ranks, variant, merge):
    pr = synth.make_prefill(t, 16, 1, 128, "bf16", 300 + t, 0.5)
    _run_prefill(pr, n_ranks, variant, B.CP_SHARD_LOAD_BALANCED, merge=merge)


def test_fp32_ring_fewer_tokens_than_chunks():
    pr = synth.make_prefill(3, 4, 1, 64, "f32", 9, 1.0)
    _run_prefill(pr, 4, B.CP_PASS_KV, B.CP_SHARD_LOAD_BALANCED)


def test_decode_all_requests_empty():
    lens = [0, 0, 0]
    dc = synth.make_decode(len(lens), 16, 1, 128, lens, 90, 0.5)
    q = dev(dc.q_raw, "bf16")
    k = torch.zeros((1, 1, 128), dtype=torch.bfloat16, device="cuda")
    off = torch.from_numpy(dc.offsets).cuda()
    out = torch.full((3, 16, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((3, 16), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.zeros(B.cp_workspace_size(B.CP_OP_DECODE, 3, 16, 128, 8), dtype=torch.uint8, device="cuda")
    B.cp_decode(q, k, k, off, 16, 1, 8, 1 / math.sqrt(128), out, lse, ws)
    B.cp_check_status(ws)
    assert torch.all(out.float() == 0) and torch.all(torch.isneginf(lse))


# ---------------------------------------------------------------------------- running-max growth
@pytest.mark.parametrize("c,variant", [(4.0, B.CP_PASS_KV), (12.0, B.CP_PASS_KV), (12.0, B.CP_PASS_Q),
                                       (16.0, B.CP_PASS_KV)])
def test_bf16_score_jumps(c, variant):
    """Queries share a common direction and a few keys point along it with
    growing magnitude, so a row's max jumps by about 8c log2 units between KV
    tiles: c = 4 exercises the deferred move to a new reference (growth past
    2^8), c >= 12 the repeated step (growth past 2^64)."""
    rng = np.random.default_rng(int(c * 10) + variant)
    t, n_h, n_kv, d = 1100, 16, 1, 128
    q = (0.5 + 0.1 * rng.standard_normal((t, n_h, d))).astype(np.float32)
    k = (0.5 * rng.standard_normal((t, n_kv, d))).astype(np.float32)
    v = rng.standard_normal((t, n_kv, d)).astype(np.float32)
    for pos, mult in ((300, 0.5), (650, 1.0), (900, 1.5)):
        k[pos] = c * mult
    q_raw, k_raw, v_raw = synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v)
    qd, kd, vd = dev(q_raw, "bf16"), dev(k_raw, "bf16"), dev(v_raw, "bf16")
    segs = [ring.Segment(t, 0, 0, 0)]
    sched = ring.RingSchedule(segs, segs, 2, variant)
    out = torch.empty((t, n_h, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((t, n_h), dtype=torch.float32, device="cuda")
    ws = _ws()
    ring.run_ring(sched, qd, kd, vd, n_h, n_kv, out, lse, workspace=ws)
    torch.cuda.synchronize()
    B.cp_check_status(ws)
    qv, kv_, vv = (synth.bf16_bits_to_f32(x) for x in (q_raw, k_raw, v_raw))
    o_ref, l_ref = OA.attention(qv, kv_, vv, np.arange(t), np.arange(t))
    check(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, "bf16", f"jumps c={c}")


# ---------------------------------------------------------------------------- bounded waits
def test_bounded_wait_reports_timeout_and_context_survives():
    """A device-side wait on a barrier nothing completes gives up after its
    budget and records CP_ERR_TIMEOUT; nothing faults, and the same context
    then runs a decode correctly."""
    ws = _ws()
    B.cp_wait_selftest(ws, 20_000_000)   # 20 ms
    torch.cuda.synchronize()
    with pytest.raises(B.CpError) as e:
        B.cp_check_status(ws)
    assert e.value.code == B.CP_ERR_TIMEOUT
    B.cp_reset_status(ws)
    B.cp_check_status(ws)
    lens = [100, 37]
    dc, q, k, v, off = _decode_case(lens, 16, 1, 95)
    out = torch.empty((2, 16, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((2, 16), dtype=torch.float32, device="cuda")
    dws = torch.zeros(B.cp_workspace_size(B.CP_OP_DECODE, 2, 16, 128, 4), dtype=torch.uint8, device="cuda")
    B.cp_decode(q, k, v, off, 16, 1, 4, 1 / math.sqrt(128), out, lse, dws)
    B.cp_check_status(dws)
    o_ref, l_ref = OD.decode(dc.q, dc.k, dc.v, dc.offsets)
    check(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, "bf16", "after timeout")


# ---------------------------------------------------------------------------- canaries after the outputs
GUARD = 96   # rows of NaN after every output; no kernel may touch them


def _guarded(shape, dtype):
    t = torch.full((shape[0] + GUARD,) + tuple(shape[1:]), float("nan"), dtype=dtype, device="cuda")
    return t, t[:shape[0]]


def _guard_intact(t, rows):
    return bool(torch.isnan(t[rows:].float()).all())


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_outputs_leave_guard_rows_untouched(dtype):
    t, n_h, n_kv, d = 700, 16, 2, (128 if dtype == "bf16" else 64)
    pr = synth.make_prefill(t, n_h, n_kv, d, dtype, 500, 0.5)
    q_raw = pr.q_raw if dtype == "bf16" else pr.q.astype(np.float32)
    q, k, v = dev(q_raw, dtype), dev(pr.k_raw, dtype), dev(pr.v_raw, dtype)
    segs = [ring.Segment(t, 0, 0, 0)]
    sched = ring.RingSchedule(segs, segs, 3, B.CP_PASS_KV)
    o_full, o_parts = _guarded((3 * t, n_h, d), torch.float32)
    l_full, l_parts = _guarded((3 * t, n_h), torch.float32)
    out_dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out_full, out = _guarded((t, n_h, d), out_dt)
    lse_full, lse = _guarded((t, n_h), torch.float32)
    ws = _ws()
    ring.run_ring(sched, q, k, v, n_h, n_kv, out, lse, o_parts=o_parts, lse_parts=l_parts, workspace=ws)
    torch.cuda.synchronize()
    B.cp_check_status(ws)
    for full, rows in ((o_full, 3 * t), (l_full, 3 * t), (out_full, t), (lse_full, t)):
        assert _guard_intact(full, rows)
    assert torch.isfinite(out.float()).all()


def test_decode_leaves_guard_rows_untouched():
    lens = [0, 300, 5000, 77]
    dc, q, k, v, off = _decode_case(lens, 16, 1, 97)
    out_full, out = _guarded((4, 16, 128), torch.bfloat16)
    lse_full, lse = _guarded((4, 16), torch.float32)
    o_full, o_part = _guarded((4, 16, 128), torch.float32)
    lp_full, l_part = _guarded((4, 16), torch.float32)
    ws = torch.zeros(B.cp_workspace_size(B.CP_OP_DECODE, 4, 16, 128, 64), dtype=torch.uint8, device="cuda")
    B.cp_decode(q, k, v, off, 16, 1, 64, 1 / math.sqrt(128), out, lse, ws)
    B.cp_decode_partial(q, k, v, off, 16, 1, 64, 1 / math.sqrt(128), o_part, l_part, ws)
    torch.cuda.synchronize()
    B.cp_check_status(ws)
    for full, rows in ((out_full, 4), (lse_full, 4), (o_full, 4), (lp_full, 4)):
        assert _guard_intact(full, rows)


@pytest.mark.parametrize("t,n_h,n_kv,variant", [
    (301, 32, 1, B.CP_PASS_KV),     # G = 32: 8 tokens per CTA tile
    (129, 64, 1, B.CP_PASS_Q),      # G = 64
    (77, 128, 1, B.CP_PASS_KV),     # G = 128: 2 tokens per CTA, one row per (token, head)
    (150, 128, 2, B.CP_PASS_Q),     # G = 64 on two KV heads
])
def test_bf16_ring_large_gqa_groups(t, n_h, n_kv, variant):
    pr = synth.make_prefill(t, n_h, n_kv, 128, "bf16", 600 + t, 0.5)
    _run_prefill(pr, 2, variant, B.CP_SHARD_LOAD_BALANCED)
