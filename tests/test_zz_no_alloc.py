"""cp_decode_static: split-KV decode for callers that cannot allocate device
memory when they decode (code inside an allocator or memory pool, plugins that
only receive their inputs and outputs, serving loops that forbid allocation
after start-up). It must give the results of cp_decode, which takes a
caller-allocated workspace, and of the fp64 reference, including on
back-to-back calls that reuse the library's fixed scratch array; it must check
every argument before it enqueues anything, and report device-side failures
through cp_decode_static_status.

This file is collected last so that a run stopping at the first failure has
already run every other test."""
import math

import numpy as np
import pytest
import torch

from context_ring_attn_b200 import binding as B
from context_ring_attn_b200 import synth
from oracle import decode as OD

pytestmark = pytest.mark.gpu

TOL_MAX, TOL_MEAN, TOL_LSE = 2e-2, 2e-3, 1e-3   # the bf16 tolerances of the other tests


def _bf16(raw):
    return torch.from_numpy(np.ascontiguousarray(raw).view(np.int16)).view(torch.bfloat16).cuda()


def _case(seed, lens, n_h=16, n_kv=1, d=128):
    dc = synth.make_decode(len(lens), n_h, n_kv, d, lens, seed, 0.5)
    return dc, (_bf16(dc.q_raw), _bf16(dc.k_raw), _bf16(dc.v_raw), torch.from_numpy(dc.offsets).cuda(), n_h, n_kv)


def _with_workspace(q, k, v, off, n_h, n_kv, n_splits):
    d = q.shape[-1]
    out = torch.empty((q.shape[0], n_h, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((q.shape[0], n_h), dtype=torch.float32, device="cuda")
    ws = torch.zeros(B.cp_workspace_size(B.CP_OP_DECODE, q.shape[0], n_h, d, n_splits), dtype=torch.uint8,
                     device="cuda")
    B.cp_decode(q, k, v, off, n_h, n_kv, n_splits, 1 / math.sqrt(d), out, lse, ws)
    B.cp_check_status(ws)
    return out, lse


def _static(q, k, v, off, n_h, n_kv, n_splits):
    d = q.shape[-1]
    out = torch.full((q.shape[0], n_h, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((q.shape[0], n_h), float("nan"), dtype=torch.float32, device="cuda")
    B.cp_decode_static(q, k, v, off, n_h, n_kv, n_splits, 1 / math.sqrt(d), out, lse)
    B.cp_decode_static_status()
    return out, lse


def _close(a, b):
    (oa, la), (ob, lb) = a, b
    oa, ob = torch.as_tensor(oa).double().cpu(), torch.as_tensor(ob).double().cpu()
    la, lb = torch.as_tensor(la).double().cpu(), torch.as_tensor(lb).double().cpu()
    err = (oa - ob).abs()
    assert torch.isfinite(oa).all()
    assert err.max().item() <= TOL_MAX and err.mean().item() <= TOL_MEAN, (err.max().item(), err.mean().item())
    fin = torch.isfinite(lb)
    assert torch.equal(torch.isfinite(la), fin)
    if fin.any():
        assert (la[fin] - lb[fin]).abs().max().item() <= TOL_LSE


def _oracle(dc):
    return OD.decode(dc.q, dc.k, dc.v, dc.offsets)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    B.lib()


def test_matches_workspace_decode_and_reference_on_two_calls_in_a_row():
    n_splits = 64
    dc1, first = _case(71, [300, 5000, 77, 12000, 1, 2048])
    dc2, second = _case(72, [9000, 0, 640, 33], n_h=16, n_kv=2)   # different shapes: nothing stale may leak
    ref1 = _with_workspace(*first, n_splits)
    ref2 = _with_workspace(*second, n_splits)
    got1 = _static(*first, n_splits)
    got2 = _static(*second, n_splits)
    _close(got1, ref1)
    _close(got2, ref2)
    _close(got1, _oracle(dc1))
    _close(got2, _oracle(dc2))


@pytest.mark.parametrize("n_h,n_kv,d", [(64, 2, 128), (16, 1, 64), (128, 1, 64)])
def test_other_head_shapes(n_h, n_kv, d):
    """Groups above 16 heads (several 16-head units per KV head) and d = 64."""
    dc, case = _case(80 + n_h + d, [700, 3, 4100], n_h=n_h, n_kv=n_kv, d=d)
    got = _static(*case, 32)
    _close(got, _with_workspace(*case, 32))
    _close(got, _oracle(dc))


def test_reports_bad_offsets_and_checks_arguments_before_enqueueing():
    dc, (q, k, v, off, n_h, n_kv) = _case(74, [100, 60, 140])
    out = torch.empty((3, n_h, 128), dtype=torch.bfloat16, device="cuda")
    bad = torch.tensor([0, 100, 50, 300], dtype=torch.int64, device="cuda")   # request 1 ends before it starts
    B.cp_decode_static(q, k, v, bad, n_h, n_kv, 16, 1 / math.sqrt(128), out, None)
    with pytest.raises(B.CpError) as e:
        B.cp_decode_static_status()
    assert e.value.code == B.CP_ERR_INTERNAL
    # An invalid call returns its error without enqueueing anything: the status
    # word (cleared at the start of every accepted call) still holds the failure.
    q64 = torch.zeros((3, n_h, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B.CpError) as e:
        B.cp_decode_static(q64, k, v, off, n_h, n_kv, 16, 0.1, out, None)
    assert e.value.code == B.CP_ERR_UNSUPPORTED
    with pytest.raises(B.CpError) as e:
        B.cp_decode_static_status()
    assert e.value.code == B.CP_ERR_INTERNAL
    # the next valid call clears it and decodes correctly
    lse = torch.empty((3, n_h), dtype=torch.float32, device="cuda")
    B.cp_decode_static(q, k, v, off, n_h, n_kv, 16, 1 / math.sqrt(128), out, lse)
    B.cp_decode_static_status()
    _close((out, lse), _oracle(dc))


def test_rejects_requests_beyond_the_scratch_limit():
    dc, (q, k, v, off, n_h, n_kv) = _case(73, [64, 64])
    out = torch.empty((2, n_h, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((2, n_h), dtype=torch.float32, device="cuda")
    # 2 requests fit; 5000 requests do not: (8 x 148 ranges + 5000 pairs) x 16 heads x 129 floats > 32 MiB
    big_q = torch.zeros((5000, n_h, 128), dtype=torch.bfloat16, device="cuda")
    big_off = torch.zeros(5001, dtype=torch.int64, device="cuda")
    big_out = torch.empty((5000, n_h, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B.CpError) as e:
        B.cp_decode_static(big_q, k, v, big_off, n_h, n_kv, 1024, 0.1, big_out, None)
    assert e.value.code == B.CP_ERR_WORKSPACE
    B.cp_decode_static(q, k, v, off, n_h, n_kv, 1024, 1 / math.sqrt(128), out, lse)
    B.cp_decode_static_status()
    _close((out, lse), _with_workspace(q, k, v, off, n_h, n_kv, 1024))
    _close((out, lse), _oracle(dc))
