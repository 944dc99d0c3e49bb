"""cp_decode_static: split-KV decode for callers that cannot allocate device
memory when they decode (code inside an allocator or memory pool, plugins that
only receive their inputs and outputs, serving loops that forbid allocation
after start-up). It must give the same results as cp_decode, which takes a
caller-allocated workspace, including on back-to-back calls that reuse the
library's fixed scratch array.

This file is collected last so that a run stopping at the first failure has
already run every other test."""
import math

import numpy as np
import pytest
import torch

from context_ring_attn_b200 import binding as B
from context_ring_attn_b200 import synth

pytestmark = pytest.mark.gpu

TOL_MAX, TOL_MEAN, TOL_LSE = 2e-2, 2e-3, 1e-3   # the bf16 tolerances of the other tests


def _bf16(raw):
    return torch.from_numpy(np.ascontiguousarray(raw).view(np.int16)).view(torch.bfloat16).cuda()


def _case(seed, lens, n_h=16, n_kv=1):
    dc = synth.make_decode(len(lens), n_h, n_kv, 128, lens, seed, 0.5)
    return (_bf16(dc.q_raw), _bf16(dc.k_raw), _bf16(dc.v_raw), torch.from_numpy(dc.offsets).cuda(), n_h, n_kv)


def _with_workspace(q, k, v, off, n_h, n_kv, n_splits):
    out = torch.empty((q.shape[0], n_h, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((q.shape[0], n_h), dtype=torch.float32, device="cuda")
    ws = torch.zeros(B.cp_workspace_size(B.CP_OP_DECODE, q.shape[0], n_h, 128, n_splits), dtype=torch.uint8,
                     device="cuda")
    B.cp_decode(q, k, v, off, n_h, n_kv, n_splits, 1 / math.sqrt(128), out, lse, ws)
    B.cp_check_status(ws)
    return out, lse


def _static(q, k, v, off, n_h, n_kv, n_splits):
    out = torch.full((q.shape[0], n_h, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((q.shape[0], n_h), float("nan"), dtype=torch.float32, device="cuda")
    B.cp_decode_static(q, k, v, off, n_h, n_kv, n_splits, 1 / math.sqrt(128), out, lse)
    torch.cuda.synchronize()
    return out, lse


def _close(a, b):
    (oa, la), (ob, lb) = a, b
    err = (oa.float() - ob.float()).abs()
    assert torch.isfinite(oa.float()).all()
    assert err.max().item() <= TOL_MAX and err.mean().item() <= TOL_MEAN
    fin = torch.isfinite(lb)
    assert torch.equal(torch.isfinite(la), fin)
    assert (la[fin] - lb[fin]).abs().max().item() <= TOL_LSE


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    B.lib()


def test_matches_workspace_decode_on_two_calls_in_a_row():
    n_splits = 64
    first = _case(71, [300, 5000, 77, 12000, 1, 2048])
    second = _case(72, [9000, 0, 640, 33], n_h=16, n_kv=2)   # different shapes: nothing stale may leak
    ref1 = _with_workspace(*first, n_splits)
    ref2 = _with_workspace(*second, n_splits)
    _close(_static(*first, n_splits), ref1)
    _close(_static(*second, n_splits), ref2)


def test_rejects_requests_beyond_the_scratch_limit():
    q, k, v, off, n_h, n_kv = _case(73, [64, 64])
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
    torch.cuda.synchronize()
    _close((out, lse), _with_workspace(q, k, v, off, n_h, n_kv, 1024))
