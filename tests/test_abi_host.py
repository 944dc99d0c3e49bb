"""The C ABI on the host: the library loads, exports every symbol the header
declares, and rejects bad arguments before touching the GPU."""
import ctypes
import os
import re

import pytest

from context_ring_attn_b200 import binding as B
from context_ring_attn_b200 import build as BUILD

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    BUILD.build()
    return B.lib()


def header_functions():
    src = open(os.path.join(ROOT, "include", "cp_attn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(cp_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = header_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(L, n), n
    assert sorted(B.EXPORTED) == names


def test_version_and_strings(L):
    assert B.cp_abi_version() == 2
    for code in range(7):
        assert B.status_string(code)
    assert "unknown" in B.status_string(99)


def test_struct_sizes():
    assert ctypes.sizeof(B.cp_range) == 32
    assert ctypes.sizeof(B.cp_block) == 24
    assert ctypes.sizeof(B.cp_segment) == 32


def test_workspace_sizes(L):
    assert B.cp_workspace_size(B.CP_OP_PARTIAL, 0, 16, 128, 1) == 256
    assert B.cp_workspace_size(B.CP_OP_MERGE, 10, 16, 128, 1) == 256
    ws = B.cp_workspace_size(B.CP_OP_DECODE, 32, 16, 128, 256)
    # bound on the partial rows: (n_splits + 1) * batch * n_h + 7 * n_h, d + 1 floats each
    assert ws % 256 == 0 and ws >= 256 + (257 * 32 * 16 + 7 * 16) * 129 * 4


FAKE = 1 << 20  # a 256-byte aligned non-null address that is never dereferenced


def _partial(L, **kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, dtype=B.CP_BF16, q_rows=256, kv_rows=256, n_h=16, n_kv=1, d=128,
                scale=0.1, causal=1, ranges=None, n_ranges=0, blocks=None, n_blocks=0, o=FAKE, lse=FAKE,
                out_rows=256, ws=FAKE, ws_bytes=256)
    args.update(kw)
    return L.cp_attn_partial(args["q"], args["k"], args["v"], args["dtype"], args["q_rows"], args["kv_rows"],
                             args["n_h"], args["n_kv"], args["d"], args["scale"], args["causal"], args["ranges"],
                             args["n_ranges"], args["blocks"], args["n_blocks"], args["o"], args["lse"],
                             args["out_rows"], args["ws"], args["ws_bytes"], None)


def _one_block(q_range, kv_range):
    ranges = (B.cp_range * 2)(q_range, kv_range)
    blocks = (B.cp_block * 1)(B.cp_block(0, 1, 1, 1, 0))
    return ranges, blocks


def test_partial_rejects_bad_arguments(L):
    assert _partial(L, q=None) == B.CP_ERR_INVALID_ARG
    assert _partial(L, n_h=15, n_kv=2) == B.CP_ERR_INVALID_ARG
    assert _partial(L, scale=0.0) == B.CP_ERR_INVALID_ARG
    assert _partial(L, ws=None) == B.CP_ERR_WORKSPACE
    assert _partial(L, ws_bytes=16) == B.CP_ERR_WORKSPACE
    assert _partial(L, ws=FAKE + 8) == B.CP_ERR_WORKSPACE
    assert _partial(L, d=96) == B.CP_ERR_UNSUPPORTED
    assert _partial(L, n_h=24, n_kv=1) == B.CP_ERR_UNSUPPORTED       # group 24 not a power of two
    assert _partial(L, dtype=B.CP_F32, d=96) == B.CP_ERR_UNSUPPORTED
    assert _partial(L, dtype=7) == B.CP_ERR_UNSUPPORTED
    assert _partial(L, q=FAKE + 2) == B.CP_ERR_INVALID_ARG            # misaligned bf16 operand
    ranges, blocks = _one_block(B.cp_range(200, 200, 100, 0, 0), B.cp_range(0, 0, 10, 0, 0))
    assert _partial(L, ranges=ranges, n_ranges=2, blocks=blocks, n_blocks=1) == B.CP_ERR_INVALID_ARG
    ranges, blocks = _one_block(B.cp_range(0, 0, 10, 0, 0), B.cp_range(250, 0, 10, 0, 0))
    assert _partial(L, ranges=ranges, n_ranges=2, blocks=blocks, n_blocks=1) == B.CP_ERR_INVALID_ARG
    ranges, blocks = _one_block(B.cp_range(0, 0, 10, 0, 1), B.cp_range(0, 0, 10, 0, 0))  # reserved != 0
    assert _partial(L, ranges=ranges, n_ranges=2, blocks=blocks, n_blocks=1) == B.CP_ERR_INVALID_ARG
    ranges, blocks = _one_block(B.cp_range(0, 0, 10, 0, 0), B.cp_range(0, 0, 10, 0, 0))
    assert _partial(L, ranges=ranges, n_ranges=1, blocks=blocks, n_blocks=1) == B.CP_ERR_INVALID_ARG
    assert _partial(L, ranges=ranges, n_ranges=2, blocks=blocks, n_blocks=1, out_rows=5) == B.CP_ERR_INVALID_ARG


def test_merge_and_decode_reject_bad_arguments(L):
    assert L.cp_attn_merge(None, FAKE, 2, 10, 10, 4, 128, FAKE, B.CP_F32, None, None) == B.CP_ERR_INVALID_ARG
    assert L.cp_attn_merge(FAKE, FAKE, 0, 10, 10, 4, 128, FAKE, B.CP_F32, None, None) == B.CP_ERR_INVALID_ARG
    assert L.cp_attn_merge(FAKE, FAKE, 2, 5, 10, 4, 128, FAKE, B.CP_F32, None, None) == B.CP_ERR_INVALID_ARG
    assert L.cp_attn_merge(FAKE, FAKE, 2, 10, 10, 4, 126, FAKE, B.CP_F32, None, None) == B.CP_ERR_INVALID_ARG
    assert L.cp_attn_merge(FAKE + 4, FAKE, 2, 10, 10, 4, 128, FAKE, B.CP_F32, None, None) == B.CP_ERR_INVALID_ARG
    assert L.cp_attn_merge(FAKE, FAKE, 2, 10, 10, 4, 128, FAKE, 5, None, None) == B.CP_ERR_UNSUPPORTED

    def dec(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, dtype=B.CP_BF16, off=FAKE, batch=4, kv_rows=100, n_h=16, n_kv=1, d=128,
                 splits=256, scale=0.1, out=FAKE, lse=FAKE, ws=FAKE, ws_bytes=1 << 30)
        a.update(kw)
        return L.cp_decode(a["q"], a["k"], a["v"], a["dtype"], a["off"], a["batch"], a["kv_rows"], a["n_h"],
                           a["n_kv"], a["d"], a["splits"], a["scale"], a["out"], a["lse"], a["ws"],
                           a["ws_bytes"], None)
    assert dec(off=None) == B.CP_ERR_INVALID_ARG
    assert dec(splits=0) == B.CP_ERR_UNSUPPORTED
    assert dec(splits=5000) == B.CP_ERR_UNSUPPORTED
    assert dec(n_h=40, n_kv=1) == B.CP_ERR_UNSUPPORTED   # a group above 16 must be a multiple of 16
    assert dec(n_h=256, n_kv=1) == B.CP_ERR_UNSUPPORTED  # groups above 128
    assert dec(d=96) == B.CP_ERR_UNSUPPORTED
    assert dec(dtype=B.CP_F32) == B.CP_ERR_UNSUPPORTED
    assert dec(ws_bytes=1024) == B.CP_ERR_WORKSPACE
    assert dec(ws=None) == B.CP_ERR_WORKSPACE
    assert dec(k=FAKE + 8) == B.CP_ERR_INVALID_ARG


def test_planning_rejects_bad_arguments(L):
    segs = B.segments([(10, 0, 0, 0)])
    n = ctypes.c_int32(0)
    out = (B.cp_range * 4)()
    assert L.cp_rank_ranges(segs, 1, 0, 0, 0, out, ctypes.byref(n)) == B.CP_ERR_INVALID_ARG
    assert L.cp_rank_ranges(segs, 1, 2, 0, 2, out, ctypes.byref(n)) == B.CP_ERR_INVALID_ARG
    assert L.cp_rank_ranges(segs, 1, 2, 9, 0, out, ctypes.byref(n)) == B.CP_ERR_INVALID_ARG
    bad = B.segments([(-1, 0, 0, 0)])
    assert L.cp_shard_plan(bad, 1, 2, 0, None, None, None, None) == B.CP_ERR_INVALID_ARG
    ranges = (B.cp_range * 2)()
    blocks = (B.cp_block * 4)()
    assert L.cp_ring_schedule(segs, 1, segs, 1, 2, 0, 0, ranges, 2, ctypes.byref(n), blocks, None) == \
        B.CP_ERR_INVALID_ARG   # needs 8 ranges, capacity 2
    assert L.cp_ring_schedule(segs, 1, segs, 1, 2, 0, 3, ranges, 2, ctypes.byref(n), blocks, None) == \
        B.CP_ERR_INVALID_ARG


def test_wait_selftest_rejects_bad_arguments(L):
    """Checked on the host before any launch."""
    assert L.cp_wait_selftest(None, 256, 1000, None) == B.CP_ERR_WORKSPACE
    assert L.cp_wait_selftest(FAKE, 128, 1000, None) == B.CP_ERR_WORKSPACE
    assert L.cp_wait_selftest(FAKE, 256, 0, None) == B.CP_ERR_INVALID_ARG
    assert L.cp_wait_selftest(FAKE, 256, 2_000_000_000, None) == B.CP_ERR_INVALID_ARG


def test_decode_takes_every_listed_shape(L):
    """Head dims 64 and 128 and every GQA group up to 128 heads that the
    boundary lists get past the shape checks (the call then stops at the
    missing workspace, before any CUDA call)."""
    for d in (64, 128):
        for n_h, n_kv in ((16, 1), (16, 16), (12, 4), (8, 1), (32, 1), (64, 4), (128, 8), (128, 1), (64, 2)):
            for fn in ("cp_decode", "cp_decode_partial"):
                code = getattr(L, fn)(FAKE, FAKE, FAKE, B.CP_BF16, FAKE, 4, 100, n_h, n_kv, d, 256, 0.1, FAKE, FAKE,
                                      FAKE, 0, None)
                assert code == B.CP_ERR_WORKSPACE, (fn, d, n_h, n_kv, code)


def test_decode_static_checks_arguments_on_the_host(L):
    """Rejected before any CUDA call (this test runs without a GPU)."""
    def st(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, dtype=B.CP_BF16, off=FAKE, batch=4, kv_rows=100, n_h=16, n_kv=1, d=128,
                 splits=256, scale=0.1, out=FAKE, lse=FAKE)
        a.update(kw)
        return L.cp_decode_static(a["q"], a["k"], a["v"], a["dtype"], a["off"], a["batch"], a["kv_rows"], a["n_h"],
                                  a["n_kv"], a["d"], a["splits"], a["scale"], a["out"], a["lse"], None)
    assert st(q=None) == B.CP_ERR_INVALID_ARG
    assert st(d=96) == B.CP_ERR_UNSUPPORTED
    assert st(n_h=40) == B.CP_ERR_UNSUPPORTED
    assert st(splits=0) == B.CP_ERR_UNSUPPORTED
    assert st(scale=float("inf")) == B.CP_ERR_INVALID_ARG
    assert st(k=FAKE + 8) == B.CP_ERR_INVALID_ARG


def test_shard_plan_sizes_query(L):
    segs = B.segments([(10, 0, 0, 0), (7, 10, 0, 1)])
    sz = (ctypes.c_int64 * 3)()
    assert L.cp_shard_plan(segs, 2, 3, 0, None, None, None, sz) == B.CP_OK
    assert list(sz) == [2 * 7, 4, 17]


def test_partial_takes_every_listed_shape(L):
    """bf16 with D_H 64 or 128 and every power-of-two GQA group up to 128, and
    fp32 with D_H 64 or 128, get past every check (no block: nothing is
    launched)."""
    for d in (64, 128):
        for n_h, n_kv in ((16, 1), (16, 16), (8, 2), (32, 1), (64, 1), (128, 8), (128, 1)):
            assert _partial(L, d=d, n_h=n_h, n_kv=n_kv) == B.CP_OK, (d, n_h, n_kv)
        assert _partial(L, dtype=B.CP_F32, d=d, n_h=16, n_kv=1) == B.CP_OK
    assert _partial(L, d=96) == B.CP_ERR_UNSUPPORTED
    assert _partial(L, n_h=24, n_kv=2) == B.CP_ERR_UNSUPPORTED   # bf16 groups are powers of two
