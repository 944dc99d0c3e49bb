"""ctypes binding of libcpattn.so (include/cp_attn.h), one Python function per
C entry point with the same name. Argument marshalling only: device tensors
are passed by data pointer, the stream is torch's current stream, and every
non-OK status raises CpError. There is no fallback: if the shared library is
missing, the first call raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcpattn.so")

CP_OK = 0
CP_ERR_INVALID_ARG = 1
CP_ERR_UNSUPPORTED = 2
CP_ERR_WORKSPACE = 3
CP_ERR_CUDA = 4
CP_ERR_TIMEOUT = 5
CP_ERR_INTERNAL = 6

CP_F32 = 0
CP_BF16 = 1

CP_SHARD_LOAD_BALANCED = 0
CP_SHARD_CONTIGUOUS = 1

CP_PASS_KV = 0
CP_PASS_Q = 1

CP_PAIR_FULL = 0
CP_PAIR_PARTIAL = 1
CP_PAIR_SKIP = 2

CP_OP_PARTIAL = 0
CP_OP_DECODE = 1
CP_OP_MERGE = 2

EXPORTED = (
    "cp_status_string", "cp_abi_version", "cp_shard_plan", "cp_rank_ranges", "cp_ring_schedule",
    "cp_classify_pair", "cp_block_pairs", "cp_ring_comm_volume", "cp_workspace_size",
    "cp_reset_status", "cp_check_status", "cp_attn_partial", "cp_attn_merge", "cp_decode",
    "cp_decode_static", "cp_decode_partial", "cp_select_ring_variant", "cp_attn_partial_fused",
    "cp_wait_selftest", "cp_decode_static_status", "cp_attn_partial_bf16_parts", "cp_attn_merge_bf16_parts",
)


class CpError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn}: {status_string(code)} (status {code})")


class cp_segment(ctypes.Structure):
    _fields_ = [("len", ctypes.c_int64), ("row0", ctypes.c_int64), ("pos0", ctypes.c_int64),
                ("seq", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class cp_range(ctypes.Structure):
    _fields_ = [("row0", ctypes.c_int64), ("pos0", ctypes.c_int64), ("len", ctypes.c_int64),
                ("seq", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class cp_block(ctypes.Structure):
    _fields_ = [("q_begin", ctypes.c_int32), ("q_count", ctypes.c_int32), ("kv_begin", ctypes.c_int32),
                ("kv_count", ctypes.c_int32), ("out_row0", ctypes.c_int64)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load the shared library (once). Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m context_ring_attn_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    i32, i64, vp, f32, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_float, ctypes.c_size_t
    P = ctypes.POINTER
    sig = {
        "cp_status_string": (ctypes.c_char_p, [i32]),
        "cp_abi_version": (i32, []),
        "cp_shard_plan": (i32, [P(cp_segment), i32, i32, i32, P(i64), P(i64), P(i64), P(i64)]),
        "cp_rank_ranges": (i32, [P(cp_segment), i32, i32, i32, i32, P(cp_range), P(i32)]),
        "cp_ring_schedule": (i32, [P(cp_segment), i32, P(cp_segment), i32, i32, i32, i32, P(cp_range), i32,
                                   P(i32), P(cp_block), P(i32)]),
        "cp_classify_pair": (i32, [P(cp_range), P(cp_range), i32]),
        "cp_block_pairs": (i64, [P(cp_range), P(cp_block), i32]),
        "cp_ring_comm_volume": (i32, [P(cp_range), P(cp_block), i32, i32, i32, i32, i32, P(i64), P(i64), P(i64)]),
        "cp_workspace_size": (sz, [i32, i64, i32, i32, i32]),
        "cp_reset_status": (i32, [vp, vp]),
        "cp_check_status": (i32, [vp, vp]),
        "cp_attn_partial": (i32, [vp, vp, vp, i32, i64, i64, i32, i32, i32, f32, i32, P(cp_range), i32,
                                  P(cp_block), i32, vp, vp, i64, vp, sz, vp]),
        "cp_wait_selftest": (i32, [vp, sz, ctypes.c_uint64, vp]),
        "cp_attn_partial_fused": (i32, [vp, vp, vp, i32, i64, i64, i32, i32, i32, f32, i32, P(cp_range), i32,
                                        P(cp_block), i32, vp, vp, i64, i32, vp, vp, sz, vp]),
        "cp_attn_merge": (i32, [vp, vp, i32, i64, i64, i32, i32, vp, i32, vp, vp]),
        "cp_attn_merge_bf16_parts": (i32, [vp, vp, i32, i64, i64, i32, i32, vp, i32, vp, vp]),
        "cp_attn_partial_bf16_parts": (i32, [vp, vp, vp, i32, i64, i64, i32, i32, i32, f32, i32, P(cp_range), i32,
                                             P(cp_block), i32, vp, vp, i64, vp, sz, vp]),
        "cp_decode": (i32, [vp, vp, vp, i32, vp, i32, i64, i32, i32, i32, i32, f32, vp, vp, vp, sz, vp]),
        "cp_decode_static": (i32, [vp, vp, vp, i32, vp, i32, i64, i32, i32, i32, i32, f32, vp, vp, vp]),
        "cp_decode_static_status": (i32, [vp]),
        "cp_select_ring_variant": (i32, [i64, i64, i32, i32, i32, i32, i32, ctypes.c_double, ctypes.c_double,
                                          vp, vp]),
        "cp_decode_partial": (i32, [vp, vp, vp, i32, vp, i32, i64, i32, i32, i32, i32, f32, vp, vp, vp, sz, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def status_string(code: int) -> str:
    return lib().cp_status_string(int(code)).decode()


def _check(fn: str, code: int) -> None:
    if code != CP_OK:
        raise CpError(fn, code)


def _ptr(t) -> int | None:
    if t is None:
        return None
    return int(t.data_ptr())


def _stream(stream) -> int | None:
    """A raw cudaStream_t handle, or a torch.cuda.Stream; None: torch's current stream."""
    if stream is not None:
        return int(getattr(stream, "cuda_stream", stream))
    import torch
    return int(torch.cuda.current_stream().cuda_stream)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return CP_BF16
    if t.dtype == torch.float32:
        return CP_F32
    raise CpError("dtype", CP_ERR_UNSUPPORTED)


# ----------------------------------------------------------------------------- host planning
def segments(items) -> ctypes.Array:
    """Array of cp_segment from (len, row0, pos0, seq) tuples."""
    arr = (cp_segment * max(1, len(items)))()
    for i, (ln, row0, pos0, seq) in enumerate(items):
        arr[i] = cp_segment(ln, row0, pos0, seq, 0)
    return arr


def cp_abi_version() -> int:
    return lib().cp_abi_version()


def cp_shard_plan_sizes(segs, n_seg: int, n_ranks: int, mode: int):
    """(len of chunk_bounds, len of rank_rows, len of token_index) for cp_shard_plan."""
    sz = np.zeros(3, dtype=np.int64)
    p64 = ctypes.POINTER(ctypes.c_int64)
    _check("cp_shard_plan", lib().cp_shard_plan(segs, n_seg, n_ranks, mode, None, None, None,
                                                sz.ctypes.data_as(p64)))
    return tuple(int(x) for x in sz)


def cp_shard_plan(segs, n_seg: int, n_ranks: int, mode: int):
    """Returns (chunk_bounds [n_seg, 2N+1], rank_rows [N+1], token_index [sum len]) as int64 arrays,
    sized by the library's own sizes query."""
    n_cb, n_rr, n_ti = cp_shard_plan_sizes(segs, n_seg, n_ranks, mode)
    cb = np.zeros(max(1, n_cb), dtype=np.int64)
    rr = np.zeros(n_rr, dtype=np.int64)
    ti = np.zeros(max(1, n_ti), dtype=np.int64)
    p64 = ctypes.POINTER(ctypes.c_int64)
    _check("cp_shard_plan", lib().cp_shard_plan(segs, n_seg, n_ranks, mode, cb.ctypes.data_as(p64),
                                                rr.ctypes.data_as(p64), ti.ctypes.data_as(p64), None))
    return cb[:n_cb].reshape(n_seg, 2 * n_ranks + 1), rr, ti[:n_ti]


def cp_rank_ranges(segs, n_seg: int, n_ranks: int, mode: int, rank: int):
    out = (cp_range * max(1, 2 * n_seg))()
    n = ctypes.c_int32(0)
    _check("cp_rank_ranges", lib().cp_rank_ranges(segs, n_seg, n_ranks, mode, rank, out, ctypes.byref(n)))
    return [out[i] for i in range(n.value)]


def cp_ring_schedule(q_segs, n_q_seg: int, kv_segs, n_kv_seg: int, n_ranks: int, mode: int, variant: int):
    """Returns (ranges ctypes array, n_ranges, blocks ctypes array [N*N], parts list [N*N])."""
    cap = 2 * n_ranks * (n_q_seg + n_kv_seg) + 1
    ranges = (cp_range * cap)()
    blocks = (cp_block * (n_ranks * n_ranks))()
    parts = (ctypes.c_int32 * (n_ranks * n_ranks))()
    n = ctypes.c_int32(0)
    _check("cp_ring_schedule", lib().cp_ring_schedule(q_segs, n_q_seg, kv_segs, n_kv_seg, n_ranks, mode, variant,
                                                      ranges, cap, ctypes.byref(n), blocks, parts))
    return ranges, n.value, blocks, list(parts)


def cp_select_ring_variant(t: int, p: int, n_h: int, n_kv: int, d: int, n_ranks: int, elem_bytes: int,
                           link_bytes_per_s: float, step_attn_s: float):
    """Algorithm 1: returns (variant, reason) with reason 1 or 2 for the
    condition that chose pass-KV and 0 for pass-Q."""
    var = ctypes.c_int32(-1)
    why = ctypes.c_int32(-1)
    _check("cp_select_ring_variant", lib().cp_select_ring_variant(
        t, p, n_h, n_kv, d, n_ranks, elem_bytes, float(link_bytes_per_s), float(step_attn_s), ctypes.byref(var),
        ctypes.byref(why)))
    return var.value, why.value


def cp_classify_pair(q: cp_range, kv: cp_range, causal: bool = True) -> int:
    return lib().cp_classify_pair(ctypes.byref(q), ctypes.byref(kv), int(causal))


def cp_block_pairs(ranges, block: cp_block, causal: bool = True) -> int:
    return lib().cp_block_pairs(ranges, ctypes.byref(block), int(causal))


def cp_ring_comm_volume(ranges, blocks, n_ranks: int, variant: int, n_h: int, n_kv: int, d: int):
    hops = np.zeros(max(1, (n_ranks - 1) * n_ranks), dtype=np.int64)
    total, a2a = ctypes.c_int64(0), ctypes.c_int64(0)
    p64 = ctypes.POINTER(ctypes.c_int64)
    _check("cp_ring_comm_volume", lib().cp_ring_comm_volume(ranges, blocks, n_ranks, variant, n_h, n_kv, d,
                                                            hops.ctypes.data_as(p64), ctypes.byref(total),
                                                            ctypes.byref(a2a)))
    return hops[:(n_ranks - 1) * n_ranks].reshape(n_ranks - 1, n_ranks), total.value, a2a.value


# ----------------------------------------------------------------------------- device entry points
def cp_workspace_size(op: int, rows: int, n_h: int, d: int, n_splits: int) -> int:
    return int(lib().cp_workspace_size(op, rows, n_h, d, n_splits))


def cp_reset_status(workspace, stream=None) -> None:
    _check("cp_reset_status", lib().cp_reset_status(_ptr(workspace), _stream(stream)))


def cp_wait_selftest(workspace, budget_ns: int, stream=None) -> None:
    """Launch the bounded-wait self-test: the status word of `workspace` then
    holds a timeout (cp_check_status raises CP_ERR_TIMEOUT)."""
    _check("cp_wait_selftest", lib().cp_wait_selftest(_ptr(workspace), int(workspace.numel() * workspace.element_size()),
                                                      int(budget_ns), _stream(stream)))


def cp_check_status(workspace, stream=None) -> None:
    _check("cp_check_status", lib().cp_check_status(_ptr(workspace), _stream(stream)))


def cp_attn_partial(q, k, v, n_h: int, n_kv: int, softmax_scale: float, causal: bool, ranges, n_ranges: int,
                    blocks, n_blocks: int, o_part, lse_part, workspace, stream=None) -> None:
    """q [q_rows, n_h, d], k/v [kv_rows, n_kv, d] (same dtype), o_part [out_rows, n_h, d] fp32,
    lse_part [out_rows, n_h] fp32; ranges/blocks are ctypes arrays (or pointers into them)."""
    d = int(q.shape[-1])
    code = lib().cp_attn_partial(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), int(q.shape[0]), int(k.shape[0]),
                                 n_h, n_kv, d, float(softmax_scale), int(causal), ranges, n_ranges, blocks,
                                 n_blocks, _ptr(o_part), _ptr(lse_part), int(o_part.shape[0]), _ptr(workspace),
                                 int(workspace.numel() * workspace.element_size()), _stream(stream))
    _check("cp_attn_partial", code)


def cp_attn_partial_fused(q, k, v, n_h: int, n_kv: int, softmax_scale: float, causal: bool, ranges, n_ranges: int,
                          blocks, n_blocks: int, o_acc, lse_acc, accumulate: bool, out=None, workspace=None,
                          stream=None) -> None:
    """cp_attn_partial merging into the running (o_acc, lse_acc) when `accumulate`;
    with `out` (bf16 [rows, n_h, d]) the merged rows are written there normalised."""
    d = int(q.shape[-1])
    code = lib().cp_attn_partial_fused(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), int(q.shape[0]), int(k.shape[0]),
                                       n_h, n_kv, d, float(softmax_scale), int(causal), ranges, n_ranges, blocks,
                                       n_blocks, _ptr(o_acc), _ptr(lse_acc), int(o_acc.shape[0]), int(bool(accumulate)),
                                       _ptr(out), _ptr(workspace), int(workspace.numel() * workspace.element_size()),
                                       _stream(stream))
    _check("cp_attn_partial_fused", code)


def cp_attn_merge(o_parts, lse_parts, n_parts: int, part_stride_rows: int, rows: int, n_h: int, d: int, out,
                  lse_out=None, stream=None) -> None:
    """LSE merge; o_parts fp32 (cp_attn_merge) or bf16 (cp_attn_merge_bf16_parts), chosen by its dtype."""
    fn = "cp_attn_merge_bf16_parts" if _dtype_code(o_parts) == CP_BF16 else "cp_attn_merge"
    code = getattr(lib(), fn)(_ptr(o_parts), _ptr(lse_parts), n_parts, part_stride_rows, rows, n_h, d,
                              _ptr(out), _dtype_code(out), _ptr(lse_out), _stream(stream))
    _check(fn, code)


def cp_attn_partial_bf16_parts(q, k, v, n_h: int, n_kv: int, softmax_scale: float, causal: bool, ranges,
                               n_ranges: int, blocks, n_blocks: int, o_part, lse_part, workspace, stream=None) -> None:
    """cp_attn_partial writing bf16 O partials (o_part bf16 [out_rows, n_h, d]); LSE fp32."""
    d = int(q.shape[-1])
    code = lib().cp_attn_partial_bf16_parts(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), int(q.shape[0]),
                                            int(k.shape[0]), n_h, n_kv, d, float(softmax_scale), int(causal), ranges,
                                            n_ranges, blocks, n_blocks, _ptr(o_part), _ptr(lse_part),
                                            int(o_part.shape[0]), _ptr(workspace),
                                            int(workspace.numel() * workspace.element_size()), _stream(stream))
    _check("cp_attn_partial_bf16_parts", code)


def cp_decode(q, k, v, kv_offsets, n_h: int, n_kv: int, n_splits: int, softmax_scale: float, out, lse_out,
              workspace, stream=None) -> None:
    """q [batch, n_h, d] bf16; k/v packed [kv_rows, n_kv, d] bf16; kv_offsets device int64 [batch+1]."""
    code = lib().cp_decode(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), _ptr(kv_offsets), int(q.shape[0]),
                           int(k.shape[0]), n_h, n_kv, int(q.shape[-1]), n_splits, float(softmax_scale),
                           _ptr(out), _ptr(lse_out), _ptr(workspace),
                           int(workspace.numel() * workspace.element_size()), _stream(stream))
    _check("cp_decode", code)


def cp_decode_partial(q, k, v, kv_offsets, n_h: int, n_kv: int, n_splits: int, softmax_scale: float, o_part,
                      lse_part, workspace, stream=None) -> None:
    """cp_decode's partial: o_part [batch, n_h, d] fp32 and lse_part [batch, n_h]
    fp32 over the keys k/v hold, for a later cp_attn_merge across ranks."""
    code = lib().cp_decode_partial(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), _ptr(kv_offsets), int(q.shape[0]),
                                   int(k.shape[0]), n_h, n_kv, int(q.shape[-1]), n_splits, float(softmax_scale),
                                   _ptr(o_part), _ptr(lse_part), _ptr(workspace),
                                   int(workspace.numel() * workspace.element_size()), _stream(stream))
    _check("cp_decode_partial", code)


def cp_decode_static(q, k, v, kv_offsets, n_h: int, n_kv: int, n_splits: int, softmax_scale: float, out, lse_out,
                     stream=None) -> None:
    """cp_decode without a workspace, for callers that cannot allocate device
    memory while decoding: the split partials and the status word use the
    library's fixed 32 MiB array on the current device. Calls must not overlap
    on the GPU; cp_decode_static_status reports the latest call's device-side
    status."""
    code = lib().cp_decode_static(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), _ptr(kv_offsets), int(q.shape[0]),
                                  int(k.shape[0]), n_h, n_kv, int(q.shape[-1]), n_splits, float(softmax_scale),
                                  _ptr(out), _ptr(lse_out), _stream(stream))
    _check("cp_decode_static", code)


def cp_decode_static_status(stream=None) -> None:
    """Synchronise the stream and raise CpError if the latest cp_decode_static
    call on the current device recorded a device-side failure."""
    _check("cp_decode_static_status", lib().cp_decode_static_status(_stream(stream)))
