"""Seeded synthetic inputs for the context-parallel attention path.

This module is the one piece shared by the CUDA path's callers (tests, bench)
and the fp64 reference: it only draws numbers and rounds them to the storage
dtype. It holds none of the attention arithmetic.

Recipe (the pages fix shapes but not distributions or seeds):
  * every tensor is iid normal, drawn in float32 with numpy's PCG64 generator;
  * std is 1.0 for the fp32 tiny check and 0.5 for the bf16 workloads;
  * bf16 tensors are rounded on the host, round-to-nearest-even, and every
    consumer (GPU kernels and the reference) sees the rounded values;
  * rows are drawn in blocks of ``ROW_BLOCK`` rows, each block from its own
    ``SeedSequence([seed, tensor_id, block])`` so any subset of rows can be
    regenerated without drawing the whole tensor.

Shapes follow "Context Parallelism for Scalable Million-Token Inference"
(page review, section 3, core formulas): Q is [T, N_H, D_H] and K = V are
[(T+P), N_KV, D_H], token-major.
"""
from __future__ import annotations

import itertools
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

ROW_BLOCK = 4096

TENSOR_Q = 0
TENSOR_K = 1
TENSOR_V = 2
TENSOR_LENGTHS = 3


# --------------------------------------------------------------------------
# bf16 storage rounding
# --------------------------------------------------------------------------
def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even).

    Returns the raw 16-bit patterns as uint16. Inputs are finite normals here;
    NaN/Inf are passed through by truncation of the payload-free patterns.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    rounded = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    nonfinite = (u & np.uint32(0x7F800000)) == np.uint32(0x7F800000)
    rounded = np.where(nonfinite, u >> np.uint32(16), rounded)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen raw bf16 patterns (uint16) to float32 exactly."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------
# row-blocked normal tensors
# --------------------------------------------------------------------------
def _block_rng(seed: int, tensor_id: int, block: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tensor_id, block])))


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _blocked(seed, tensor_id, n_rows, row_shape, std, rows, transform, out_dtype):
    width = int(np.prod(row_shape))
    if rows is None:
        rows = np.arange(n_rows, dtype=np.int64)
        contiguous = True
    else:
        rows = np.asarray(rows, dtype=np.int64)
        contiguous = False
    out = np.empty((rows.size, width), dtype=out_dtype)
    blocks = np.unique(rows // ROW_BLOCK)

    def fill(blk):
        g = _block_rng(seed, tensor_id, int(blk))
        full = g.standard_normal((ROW_BLOCK, width), dtype=np.float32)
        full *= np.float32(std)
        if contiguous:
            r0 = int(blk) * ROW_BLOCK
            nb = min(ROW_BLOCK, n_rows - r0)
            out[r0:r0 + nb] = transform(full[:nb])
        else:
            sel = np.nonzero(rows // ROW_BLOCK == blk)[0]
            out[sel] = transform(full[rows[sel] - blk * ROW_BLOCK])

    if len(blocks) > 1:
        with ThreadPoolExecutor(max_workers=_threads()) as ex:
            list(ex.map(fill, blocks))
    else:
        for blk in blocks:
            fill(blk)
    return out.reshape((rows.size,) + tuple(row_shape))


def normal_rows(seed: int, tensor_id: int, n_rows: int, row_shape: tuple, std: float,
                rows: np.ndarray | None = None) -> np.ndarray:
    """float32 normal tensor [n_rows, *row_shape] (or only ``rows`` of it).

    Blocks are drawn on a thread pool (each block has its own generator, so
    the values do not depend on the thread count)."""
    return _blocked(seed, tensor_id, n_rows, row_shape, std, rows, lambda x: x, np.float32)


def raw_rows(seed: int, tensor_id: int, n_rows: int, row_shape: tuple, std: float, dtype: str,
             rows: np.ndarray | None = None) -> np.ndarray:
    """The stored form of normal_rows: float32, or bf16 bit patterns (uint16)."""
    if dtype == "f32":
        return normal_rows(seed, tensor_id, n_rows, row_shape, std, rows)
    return _blocked(seed, tensor_id, n_rows, row_shape, std, rows, bf16_bits, np.uint16)


def stored_values(x32: np.ndarray, dtype: str) -> tuple[np.ndarray, np.ndarray]:
    """(values as float32 exactly as stored, raw storage array) for ``dtype``."""
    if dtype == "f32":
        return x32, x32
    if dtype == "bf16":
        bits = bf16_bits(x32)
        return bf16_bits_to_f32(bits), bits
    raise ValueError(dtype)


# --------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------
@dataclass
class Prefill:
    """One prefill problem. q/k/v hold float32 copies of the stored values."""
    t: int
    p: int
    n_h: int
    n_kv: int
    d: int
    dtype: str
    seed: int
    std: float
    seq_lens: list = field(default_factory=list)   # varlen: tokens per sequence
    q: np.ndarray | None = None
    k: np.ndarray | None = None
    v: np.ndarray | None = None
    q_raw: np.ndarray | None = None
    k_raw: np.ndarray | None = None
    v_raw: np.ndarray | None = None

    def q_rows(self, rows) -> np.ndarray:
        """Stored Q values (float32) of selected token rows, regenerated."""
        x = normal_rows(self.seed, TENSOR_Q, self.t, (self.n_h, self.d), self.std, rows)
        return stored_values(x, self.dtype)[0]


def make_prefill(t: int, n_h: int, n_kv: int, d: int, dtype: str, seed: int, std: float,
                 p: int = 0, seq_lens=None, with_q: bool = True) -> Prefill:
    """Q [t, n_h, d] at positions p..p+t-1; K, V [p+t, n_kv, d]."""
    pr = Prefill(t=t, p=p, n_h=n_h, n_kv=n_kv, d=d, dtype=dtype, seed=seed, std=std,
                 seq_lens=list(seq_lens) if seq_lens is not None else [t])
    if with_q:
        pr.q, pr.q_raw = stored_values(normal_rows(seed, TENSOR_Q, t, (n_h, d), std), dtype)
    pr.k, pr.k_raw = stored_values(normal_rows(seed, TENSOR_K, p + t, (n_kv, d), std), dtype)
    pr.v, pr.v_raw = stored_values(normal_rows(seed, TENSOR_V, p + t, (n_kv, d), std), dtype)
    return pr


@dataclass
class Decode:
    batch: int
    n_h: int
    n_kv: int
    d: int
    lens: np.ndarray          # int64 [batch]
    offsets: np.ndarray       # int64 [batch + 1]
    q: np.ndarray             # float32 [batch, n_h, d]
    k: np.ndarray             # float32 [sum lens, n_kv, d]
    v: np.ndarray
    q_raw: np.ndarray
    k_raw: np.ndarray
    v_raw: np.ndarray


def decode_lengths(seed: int, batch: int, lo: int, hi: int) -> np.ndarray:
    """Per-request context lengths, uniform integers in [lo, hi]."""
    g = _block_rng(seed, TENSOR_LENGTHS, 0)
    return g.integers(lo, hi, endpoint=True, size=batch).astype(np.int64)


def make_decode(batch: int, n_h: int, n_kv: int, d: int, lens, seed: int, std: float,
                dtype: str = "bf16") -> Decode:
    lens = np.asarray(lens, dtype=np.int64)
    offsets = np.zeros(batch + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(lens)
    total = int(offsets[-1])
    q, q_raw = stored_values(normal_rows(seed, TENSOR_Q, batch, (n_h, d), std), dtype)
    k, k_raw = stored_values(normal_rows(seed, TENSOR_K, total, (n_kv, d), std), dtype)
    v, v_raw = stored_values(normal_rows(seed, TENSOR_V, total, (n_kv, d), std), dtype)
    return Decode(batch, n_h, n_kv, d, lens, offsets, q, k, v, q_raw, k_raw, v_raw)


VARLEN_CHOICES = (4096, 8192, 16384, 32768, 65536)


def varlen_lengths(seed: int, n_seq: int = 8, total: int = 262144,
                   choices=VARLEN_CHOICES) -> list[int]:
    """Pick one ordered n_seq-tuple from ``choices`` with the given sum, uniformly."""
    tuples = [tp for tp in itertools.product(choices, repeat=n_seq) if sum(tp) == total]
    g = _block_rng(seed, TENSOR_LENGTHS, 0)
    return list(tuples[int(g.integers(0, len(tuples)))])


# The five workloads (sizes as the method's shapes give them; seeds 1000 + index).
WORKLOADS = {
    "tiny_exact": dict(t=256, p=0, n_h=4, n_kv=1, d=64, dtype="f32", seed=1001, std=1.0, n_ranks=4),
    "prefill_128k": dict(t=131072, p=0, n_h=16, n_kv=1, d=128, dtype="bf16", seed=1002, std=0.5, n_ranks=8),
    "persistent_kv": dict(t=4096, p=126976, n_h=128, n_kv=8, d=128, dtype="bf16", seed=1003, std=0.5, n_ranks=8),
    "decode_split": dict(batch=32, n_h=16, n_kv=1, d=128, lo=32768, hi=131072, n_splits=256,
                         dtype="bf16", seed=1004, std=0.5),
    "varlen_prefill": dict(total=262144, n_seq=8, n_h=128, n_kv=8, d=128, dtype="bf16", seed=1005,
                           std=0.5, n_ranks=8),
}


# --------------------------------------------------------------------------
# device upload (chunked: a full-size Q never exists in fp32 on the host)
# --------------------------------------------------------------------------
def device_rows(seed: int, tensor_id: int, n_rows: int, row_shape: tuple, std: float, dtype: str,
                device="cuda"):
    """Generate a tensor block by block and copy each block to the device.
    Returns a torch tensor [n_rows, *row_shape] of bf16 or fp32."""
    import torch

    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = torch.empty((n_rows,) + tuple(row_shape), dtype=tdt, device=device)
    step = ROW_BLOCK * 64
    for r0 in range(0, n_rows, step):
        r1 = min(n_rows, r0 + step)
        raw = raw_rows(seed, tensor_id, n_rows, row_shape, std, dtype, np.arange(r0, r1))
        src = torch.from_numpy(raw.view(np.int16)).view(torch.bfloat16) if dtype == "bf16" else torch.from_numpy(raw)
        out[r0:r1].copy_(src)
    return out
