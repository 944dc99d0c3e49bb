"""Single-token decode against a packed KV cache, whole and split (test infrastructure).

Decode ("Context Parallelism과 Expert Parallelism", section 5.2): one new query
per request attends to the whole cached K/V of that request, including the
token just appended, so no mask is needed. Flash Decoding ("Context
Parallelism for Scalable Million-Token Inference", section 5 software stack)
splits the keys of a request into 256 chunks, computes a partial per chunk and
merges them; split s covers keys [floor(s*L/S), floor((s+1)*L/S)).
"""
from __future__ import annotations

import numpy as np

from .attention import attention, merge


def decode(q, k, v, offsets, scale=None):
    """q [B, N_H, D]; k, v packed [sum L_b, N_KV, D]; offsets [B+1].
    Returns (O [B, N_H, D], LSE [B, N_H]) in float64."""
    q = np.asarray(q, dtype=np.float64)
    b_count, n_h, d = q.shape
    o = np.zeros((b_count, n_h, d))
    lse = np.zeros((b_count, n_h))
    for b in range(b_count):
        lo, hi = int(offsets[b]), int(offsets[b + 1])
        length = hi - lo
        ob, lb = attention(q[b:b + 1], k[lo:hi], v[lo:hi], np.array([length - 1]),
                           np.arange(length), scale=scale, causal=True)
        o[b], lse[b] = ob[0], lb[0]
    return o, lse


def split_bounds(length: int, n_splits: int) -> list[int]:
    return [(s * length) // n_splits for s in range(n_splits + 1)]


def decode_split(q, k, v, offsets, n_splits: int, scale=None):
    """The same result computed as n_splits partials per request, then merged."""
    q = np.asarray(q, dtype=np.float64)
    b_count, n_h, d = q.shape
    o = np.zeros((b_count, n_h, d))
    lse = np.zeros((b_count, n_h))
    for b in range(b_count):
        lo, hi = int(offsets[b]), int(offsets[b + 1])
        length = hi - lo
        bounds = split_bounds(length, n_splits)
        o_parts, l_parts = [], []
        for s in range(n_splits):
            a, e = lo + bounds[s], lo + bounds[s + 1]
            op, lp = attention(q[b:b + 1], k[a:e], v[a:e], np.array([length - 1]),
                               np.arange(bounds[s], bounds[s + 1]), scale=scale, causal=True)
            o_parts.append(op[0])
            l_parts.append(lp[0])
        o[b], lse[b] = merge(o_parts, l_parts)
    return o, lse
