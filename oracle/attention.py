"""Unsharded exact attention, per-block partials and the LSE merge, in fp64.

Test infrastructure (see the package docstring): only tests and the bench's
CPU-baseline leg use this module.

Definition followed ("Context Parallelism과 Expert Parallelism", section 5.1;
"Context Parallelism for Scalable Million-Token Inference", section 3 core
formulas): for query row i at global position p_i and query head h, the KV head
is g = floor(h / (N_H / N_KV)) (GQA groups of consecutive query heads, section
8.2 of the first page). The visible keys are V_i = {j : seq(j) = seq(i),
p_j <= p_i} (causal, inclusive of the token itself). With s_j = scale * <q_ih,
k_jg>:

    LSE_ih = ln sum_{j in V_i} exp(s_j)
    O_ih   = sum_{j in V_i} exp(s_j - LSE_ih) * v_jg

which is softmax(q K^T) V restricted to the visible keys. A row with no
visible key has O = 0 and LSE = -inf (it contributes nothing to a merge).

Rows are independent, so they are processed a group of rows at a time to bound
memory; each row's softmax is still taken over all of its visible keys at once.
"""
from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


def default_scale(d: int) -> float:
    """Softmax scale 1/sqrt(D_H) (the pages print an unscaled softmax; the
    standard scaled dot-product value is the reading used throughout)."""
    return 1.0 / np.sqrt(d)


def attention(q, k, v, q_pos, k_pos, q_seq=None, k_seq=None, scale=None, causal=True,
              row_group: int = 256):
    """Exact attention of every query row against the visible keys.

    q: [Tq, N_H, D]; k, v: [Tk, N_KV, D]; q_pos: [Tq]; k_pos: [Tk]; optional
    sequence ids q_seq [Tq], k_seq [Tk] (keys of another sequence are never
    visible). Returns (O [Tq, N_H, D] float64, LSE [Tq, N_H] float64).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    tq, n_h, d = q.shape
    tk, n_kv, _ = k.shape
    assert n_h % n_kv == 0
    group = n_h // n_kv
    if scale is None:
        scale = default_scale(d)
    q_pos = np.asarray(q_pos, dtype=np.int64)
    k_pos = np.asarray(k_pos, dtype=np.int64)
    if q_seq is None:
        q_seq = np.zeros(tq, dtype=np.int64)
    if k_seq is None:
        k_seq = np.zeros(tk, dtype=np.int64)
    q_seq = np.asarray(q_seq)
    k_seq = np.asarray(k_seq)

    o = np.zeros((tq, n_h, d), dtype=np.float64)
    lse = np.full((tq, n_h), NEG_INF, dtype=np.float64)
    for r0 in range(0, tq, row_group):
        r1 = min(tq, r0 + row_group)
        visible = k_seq[None, :] == q_seq[r0:r1, None]
        if causal:
            visible &= k_pos[None, :] <= q_pos[r0:r1, None]
        # keys no row of this group can see contribute exactly zero: drop them
        cols = np.nonzero(visible.any(axis=0))[0]
        if cols.size == 0:
            continue
        vis = visible[:, cols]
        for h in range(n_h):
            g = h // group
            s = scale * (q[r0:r1, h, :] @ k[cols, g, :].T)
            s = np.where(vis, s, NEG_INF)
            m = s.max(axis=1)
            has = np.isfinite(m)
            m0 = np.where(has, m, 0.0)
            e = np.exp(s - m0[:, None])
            l = e.sum(axis=1)
            l_safe = np.where(has, l, 1.0)
            lse[r0:r1, h] = np.where(has, m0 + np.log(l_safe), NEG_INF)
            o[r0:r1, h, :] = np.where(has[:, None], (e @ v[cols, g, :]) / l_safe[:, None], 0.0)
    return o, lse


def block_partial(q, k, v, q_pos, k_pos, kv_rows, q_seq=None, k_seq=None, scale=None,
                  causal=True):
    """Partial attention of all query rows against the key rows ``kv_rows`` only.

    This is one ring block: a query shard against one KV shard. The output is
    normalised within the block and LSE is the block's log-sum-exp, so that
    merging the blocks of a row reproduces the unsharded row.
    """
    kv_rows = np.asarray(kv_rows, dtype=np.int64)
    ks = None if k_seq is None else np.asarray(k_seq)[kv_rows]
    return attention(q, np.asarray(k)[kv_rows], np.asarray(v)[kv_rows], q_pos,
                     np.asarray(k_pos)[kv_rows], q_seq, ks, scale, causal)


def merge(o_parts, lse_parts):
    """Combine partials of the same rows by LSE weighting.

    With M = max_j LSE_j:  LSE = M + ln sum_j exp(LSE_j - M),
    O = sum_j exp(LSE_j - LSE) * O_j. Parts with LSE = -inf get weight 0; if
    every part is -inf the row stays O = 0, LSE = -inf. This is the "merge
    attention" step the method runs after the pass-Q ring (section 5,
    implementation details item 3), applied in the order the parts are given.
    """
    lse_stack = np.stack([np.asarray(x, dtype=np.float64) for x in lse_parts])
    m = lse_stack.max(axis=0)
    has = np.isfinite(m)
    m0 = np.where(has, m, 0.0)
    w_sum = np.zeros_like(m0)
    for lj in lse_stack:
        w_sum = w_sum + np.exp(lj - m0)
    lse = np.where(has, m0 + np.log(np.where(has, w_sum, 1.0)), NEG_INF)
    lse0 = np.where(has, lse, 0.0)
    o = np.zeros(np.asarray(o_parts[0]).shape, dtype=np.float64)
    for oj, lj in zip(o_parts, lse_stack):
        w = np.where(has, np.exp(lj - lse0), 0.0)
        o = o + w[..., None] * np.asarray(oj, dtype=np.float64)
    return o, lse
