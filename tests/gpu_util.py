"""Helpers for the GPU parity tests: device copies of synthetic inputs,
tolerance checks against the fp64 reference."""
from __future__ import annotations

import numpy as np
import torch

# Tolerances: fp32 inputs max-abs 1e-5; bf16 inputs with fp32 accumulation
# max-abs 2e-2, mean-abs 2e-3, LSE 1e-3. The relative row-norm bound guards
# against diffuse attention where |O| is tiny and an all-zero output would
# pass an absolute bound: bf16 rounding of P and of the output is ~2^-9 per
# element, so 1e-2 of the row norm is generous but far below a wrong answer.
TOL = {
    "f32": dict(max_abs=1e-5, mean_abs=1e-6, lse=1e-5, row_rel=1e-4),
    "bf16": dict(max_abs=2e-2, mean_abs=2e-3, lse=1e-3, row_rel=1e-2),
}


def dev(raw: np.ndarray, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(raw).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(raw, dtype=np.float32)).cuda()


def check(o_gpu, lse_gpu, o_ref, lse_ref, dtype: str, what: str = ""):
    """Compare (O, LSE) with the reference; rows with LSE = -inf must match
    exactly (O = 0). Returns the error statistics."""
    tol = TOL[dtype]
    o = np.asarray(o_gpu, dtype=np.float64)
    lg = np.asarray(lse_gpu, dtype=np.float64)
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert np.all(np.isfinite(o)), f"{what}: non-finite output"
    neg = ~np.isfinite(lse_ref)
    assert np.array_equal(~np.isfinite(lg), neg), f"{what}: -inf rows differ"
    if neg.any():
        assert np.all(lg[neg] == -np.inf) and np.all(o[neg] == 0.0), f"{what}: empty rows not zero/-inf"
    err = np.abs(o - o_ref)
    stats = dict(max_abs=float(err.max(initial=0.0)), mean_abs=float(err.mean()) if err.size else 0.0)
    fin = ~neg
    stats["lse"] = float(np.abs(lg[fin] - lse_ref[fin]).max(initial=0.0))
    ref_norm = np.linalg.norm(o_ref, axis=-1)
    err_norm = np.linalg.norm(o - o_ref, axis=-1)
    ok = ref_norm > 1e-6
    stats["row_rel"] = float((err_norm[ok] / ref_norm[ok]).max(initial=0.0))
    for key in ("max_abs", "mean_abs", "lse", "row_rel"):
        assert stats[key] <= tol[key], f"{what}: {key} {stats[key]:.3g} > {tol[key]:.3g} ({stats})"
    return stats


def sample_rows(rng, n_rows: int, n_sample: int, must=()) -> np.ndarray:
    """Sorted unique rows: every row of `must` plus seeded random others, at
    least n_sample in all (or every row if there are fewer)."""
    must = np.unique(np.asarray([m for m in must if 0 <= m < n_rows], dtype=np.int64))
    others = np.setdiff1d(np.arange(n_rows, dtype=np.int64), must, assume_unique=True)
    rest = rng.choice(others, size=min(others.size, max(0, n_sample - must.size)), replace=False)
    return np.unique(np.concatenate([must, rest]))


def oracle_rows(fn, n_rows: int, chunk: int = 128, workers: int | None = None):
    """Run fn(lo, hi) -> (O, LSE) of rows lo..hi-1 of a sample on a thread
    pool (numpy's BLAS and ufunc loops release the GIL) and stack the results
    in row order. Only the reference runs here; it is called unchanged, on
    slices of the sampled rows."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    bounds = [(lo, min(n_rows, lo + chunk)) for lo in range(0, n_rows, chunk)]
    workers = workers or max(1, min(16, os.cpu_count() or 1))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        parts = list(ex.map(lambda b: fn(*b), bounds))
    return np.concatenate([x[0] for x in parts]), np.concatenate([x[1] for x in parts])
