"""fp64 CPU reference for context-parallel ring attention (test infrastructure).

This package is test infrastructure, not product code. Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it. The CUDA library never calls it, and it
shares no code with the CUDA library: it is written directly from the method
pages and imports nothing from the ``context_ring_attn_b200`` package.

Sources (web pages, cited by title and section):
  * "Context Parallelism for Scalable Million-Token Inference" (a review of
    arXiv:2411.01783): attention shapes with a persistent KV prefix
    (section 3, core formulas), ring pass-KV / pass-Q (section 3), the merge
    step after pass-Q (section 5, implementation details item 3),
    load-balanced sharding (section 4), Flash Decoding with 256 splits
    (section 5, software stack), communication sizes (section 3,
    parallelism comparison table) and the Algorithm 1 threshold.
  * "Context Parallelism과 Expert Parallelism": per-token attention
    softmax(q_t K^T) V and the inclusive causal mask (section 5.1), prefill vs
    decode (section 5.2), GQA head groups (section 8.2).

Modules:
  attention  -- unsharded attention definition, block partials, LSE merge
  plan       -- independent shard planner and ring schedules
  decode     -- single-query decode, whole and split into KV chunks
  comm       -- communication-volume accounting and the pages' closed forms

Parity status: every function here is pinned by the ``-m "not gpu"`` tests
(brute force, torch SDPA on CPU, invariants, closed forms). The chunk
rounding when 2N does not divide a length is a reading of the pages that
the pages themselves cannot pin (all pages' workloads divide evenly); it is
pinned only by partition invariants.
"""
from . import attention, comm, decode, plan  # noqa: F401
