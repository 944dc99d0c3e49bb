"""Seeded randomized GPU parity: many small configurations drawn at once over
every dimension the hot path takes (sequence lengths including ragged and
one-token ones, cached prefixes, several sequences, rank counts, GQA group
sizes, head dims, ring variant, shard mode, merge mode, peaked queries), each
run through the library and checked against the fp64 reference with the bf16
tolerances of the other tests (the exact fp32 path at 1e-5); and the same
for split-KV decode (request counts, lengths including 0 and 1, groups up to
64 heads, head dims, split counts). The draws are fixed by the case index, so a failure names a
reproducible configuration."""
import math

import numpy as np
import pytest
import torch

from context_ring_attn_b200 import binding as B
from context_ring_attn_b200 import ring, synth
from oracle import decode as OD

from gpu_util import check
from test_gpu_kernels import _run_prefill

pytestmark = pytest.mark.gpu

N_RING = 96
N_EXACT = 24
N_DECODE = 48


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    B.lib()


def _ring_case(i):
    rng = np.random.default_rng(5150 + i)
    d = int(rng.choice([64, 128]))
    group = int(rng.choice([1, 2, 4, 8, 16]))
    n_kv = int(rng.choice([1, 2]))
    n_h = group * n_kv
    variant = int(rng.choice([B.CP_PASS_KV, B.CP_PASS_Q]))
    mode = int(rng.choice([B.CP_SHARD_LOAD_BALANCED, B.CP_SHARD_CONTIGUOUS]))
    n_ranks = int(rng.integers(1, 6))
    merge = str(rng.choice(["final", "final_bf16", "running", "fused"]))
    q_scale = float(rng.choice([1.0, 8.0]))
    if rng.random() < 0.35:   # several sequences of one varlen batch
        lens = [int(x) for x in rng.integers(1, 400, size=int(rng.integers(2, 5)))]
        return dict(d=d, n_h=n_h, n_kv=n_kv, variant=variant, mode=mode, n_ranks=n_ranks, merge=merge,
                    q_scale=q_scale, lens=lens, t=sum(lens), p=0)
    t = int(rng.integers(1, 600))
    p = int(rng.integers(1, 800)) if rng.random() < 0.4 else 0
    return dict(d=d, n_h=n_h, n_kv=n_kv, variant=variant, mode=mode, n_ranks=n_ranks, merge=merge,
                q_scale=q_scale, lens=None, t=t, p=p)


@pytest.mark.parametrize("i", range(N_RING))
def test_random_ring(i):
    c = _ring_case(i)
    pr = synth.make_prefill(c["t"], c["n_h"], c["n_kv"], c["d"], "bf16", 9000 + i, 0.5, p=c["p"])
    segs = None
    if c["lens"] is not None:
        segs, r0 = [], 0
        for s, n in enumerate(c["lens"]):
            segs.append(ring.Segment(n, r0, 0, s))
            r0 += n
    _run_prefill(pr, c["n_ranks"], c["variant"], c["mode"], merge=c["merge"], q_scale=c["q_scale"], segs=segs)


def _exact_case(i):
    rng = np.random.default_rng(7170 + i)
    group = int(rng.choice([1, 2, 4, 8]))
    n_kv = int(rng.choice([1, 2]))
    return dict(d=int(rng.choice([64, 128])), n_h=group * n_kv, n_kv=n_kv,
                variant=int(rng.choice([B.CP_PASS_KV, B.CP_PASS_Q])),
                mode=int(rng.choice([B.CP_SHARD_LOAD_BALANCED, B.CP_SHARD_CONTIGUOUS])),
                n_ranks=int(rng.integers(1, 6)), merge=str(rng.choice(["final", "running"])),
                t=int(rng.integers(1, 200)), p=int(rng.integers(1, 300)) if rng.random() < 0.4 else 0)


@pytest.mark.parametrize("i", range(N_EXACT))
def test_random_exact_fp32(i):
    """The exact fp32 path at its 1e-5 tolerance."""
    c = _exact_case(i)
    pr = synth.make_prefill(c["t"], c["n_h"], c["n_kv"], c["d"], "f32", 9700 + i, 1.0, p=c["p"])
    _run_prefill(pr, c["n_ranks"], c["variant"], c["mode"], merge=c["merge"])


def _decode_case(i):
    rng = np.random.default_rng(6160 + i)
    d = int(rng.choice([64, 128]))
    group = int(rng.choice([1, 4, 16, 32, 64]))
    n_kv = int(rng.choice([1, 2]))
    batch = int(rng.integers(1, 13))
    lens = rng.integers(0, 3000, size=batch)
    special = rng.random(batch)
    lens[special < 0.15] = 0    # requests without keys
    lens[(special >= 0.15) & (special < 0.3)] = 1
    n_splits = int(rng.choice([1, 7, 64, 256]))
    return dict(d=d, n_h=group * n_kv, n_kv=n_kv, lens=[int(x) for x in lens], n_splits=n_splits)


@pytest.mark.parametrize("i", range(N_DECODE))
def test_random_decode(i):
    c = _decode_case(i)
    dc = synth.make_decode(len(c["lens"]), c["n_h"], c["n_kv"], c["d"], c["lens"], 9500 + i, 0.5)
    to = lambda raw: torch.from_numpy(np.ascontiguousarray(raw).view(np.int16)).view(torch.bfloat16).cuda()  # noqa: E731
    b, n_h, d = len(c["lens"]), c["n_h"], c["d"]
    out = torch.full((b, n_h, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((b, n_h), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.zeros(B.cp_workspace_size(B.CP_OP_DECODE, b, n_h, d, c["n_splits"]), dtype=torch.uint8, device="cuda")
    B.cp_decode(to(dc.q_raw), to(dc.k_raw), to(dc.v_raw), torch.from_numpy(dc.offsets).cuda(), n_h, c["n_kv"],
                c["n_splits"], 1 / math.sqrt(d), out, lse, ws)
    B.cp_check_status(ws)
    o_ref, l_ref = OD.decode(dc.q, dc.k, dc.v, dc.offsets)
    check(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, "bf16",
          f"decode case {i}: B={b} n_h={n_h} n_kv={c['n_kv']} d={d} splits={c['n_splits']}")
