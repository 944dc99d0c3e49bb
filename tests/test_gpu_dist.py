"""The multi-process ring driver with the library's kernels, on one GPU: a
one-rank NCCL group (the exchange steps are empty), both ring variants; the
exchange itself is covered on gloo ranks by test_dist_gloo."""
import math
from datetime import timedelta
import socket

import numpy as np
import pytest
import torch

from context_ring_attn_b200 import binding as B
from context_ring_attn_b200 import synth
from oracle import attention as OA

from gpu_util import check, dev

pytestmark = pytest.mark.gpu


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.fixture(scope="module")
def group():
    import torch.distributed as dist
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_port()}", rank=0, world_size=1,
                            timeout=timedelta(seconds=60), device_id=torch.device("cuda", 0))
    yield None
    dist.destroy_process_group()


@pytest.mark.parametrize("variant", [B.CP_PASS_KV, B.CP_PASS_Q])
def test_ring_driver_runs_the_kernels(group, variant):
    from context_ring_attn_b200.dist import RingAttention, Segment
    t, p, n_h, n_kv, d = 384, 640, 16, 2, 128
    rng = np.random.default_rng(5)
    q = rng.standard_normal((t, n_h, d)) * 0.5
    k = rng.standard_normal((p + t, n_kv, d)) * 0.5
    v = rng.standard_normal((p + t, n_kv, d)) * 0.5
    qb, kb, vb = (synth.stored_values(x.astype(np.float32), "bf16") for x in (q, k, v))
    ra = RingAttention([Segment(t, 0, p, 0)], [Segment(p, 0, 0, 0), Segment(t, p, p, 0)], n_h, n_kv, d, variant)
    qi, ki = ra.q_shard_rows().numpy(), ra.kv_shard_rows().numpy()
    out, lse = ra.forward(dev(qb[1][qi], "bf16"), dev(kb[1][ki], "bf16"), dev(vb[1][ki], "bf16"), 1 / math.sqrt(d))
    torch.cuda.synchronize()
    o_ref, l_ref = OA.attention(qb[0][qi], kb[0], vb[0], np.arange(p, p + t)[qi], np.arange(p + t))
    check(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, "bf16", "ring driver")
