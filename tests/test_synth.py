"""The seeded input generator: bf16 rounding against torch, row regeneration,
length draws."""
import numpy as np
import torch

from context_ring_attn_b200 import synth


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(200000).astype(np.float32) * 3
    # exact ties and neighbours of ties
    base = np.array([1.0, -1.5, 3.0, 1e-3], dtype=np.float32).view(np.uint32)
    ties = np.concatenate([base + 0x8000, base + 0x7FFF, base + 0x8001, base + 0x18000]).view(np.float32)
    x = np.concatenate([x, ties, np.array([0.0, -0.0, 65504.0, 1e-38], np.float32)])
    ours = synth.bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = synth.bf16_bits_to_f32(ours)
    ref_back = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(back, ref_back)


def test_row_regeneration():
    full = synth.normal_rows(11, synth.TENSOR_Q, 10000, (3, 4), 0.5)
    rows = np.array([0, 4095, 4096, 9999, 17, 5000])
    part = synth.normal_rows(11, synth.TENSOR_Q, 10000, (3, 4), 0.5, rows)
    assert np.array_equal(part, full[rows])


def test_prefill_q_rows_match():
    pr = synth.make_prefill(100, 4, 2, 8, "bf16", 5, 0.5, p=10)
    assert pr.k.shape == (110, 2, 8) and pr.q.shape == (100, 4, 8)
    assert np.array_equal(pr.q_rows([3, 99]), pr.q[[3, 99]])
    assert np.array_equal(synth.bf16_bits_to_f32(pr.q_raw), pr.q)


def test_length_draws():
    lens = synth.varlen_lengths(1005)
    assert len(lens) == 8 and sum(lens) == 262144 and set(lens) <= set(synth.VARLEN_CHOICES)
    d = synth.decode_lengths(1004, 32, 32768, 131072)
    assert d.min() >= 32768 and d.max() <= 131072 and d.size == 32
    assert np.array_equal(d, synth.decode_lengths(1004, 32, 32768, 131072))
