"""The FMA-pipe 2^x used for part of the softmax numerators: the same float32
steps as the kernel (Cody-Waite reduction, the generated minimax cubic, the
exponent-field add), emulated on the CPU and held to an error bound well
below bf16 rounding (P is rounded to bf16, relative step 2^-8)."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "context_ring_attn_b200", "csrc", "exp2_poly.cuh")


def coefficients():
    txt = open(HDR).read()
    c = {int(m.group(1)): np.float32(float(m.group(2)))
         for m in re.finditer(r"kExp2C(\d) = ([-+0-9.eE]+)f;", txt)}
    return [c[i] for i in range(4)]


def fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly(x):
    c0, c1, c2, c3 = coefficients()
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-126.0))
    t = (x + f32(12582912.0)).astype(f32)
    j = (t - f32(12582912.0)).astype(f32)
    f = (x - j).astype(f32)
    n = f.size
    p = fma32(np.full(n, c3), f, np.full(n, c2))
    p = fma32(p, f, np.full(n, c1))
    p = fma32(p, f, np.full(n, c0))
    bits = p.view(np.int32) + (t.view(np.int32) << np.int32(23))
    return bits.view(np.float32)


def test_relative_error_bound():
    x = np.concatenate([np.linspace(-126.0, 8.0, 2_000_001, dtype=np.float32),
                        np.float32(np.random.default_rng(0).uniform(-30, 8, 1_000_000))])
    got = exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1.5e-4, rel.max()


def test_integers_and_halves():
    x = np.arange(-120, 9, dtype=np.float32)
    got = exp2_poly(x).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(x.astype(np.float64)) - 1) < 1e-4)
    xh = x + np.float32(0.5)
    assert np.all(np.abs(exp2_poly(xh) / np.exp2(xh.astype(np.float64)) - 1) < 1.5e-4)


def test_far_negative_is_tiny_and_nonnegative():
    x = np.array([-126.0, -127.0, -500.0, -np.inf], dtype=np.float32)
    got = exp2_poly(x)
    assert np.all(got >= 0) and np.all(got < 2.0 ** -124)
