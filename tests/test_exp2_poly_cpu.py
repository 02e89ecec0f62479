"""The FMA-pipe exp2 of the attention softmax (exp2_poly2 in the tcgen05 attention
kernel): its polynomial constants are re-derived here from their definition (the
degree-3 polynomial of least maximum relative error for 2^f on [-1/2, 1/2], found by
Lawson's iteratively reweighted least squares), and the whole evaluation (Cody-Waite
split by the 1.5 * 2^23 rounding constant, polynomial, exponent-field scaling, the -125
clamp) is replayed step by step in fp32 and compared with exp2 in fp64."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "hybrid_head_ssm_b200", "csrc", "attn_tc.cu")


def _constants():
    src = open(SRC).read()
    m = re.search(r"EXP2_C0 = ([0-9.eE+-]+)f, EXP2_C1 = ([0-9.eE+-]+)f, EXP2_C2 = ([0-9.eE+-]+)f, "
                  r"EXP2_C3 = ([0-9.eE+-]+)f", src)
    assert m, "constants not found"
    return np.array([float(v) for v in m.groups()])


def _lawson(deg, iters=300):
    x = np.linspace(-0.5, 0.5, 20001)
    y = np.exp2(x)
    V = np.vander(x, deg + 1, increasing=True)
    w = np.ones_like(x)
    for _ in range(iters):
        c, *_ = np.linalg.lstsq(V * (w / y)[:, None], w, rcond=None)
        e = (V @ c - y) / y
        w = w * np.sqrt(np.abs(e)) + 1e-30
        w /= w.max()
    return c, np.abs(e).max()


def _exp2_poly_fp32(x, c):
    """The kernel's steps in fp32 (FADD2 / FFMA2 rounding emulated by float32 ops)."""
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-125.0))
    magic = f32(12582912.0)
    t = (x + magic).astype(f32)
    f = (x + (magic + (-t)).astype(f32)).astype(f32)
    p = (f32(c[3]) * f + f32(c[2])).astype(f32)
    p = (p * f + f32(c[1])).astype(f32)
    p = (p * f + f32(c[0])).astype(f32)
    j = t.view(np.int32) - np.int32(0x4B400000)
    return (p.view(np.int32) + (j << 23)).view(np.float32)


def test_constants_are_the_minimax_fit():
    c_fit, err = _lawson(3)
    c = _constants()
    np.testing.assert_allclose(c, c_fit, rtol=0, atol=1e-6)  # the iteration converges to ~1e-7
    assert err < 8e-5


def test_fp32_evaluation_error_below_fp16_half_ulp():
    c = _constants()
    g = np.random.default_rng(3)
    x = np.concatenate([np.linspace(-30.0, 16.0, 200001), g.uniform(-24.0, 8.0, 100000),
                        np.arange(-24, 17, dtype=np.float64)])
    got = _exp2_poly_fp32(x, c).astype(np.float64)
    want = np.exp2(x.astype(np.float32).astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 1.0e-4, rel.max()  # fp16 (the P operand) half-ulp is 4.9e-4


def test_masked_and_tiny_arguments_vanish_in_fp16():
    c = _constants()
    x = np.array([-np.inf, -1e30, -200.0, -125.0, -40.0], dtype=np.float32)
    got = _exp2_poly_fp32(x, c)
    assert np.all(got >= 0) and np.all(np.isfinite(got))
    assert np.all(got.astype(np.float16) == 0)
    assert got.max() < 1e-11
