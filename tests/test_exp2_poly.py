"""Error bound of the attention kernel's polynomial 2^x (exp2_poly in
attn_partial.cu), restated operation by operation in float32 (each fused
multiply-add evaluated exactly in float64 and rounded once, as the GPU's
FFMA does) and compared with numpy's exp2 in float64.

The kernel feeds these values, rounded to bf16 (relative step 2^-8), into
the P V product, so a relative error of 1.1e-4 is far below what the output
tolerance allows."""
import re
import os

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(__file__)), "sparse_state_reuse_b200", "csrc",
                   "attn_partial.cu")


def coeffs():
    text = open(SRC).read()
    return [np.float32(float(re.search(rf"kExpC{i} = ([0-9.e+-]+)f", text).group(1)))
            for i in (1, 2, 3)]


def fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly(x):
    c1, c2, c3 = coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    kr = np.float32(12582912.0)
    t = (x + kr).astype(np.float32)
    n = (t - kr).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = fma32(fma32(fma32(np.full_like(f, c3), f, np.full_like(f, c2)), f, np.full_like(f, c1)), f,
              np.ones_like(f))
    bits = p.view(np.int32) + (t.view(np.int32) << np.int32(23))
    return bits.astype(np.int32).view(np.float32)


def test_relative_error_bound_over_softmax_range():
    x = np.linspace(-100.0, 8.0, 2_000_001, dtype=np.float32)
    y = exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 1.1e-4, rel.max()


def test_integers_are_exact_and_tiny_inputs_vanish():
    k = np.arange(-120, 9, dtype=np.float32)
    np.testing.assert_array_equal(exp2_poly(k), np.exp2(k.astype(np.float64)).astype(np.float32))
    z = exp2_poly(np.array([-np.inf, -1e30, -200.0], dtype=np.float32))
    assert (z >= 0).all() and (z < 2e-38).all()


def test_monotone_on_a_fine_grid():
    x = np.linspace(-20.0, 8.0, 1_000_001, dtype=np.float32)
    y = exp2_poly(x)
    assert (np.diff(y.astype(np.float64)) >= -1e-4 * y[1:]).all()
