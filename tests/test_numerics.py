"""Numerics of the library's FMA-pipe exp2 building block.

The routine computes 2^x without the MUFU: x = j + f, j = round(x) via the
1.5 * 2^23 shifter, |f| <= 1/2, 2^f by a degree-3 polynomial, 2^j added to the
exponent field.  The softmax of the default tcgen05 kernel computes one weight pair
in eight with it and the unmasking scan one pair in four (the rest with the hardware
ex2.approx).  The CPU test re-derives the
error bound of the recipe with the coefficients the library uses (read from its
source) in float32 numpy; the GPU test checks the device routine against float64
exp2 through the self-test entry point."""
import os
import re

import numpy as np
import pytest

from two_tower_block_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def coefficients():
    src = open(os.path.join(ROOT, "two_tower_block_b200", "csrc", "ptx.cuh")).read()
    body = src[src.index("exp2_poly2(float2 x)"):]
    body = body[:body.index("return make_float2")]
    vals = [float(v) for v in re.findall(r"make_float2\(([0-9]\.[0-9]{6,})f, \1f\)", body)]
    # Horner order in the source: c3, c2, then c1, then c0
    c3, c2, c1, c0 = vals
    return np.float32(c0), np.float32(c1), np.float32(c2), np.float32(c3)


def exp2_recipe(x):
    """The same steps in float32 numpy (round-to-nearest float32 arithmetic)."""
    c0, c1, c2, c3 = coefficients()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    sh = np.float32(12582912.0)
    t = (x + sh).astype(np.float32)
    j = (t - sh).astype(np.float32)
    f = (x - j).astype(np.float32)
    q = (c3 * f + c2).astype(np.float32)
    q = (q * f + c1).astype(np.float32)
    q = (q * f + c0).astype(np.float32)
    jb = (t.view(np.uint32) << np.uint32(23)).astype(np.uint32)
    return (q.view(np.uint32) + jb).view(np.float32)


def test_exp2_recipe_error_bound_cpu():
    x = np.concatenate([np.linspace(-125, 127, 400001, dtype=np.float32),
                        np.random.default_rng(0).uniform(-30, 9, 200000).astype(np.float32)])
    y = exp2_recipe(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 1.0e-4, rel.max()          # bf16 half-ulp is 2^-9 ~ 2e-3
    assert exp2_recipe(np.float32(-np.inf)) == pytest.approx(2.0 ** -125, rel=1e-4)  # clamped
    assert exp2_recipe(np.float32(0.0)) == pytest.approx(1.0, rel=1e-4)


@pytest.mark.gpu
def test_exp2_device_matches_recipe_and_bound():
    x = np.concatenate([np.linspace(-125, 127, 100001, dtype=np.float32),
                        np.random.default_rng(1).uniform(-30, 9, 100001).astype(np.float32)])
    y = ops.selftest_exp2(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 1.0e-4, rel.max()
    # same float32 steps on both sides (FMA contraction may differ by an ulp)
    np.testing.assert_allclose(y, exp2_recipe(x).astype(np.float64), rtol=2e-7, atol=0)
