"""The softmax's FMA-pipe exp2 (sm100.cuh: exp2_poly) evaluated bit-for-bit in float32 on the CPU:
relative error against exp2 stays below 1e-4 over the whole range the softmax feeds it, and the
clamp keeps very negative inputs (masked logits) at a tiny positive normal value."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "free_sparse_attention_block_b200", "csrc", "sm100.cuh")


def coeffs():
    body = open(SRC).read().split("exp2_poly(float x)")[1].split("}")[0]
    c = [float(v) for v in re.findall(r"([0-9]\.[0-9]+)f", body)]
    # fmaf(fmaf(fmaf(c3, f, c2), f, c1), f, c0)
    return np.float32(c[-1]), np.float32(c[-2]), np.float32(c[-3]), np.float32(c[-4])


def exp2_poly(x):
    c0, c1, c2, c3 = coeffs()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    f = (x - (t - shift).astype(np.float32)).astype(np.float32)
    p = (((c3 * f + c2).astype(np.float32) * f + c1).astype(np.float32) * f + c0).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_relative_error_over_softmax_range():
    x = np.linspace(-60.0, 8.0, 2_000_001).astype(np.float32)
    got = exp2_poly(x).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1e-4


def test_clamp_of_masked_logits():
    y = exp2_poly(np.array([-np.inf, -1e30, -200.0, -125.0], np.float32))
    assert np.all(np.isfinite(y)) and np.all(y > 0) and np.all(y < 1e-37)


def test_integers_are_near_exact():
    for n in range(-100, 9):
        assert abs(float(exp2_poly(np.float32(n))) / 2.0 ** n - 1) < 1e-4
