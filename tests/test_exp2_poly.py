"""The polynomial 2^x that the tree-attention softmax uses for part of its exponentials
(`exp2_poly2` in csrc/device_common.cuh), re-evaluated in float32 on the CPU from the
constants in that source, against 2^x in float64: range reduction y = j + f, a cubic for 2^f
on [-1/2, 1/2], 2^j built in the exponent field, and exact zero below the clamp."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tree_verify_b200", "csrc", "device_common.cuh")


def _constants():
    text = open(SRC).read()
    body = text[text.index("float2 exp2_poly2(float2 y)"):]
    body = body[:body.index("\n}\n")]
    shift = float(re.search(r"kShift = ([0-9.e+-]+)f", body).group(1))
    clamp = float(re.search(r"fmaxf\(y\.x, (-[0-9.]+)f\)", body).group(1))
    c3, c2 = (float(v) for v in re.search(r"make_float2\(([0-9.]+)f, \1f\), f, make_float2\(([0-9.]+)f", body).group(1, 2))
    c1 = float(re.search(r"ffma2\(q, f, make_float2\(([0-9.]+)f, \1f\)\);\n  q = ffma2\(q, f, make_float2\(1\.0f", body).group(1))
    return shift, clamp, c1, c2, c3


def _exp2_poly(y):
    shift, clamp, c1, c2, c3 = (np.float32(v) for v in _constants())
    y = np.maximum(y.astype(np.float32), clamp)
    t = (y + shift).astype(np.float32)
    j = (t - shift).astype(np.float32)
    f = (y - j).astype(np.float32)
    q = ((c3 * f + c2) * f + c1) * f + np.float32(1.0)
    bits = (t.view(np.uint32).astype(np.uint64) << np.uint64(23)) + np.uint64(0x3F800000)
    sc = (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)
    return (q.astype(np.float32) * sc).astype(np.float32)


def test_constants_are_a_fit_of_2_to_the_x():
    shift, clamp, c1, c2, c3 = _constants()
    assert shift == 1.5 * 2 ** 23 and clamp == -127.0
    # a cubic near the Taylor series of 2^f (ln 2, ln^2 2 / 2, ln^3 2 / 6), nudged for
    # minimum relative error over the interval
    ln2 = np.log(2.0)
    assert abs(c1 - ln2) < 2e-3 and abs(c2 - ln2 ** 2 / 2) < 5e-3 and abs(c3 - ln2 ** 3 / 6) < 5e-3


def test_relative_error_over_the_softmax_range():
    # the softmax evaluates 2^(s c - m) <= 2^8 (lazy rescaling); below -126 the result is
    # far under any P that matters
    y = np.concatenate([np.linspace(-126.0, 8.0, 400_001), np.arange(-126, 9, dtype=np.float64)])
    got = _exp2_poly(y).astype(np.float64)
    want = np.exp2(y.astype(np.float32).astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 1.1e-4
    # integers are exact up to the cubic's value at f = 0
    ints = np.arange(-126, 9, dtype=np.float32)
    assert np.all(_exp2_poly(ints) == np.exp2(ints))


def test_masked_scores_give_exact_zero():
    y = np.array([-np.inf, -1e30, -200.0, -127.0, -126.6], dtype=np.float32)
    assert np.all(_exp2_poly(y) == 0.0)
    assert _exp2_poly(np.array([-126.0], np.float32))[0] > 0.0
