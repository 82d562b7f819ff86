"""Pins for the oracle's sampler and counter-based uniforms.

The exponential race (argmin_v E_v / w_v with E_v = -ln U_v) draws index v with
probability w_v / sum(w) -- a standard property of independent exponentials; the
chi-square test checks it, so a wrong sign, a log of the wrong quantity or a
biased uniform fails.  The Philox words are checked for the uniform mapping
(odd multiples of 2^-24, strictly inside (0, 1)), for uniformity and for
independence between counters.  Their exact values are pinned on the GPU
against cuRAND's Philox4x32-10, an implementation other than this one.
"""
import numpy as np
import pytest
from scipy import stats


def test_uniform_mapping_is_exact_and_open(orc):
    u = orc.uniforms(123, 0, 0, 0, 1, 4096)
    scaled = u * 2.0 ** 24
    np.testing.assert_array_equal(scaled, np.round(scaled))
    assert (np.round(scaled).astype(np.int64) % 2 == 1).all()
    assert (u > 0).all() and (u < 1).all()
    assert np.array_equal(u.astype(np.float32).astype(np.float64), u)  # exact in float32


def test_uniforms_are_uniform_and_counter_sensitive(orc):
    u = np.concatenate([orc.uniforms(7, off, b, node, 1, 4000)
                        for off in range(3) for b in range(5) for node in range(4)])
    counts, _ = np.histogram(u, bins=50, range=(0, 1))
    assert stats.chisquare(counts).pvalue > 0.001
    # every counter field changes the stream
    base = orc.uniforms(7, 0, 0, 0, 1, 64)
    for args in [(8, 0, 0, 0, 1), (7, 1, 0, 0, 1), (7, 0, 1, 0, 1), (7, 0, 0, 1, 1), (7, 0, 0, 0, 0)]:
        other = orc.uniforms(*args, 64)
        assert np.mean(base == other) < 0.05
    # lag-1 correlation of consecutive words is small
    assert abs(np.corrcoef(u[:-1], u[1:])[0, 1]) < 0.01


def test_uniform_uses_all_four_words(orc):
    # v and v+1 with the same v >> 2 come from different words of one Philox call
    ctr = np.array([0, (3 << 16) | (1 << 8) | 5, 9, 0], np.uint32)
    words = orc.philox(ctr, [11, 0])
    for v in range(4):
        expect = (2.0 * (int(words[v]) >> 9) + 1.0) * 2.0 ** -24
        assert orc.uniform(11, 9, 3, 5, v, 1) == expect


@pytest.mark.slow
def test_race_samples_normalised_weights(orc):
    w = np.array([3.0, 0.0, 1.0, 0.5, 2.5, 0.0, 1e-3, 7.0])
    n = 200_000
    idx = np.array([orc.race(w, 21, off, b, 3)[0] for off in range(n // 20_000) for b in range(20_000)])
    counts = np.bincount(idx, minlength=len(w))
    assert counts[1] == 0 and counts[5] == 0
    keep = w > 0
    assert stats.chisquare(counts[keep], w[keep] / w.sum() * n).pvalue > 0.01


def test_race_ignores_normalisation_and_reports_gap(orc):
    w = np.array([0.2, 0.5, 0.3])
    a = orc.race(w, 1, 2, 3, 4)
    b = orc.race(w * 123.0, 1, 2, 3, 4)
    assert a[0] == b[0]
    assert a[1] == pytest.approx(b[1], rel=1e-12) and a[1] > 0
    assert orc.race(np.array([0.0, 0.0, 5.0]), 1, 2, 3, 4)[0] == 2
