"""Pins for oracle O6 (children of draft nodes) against library routines and statistics.

EAGLE summary, appendix A.1 "Tree Structure": in greedy decoding the children are the top k
tokens by probability, in non-greedy decoding k tokens are sampled.  Checks:
  * T = 0: the tokens equal numpy's stable descending argsort of the logits (ties to the
    lower index), the confidences scipy's softmax at those tokens;
  * T > 0: the row distribution equals scipy's softmax(logits / T); over many offsets
    each of the k samples follows it (chi-square), two samples of one row are independent
    (chi-square of the joint histogram against the outer product), and a sample's
    confidence is its probability.
"""
import numpy as np
import pytest
from scipy import special, stats


def test_greedy_is_sorted_top_k(orc):
    rng = np.random.default_rng(1)
    B, F, V, k = 3, 4, 500, 10
    logits = rng.standard_normal((B, F, V)).astype(np.float32)
    logits[0, 0, 10:20] = 8.0  # a run of ties above every other value
    res = orc.draft_select(logits, 0.0, k, with_probs=True)
    for b in range(B):
        for f in range(F):
            want = np.argsort(-logits[b, f], kind="stable")[:k]
            np.testing.assert_array_equal(res["tokens"][b, f], want)
            p = special.softmax(logits[b, f].astype(np.float64))
            np.testing.assert_allclose(res["conf"][b, f], p[want], rtol=1e-12)
            np.testing.assert_allclose(res["probs"][b, f], p, rtol=1e-12)
    np.testing.assert_array_equal(res["tokens"][0, 0], np.arange(10, 20))


@pytest.mark.parametrize("T", [0.6, 1.0, 2.5])
def test_sampled_children_follow_p(orc, T):
    logits = np.array([[[1.0, 0.2, -0.5, 2.0, 0.0, -1.5]]], np.float32)
    V, k, n = logits.shape[-1], 3, 12000
    p = special.softmax(logits[0, 0].astype(np.float64) / T)
    first = np.zeros(V)
    last = np.zeros(V)
    joint = np.zeros((V, V))
    for off in range(n):
        res = orc.draft_select(logits, T, k, seed=7, offset=off, with_probs=off == 0)
        if off == 0:
            np.testing.assert_allclose(res["probs"][0, 0], p, rtol=1e-12)
        t = res["tokens"][0, 0]
        np.testing.assert_allclose(res["conf"][0, 0], p[t], rtol=1e-12)
        first[t[0]] += 1
        last[t[-1]] += 1
        joint[t[0], t[1]] += 1
    assert stats.chisquare(first, n * p).pvalue > 0.01
    assert stats.chisquare(last, n * p).pvalue > 0.01
    assert stats.chisquare(joint.ravel(), n * np.outer(p, p).ravel()).pvalue > 0.01
