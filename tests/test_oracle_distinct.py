"""Pins for oracle O7 (siblings drawn without replacement) and the study it serves.

EAGLE summary, appendix A.1 "Tree Structure": in non-greedy decoding k tokens are sampled for
a node's children; drawn without replacement, the siblings are distinct.  Checks:
  * T = 0 equals O6's top k;
  * T > 0: siblings are distinct; over many draws the first follows p and the ordered pair
    of the first two follows the law of successive draws without replacement,
    p_a * p_b / (1 - p_a) (chi-square); each confidence is its probability;
  * the row a sibling was drawn from is p renormalised without the earlier siblings (numpy);
  * the residual rule (the accept walk, O3) preserves p when every sibling's draft row is
    the row it was drawn from, and does not when the siblings share the parent's row
    (chi-square of the first emitted token over 200,000 seeded trees).
"""
import numpy as np
import pytest
from scipy import special, stats

CHUNK = 50000  # sequences per oracle call (the Philox counter holds 16 bits of sequence)


def _p(logits, T=1.0):
    return special.softmax(np.asarray(logits, np.float64) / T)


def test_distinct_at_t0_is_the_top_k(orc):
    lg = np.random.default_rng(5).standard_normal((2, 3, 40)).astype(np.float32)
    a = orc.draft_select(lg, 0.0, 6)
    b = orc.draft_select_distinct(lg, 0.0, 6)
    np.testing.assert_array_equal(a["tokens"], b["tokens"])
    np.testing.assert_array_equal(a["conf"], b["conf"])


def test_siblings_are_successive_draws_without_replacement(orc):
    logits = np.array([1.0, 0.2, -0.5, 2.0, 0.0, -1.5], np.float32)
    p = _p(logits, 0.8)
    V, k = len(p), 3
    first = np.zeros(V)
    pair = np.zeros((V, V))
    for off in range(4):
        lg = np.tile(logits, (CHUNK, 1, 1))
        r = orc.draft_select_distinct(lg, 0.8, k, seed=3, offset=off, with_probs=off == 0)
        t = r["tokens"][:, 0]
        assert (t[:, 0] != t[:, 1]).all() and (t[:, 0] != t[:, 2]).all() and (t[:, 1] != t[:, 2]).all()
        np.testing.assert_allclose(r["conf"][:, 0], p[t], rtol=1e-12)
        if off == 0:
            np.testing.assert_allclose(r["probs"][0, 0], p, rtol=1e-12)
        first += np.bincount(t[:, 0], minlength=V)
        np.add.at(pair, (t[:, 0], t[:, 1]), 1)
    n = first.sum()
    assert stats.chisquare(first, n * p).pvalue > 0.01
    law = p[:, None] * p[None, :] / (1.0 - p[:, None])
    np.fill_diagonal(law, 0.0)
    mask = ~np.eye(V, dtype=bool)
    assert stats.chisquare(pair[mask], n * law[mask]).pvalue > 0.01


def test_fewer_choosable_tokens_than_siblings(orc):
    lg = np.array([[[0.0, -np.inf, 1.0, -np.inf]]], np.float32)
    r = orc.draft_select_distinct(lg, 1.0, 4, seed=1)
    assert sorted(r["tokens"][0, 0, :2].tolist()) == [0, 2]
    assert (r["tokens"][0, 0, 2:] == -1).all() and (r["conf"][0, 0, 2:] == 0).all()


def test_child_rows_renormalise_without_earlier_siblings(orc):
    rng = np.random.default_rng(9)
    B, F, V, k = 2, 3, 12, 4
    probs = rng.dirichlet(np.ones(V), (B, F))
    tokens = np.stack([np.stack([rng.permutation(V)[:k] for _ in range(F)]) for _ in range(B)]).astype(np.int32)
    tokens[1, 2, 2:] = -1  # a row that ran out of choosable tokens
    rows = orc.draft_child_rows(probs, tokens)
    for b in range(B):
        for f in range(F):
            for j in range(k):
                gone = tokens[b, f, :j]
                if (gone < 0).any():
                    assert (rows[b, f, j] == 0).all()
                    continue
                want = probs[b, f].copy()
                want[gone] = 0.0
                want /= want.sum()
                np.testing.assert_allclose(rows[b, f, j], want, rtol=1e-12, atol=0)
    np.testing.assert_allclose(rows[:, :, 0], probs, rtol=1e-12)


def _first_emitted(orc, q_logits, p_logits, k, conditioned, seed=0):
    """Counts of the first emitted token over 4 * CHUNK trees: a root whose k children are
    drawn without replacement from softmax(q_logits), verified by the walk against
    softmax(p_logits) with the children's draft rows either conditioned or shared."""
    V = len(q_logits)
    counts = np.zeros(V, np.int64)
    N = k + 1
    parents = np.tile(np.array([-1] + [0] * k, np.int32), (CHUNK, 1))
    logits = np.zeros((CHUNK, N, V), np.float32)
    logits[:] = np.asarray(p_logits, np.float32)
    for off in range(4):
        d = orc.draft_select_distinct(np.tile(np.asarray(q_logits, np.float32), (CHUNK, 1, 1)), 1.0, k,
                                      seed=seed, offset=off, with_probs=True)
        tokens = np.zeros((CHUNK, N), np.int32)
        tokens[:, 1:] = d["tokens"][:, 0]
        dp = np.zeros((CHUNK, N, V), np.float32)
        dp[:, 1:] = (orc.draft_child_rows(d["probs"], d["tokens"])[:, 0] if conditioned
                     else d["probs"][:, 0][:, None, :])
        res = orc.tree_accept(dp, tokens, parents, 1.0, seed, off, logits=logits)
        acc, alen = res["accepted_nodes"], res["accept_len"]
        first = np.where(alen >= 1, tokens[np.arange(CHUNK), np.maximum(acc[:, 0], 0)], res["next_token"])
        counts += np.bincount(first, minlength=V)
    return counts


CASES = [([2.0, 1.0, 0.0, -1.0], [0.0, 0.5, 1.0, 1.5], 2),
         ([1.5, 1.2, 0.2, 0.0, -0.5], [0.3, 0.0, 1.0, 0.2, 0.9], 3)]


@pytest.mark.parametrize("q_logits,p_logits,k", CASES)
def test_residual_rule_preserves_p_with_conditioned_rows(orc, q_logits, p_logits, k):
    counts = _first_emitted(orc, q_logits, p_logits, k, conditioned=True)
    p = _p(p_logits)
    assert stats.chisquare(counts, counts.sum() * p).pvalue > 0.01


@pytest.mark.parametrize("q_logits,p_logits,k", CASES)
def test_residual_rule_with_shared_rows_does_not(orc, q_logits, p_logits, k):
    counts = _first_emitted(orc, q_logits, p_logits, k, conditioned=False)
    p = _p(p_logits)
    assert stats.chisquare(counts, counts.sum() * p).pvalue < 1e-6


def test_child_rows_sum_the_remaining_mass_directly(orc):
    """When the earlier siblings carry all but ~1e-9 of the mass, 1 minus their mass loses
    most of the digits of what remains; the rows must still be the exact renormalisation."""
    V, k = 64, 3
    p = np.full(V, 1e-11)
    p[[5, 9]] = 0.5 - 16e-11
    p /= p.sum()
    tokens = np.array([[[5, 9, 2]]], np.int32)
    rows = orc.draft_child_rows(p[None, None], tokens)
    rest = np.delete(np.arange(V), [5, 9])
    want = np.zeros(V)
    want[rest] = p[rest] / p[rest].sum()
    np.testing.assert_allclose(rows[0, 0, 2], want, rtol=1e-12, atol=0)
    assert abs(rows[0, 0, 2].sum() - 1.0) < 1e-12
