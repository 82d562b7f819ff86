"""Pins for oracle O5 (EAGLE-2 reranking) against checks other than its own definition.

The reading (EAGLE-2 blog, section 1: the confidence approximates the probability that the
target accepts a draft token; section 4: reranking keeps the tokens most likely to be
accepted) is that a candidate's value is the product of the confidences along its path and
the m highest-valued candidates form the verified tree.  Checks:
  * closed forms: a chain keeps its first m nodes; equal confidences keep the shallowest
    nodes (breadth-first, then index); confidence 1 everywhere keeps indices 0..m-1; a star
    keeps the root and its m-1 most confident children;
  * on random trees whose path values (float64, computed here) are well separated, every
    kept candidate outvalues every dropped one;
  * the kept set contains each kept node's ancestors, the output is a topological tree,
    and the ancestor masks equal the transitive closure of that tree's parent relation
    (boolean matrix powers in numpy);
  * NaN and negative confidences count as 0, values above 1 as 1; a tree that is not
    topological gives -1; m beyond the candidate count keeps everything.
"""
import numpy as np
import pytest

import workloads as wl


def _closure_masks(parents_out, k):
    """Ancestor-or-self masks by transitive closure of the parent relation (matrix powers)."""
    A = np.zeros((k, k), bool)
    for t in range(1, k):
        A[t, parents_out[t]] = True
    R = np.eye(k, dtype=bool) | A
    for _ in range(k):
        R = R | (R.astype(np.int64) @ R.astype(np.int64) > 0)
    return [sum(1 << j for j in range(k) if R[t, j]) for t in range(k)]


def _check_structure(res, parents, tokens, b, m):
    k = int(res["num_selected"][b])
    sel = res["sel"][b, :k]
    assert sel[0] == 0 and (np.diff(sel) > 0).all()
    kept = set(int(i) for i in sel)
    for i in kept:
        if i:
            assert int(parents[b, i]) in kept  # ancestor-closed
    po = res["parents"][b, :k]
    assert po[0] == -1 and all(0 <= po[t] < t for t in range(1, k))
    for t in range(1, k):
        assert sel[po[t]] == parents[b, sel[t]]
    np.testing.assert_array_equal(res["tokens"][b, :k], tokens[b, sel])
    assert [int(x) for x in res["masks"][b, :k]] == _closure_masks(po, k)
    assert (res["sel"][b, k:] == -1).all() and (res["masks"][b, k:] == 0).all()
    return sel


@pytest.mark.parametrize("M,m", [(20, 7), (1024, 64)])
def test_chain_keeps_its_prefix(orc, M, m):
    par = wl.chain_parents(M - 1)[None]
    rng = np.random.default_rng(1)
    conf = rng.uniform(0.05, 0.95, (1, M)).astype(np.float32)
    tok = rng.integers(0, 1000, (1, M)).astype(np.int32)
    res = orc.tree_rerank(par, tok, conf, m)
    assert res["num_selected"][0] == m
    np.testing.assert_array_equal(_check_structure(res, par, tok, 0, m), np.arange(m))


@pytest.mark.parametrize("M,m", [(40, 13), (300, 64)])
def test_equal_confidence_keeps_shallowest(orc, M, m):
    rng = np.random.default_rng(2)
    B = 4
    par = np.stack([wl.random_parents(rng, M, 5) for _ in range(B)])
    tok = rng.integers(0, 1000, (B, M)).astype(np.int32)
    conf = np.full((B, M), 0.5, np.float32)
    res = orc.tree_rerank(par, tok, conf, m)
    for b in range(B):
        depth = np.zeros(M, int)
        for i in range(1, M):
            depth[i] = depth[par[b, i]] + 1
        want = sorted(sorted(range(M), key=lambda i: (depth[i], i))[:m])
        np.testing.assert_array_equal(_check_structure(res, par, tok, b, m), want)


def test_confidence_one_keeps_first_indices(orc):
    rng = np.random.default_rng(3)
    par = np.stack([wl.random_parents(rng, 30, 6) for _ in range(3)])
    tok = rng.integers(0, 99, (3, 30)).astype(np.int32)
    res = orc.tree_rerank(par, tok, np.ones((3, 30), np.float32), 9)
    for b in range(3):
        np.testing.assert_array_equal(_check_structure(res, par, tok, b, 9), np.arange(9))


def test_star_keeps_most_confident_children(orc):
    M, m = 16, 6
    par = np.array([[-1] + [0] * (M - 1)], np.int32)
    conf = np.linspace(0.9, 0.1, M, dtype=np.float32)[None]
    conf[0, 1:] = np.random.default_rng(4).permutation(conf[0, 1:])
    tok = np.arange(M, dtype=np.int32)[None] * 3
    res = orc.tree_rerank(par, tok, conf, m)
    best = sorted(np.argsort(-conf[0, 1:])[:m - 1] + 1)
    np.testing.assert_array_equal(_check_structure(res, par, tok, 0, m), [0] + best)


@pytest.mark.parametrize("seed,M,m", [(s, 60, 20) for s in range(4)] + [(9, 500, 64), (10, 1024, 45)])
def test_kept_outvalue_dropped(orc, seed, M, m):
    rng = np.random.default_rng(100 + seed)
    B = 3
    par = np.stack([wl.random_parents(rng, M, 6) for _ in range(B)])
    tok = rng.integers(0, 1000, (B, M)).astype(np.int32)
    conf = rng.uniform(0.02, 1.0, (B, M)).astype(np.float32)
    res = orc.tree_rerank(par, tok, conf, m)
    for b in range(B):
        v = np.ones(M)
        for i in range(1, M):
            v[i] = v[par[b, i]] * float(conf[b, i])
        sel = set(int(i) for i in _check_structure(res, par, tok, b, m))
        kept = [v[i] for i in sel]
        dropped = [v[i] for i in range(M) if i not in sel]
        gap = min(kept) - max(dropped)
        # ties are broken by index; a near-tie is beyond what float32 decides identically
        assert gap > -1e-6 * max(kept), (b, min(kept), max(dropped))


def test_clamping_and_degenerate_inputs(orc):
    M = 8
    par = np.array([[-1, 0, 1, 2, 0, 4, 5, 6],
                    [-1, 0, 1, 2, 0, 4, 5, 6],
                    [-1, 0, 0, 2, 3, 9, 0, 0],    # parent 9 > index: not topological
                    [-1, 0, 1, 2, 0, 4, 5, 6]], np.int32)
    tok = np.arange(4 * M, dtype=np.int32).reshape(4, M)
    conf = np.array([[1, .5, .5, .5, np.nan, .9, .9, .9],      # NaN: the 4-5-6-7 chain is worth 0
                     [1, .5, .5, .5, -3.0, .9, .9, .9],          # negative: likewise
                     [1] * M,
                     [1, 2.0, .5, .5, .7, .9, .9, .9]], np.float32)  # 2.0 counts as 1
    res = orc.tree_rerank(par, tok, conf, 5)
    for b in (0, 1):
        np.testing.assert_array_equal(_check_structure(res, par, tok, b, 5), [0, 1, 2, 3, 4])
    assert res["num_selected"][2] == -1 and (res["sel"][2] == -1).all()
    # values: 1: 1, 2: .5, 3: .25, 4: .7, 5: .63, 6: .567, 7: .5103
    np.testing.assert_array_equal(_check_structure(res, par, tok, 3, 5), [0, 1, 4, 5, 6])
    every = orc.tree_rerank(par[:1], tok[:1], conf[3:], 12)
    assert every["num_selected"][0] == M
    np.testing.assert_array_equal(_check_structure(every, par[:1], tok[:1], 0, 12), np.arange(M))
