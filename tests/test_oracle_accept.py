"""Pins for oracle O3 (the accept/resample tree walk).

What the pages fix and what each test checks:
  * EAGLE summary, section 2 "Preliminaries" and appendix B (Algorithm 1): the
    procedure returns a sample of the *target* distribution.  Chi-square tests on
    10^6 seeded trials check the first emitted token (k = 1, 2, 4 candidates) and the
    joint law of the first two emitted tokens on a depth-2 tree.
  * The single-candidate rule min(1, p/p_hat) accepts with total probability
    sum_x min(p(x), p_hat(x)) (closed form of the textbook rule).
  * p_hat == p accepts every candidate; a one-hot p_hat on a token with p = 0 rejects
    every candidate and the emitted token is distributed as p.
  * Temperature 0 is greedy: the accepted path is the argmax-matching path, found here
    by brute force over every root-to-node path (EAGLE-2 blog, section 1; EAGLE summary,
    section 4).
A sign error in the ratio test, a residual p_hat - p, the parent's draft row used
instead of the candidate's, or a missed residual update each fails one of these.
"""
import numpy as np
import pytest
from scipy import stats

import workloads as wl

TRIALS = 1_000_000
CHUNK = 50_000  # sequences per oracle call (the counter holds b in 16 bits)


def _softmax(x):
    x = np.asarray(x, dtype=np.float64)
    e = np.exp(x - x.max())
    return e / e.sum()


def _first_tokens(res, tokens):
    B = tokens.shape[0]
    first = res["next_token"].copy()
    has = res["accept_len"] > 0
    first[has] = tokens[np.arange(B)[has], res["accepted_nodes"][has, 0]]
    return first


def _chi2_pvalue(counts, probs):
    n = counts.sum()
    keep = probs > 0
    assert counts[~keep].sum() == 0, "token with zero target probability was emitted"
    return stats.chisquare(counts[keep], probs[keep] * n).pvalue


@pytest.mark.slow
@pytest.mark.parametrize("k", [1, 2, 4])
@pytest.mark.parametrize("T", [1.0, 0.6])
def test_first_token_distribution_is_target(orc, k, T):
    rng = np.random.default_rng(100 + k)
    V = 8
    logits_row = rng.standard_normal(V) * 1.5
    p = _softmax(logits_row / T)
    q = _softmax(rng.standard_normal(V) * 1.5)  # draft distribution, full support
    N = k + 1
    counts = np.zeros(V, dtype=np.int64)
    for chunk in range(TRIALS // CHUNK):
        par = np.tile(np.array([-1] + [0] * k, np.int32), (CHUNK, 1))
        tokens = np.zeros((CHUNK, N), np.int32)
        tokens[:, 1:] = rng.choice(V, size=(CHUNK, k), p=q)
        draft = np.zeros((CHUNK, N, V), np.float32)
        draft[:, 0] = 1.0 / V  # row 0 is never a candidate's row; make it differ from q
        draft[:, 1:] = q.astype(np.float32)
        logits = np.zeros((CHUNK, N, V), np.float64)
        logits[:, 0] = logits_row
        res = orc.tree_accept(draft, tokens, par, T, seed=17, offset=chunk, logits=logits)
        counts += np.bincount(_first_tokens(res, tokens), minlength=V)
    # draft rows are float32: compare against the p the walk actually targets
    assert _chi2_pvalue(counts, p) > 0.01


@pytest.mark.slow
def test_two_token_joint_distribution(orc):
    """Depth-2 tree: the target's second-token law depends on the first token a
    (logits row of a depth-1 node = table[a]); the emitted pair must follow
    p0(a) * p1(b | a).  When the walk stops at the root, the second token is drawn
    from p1(. | a) directly, as the next verification step would."""
    rng = np.random.default_rng(202)
    V, k1, k2 = 6, 2, 2
    l0 = rng.standard_normal(V)
    l1 = rng.standard_normal((V, V)) * 1.2
    q0 = _softmax(rng.standard_normal(V))
    q1 = np.stack([_softmax(rng.standard_normal(V)) for _ in range(V)])
    p0 = _softmax(l0)
    p1 = np.stack([_softmax(r) for r in l1])
    # node layout: 0 root, 1..k1 depth 1, then k2 children for each depth-1 node
    par = [-1] + [0] * k1
    for a in range(1, k1 + 1):
        par += [a] * k2
    par = np.array(par, np.int32)
    N = len(par)
    counts = np.zeros((V, V), np.int64)
    for chunk in range(TRIALS // CHUNK):
        tokens = np.zeros((CHUNK, N), np.int32)
        tokens[:, 1:k1 + 1] = rng.choice(V, size=(CHUNK, k1), p=q0)
        draft = np.zeros((CHUNK, N, V), np.float32)
        draft[:, 0] = 1.0 / V
        draft[:, 1:k1 + 1] = q0.astype(np.float32)
        logits = np.zeros((CHUNK, N, V), np.float64)
        logits[:, 0] = l0
        for a in range(1, k1 + 1):
            ta = tokens[:, a]
            logits[:, a] = l1[ta]
            kids = [c for c in range(N) if par[c] == a]
            cdf = np.cumsum(q1[ta], axis=1)
            for c in kids:
                u = rng.random(CHUNK)[:, None]
                tokens[:, c] = np.minimum((cdf < u).sum(axis=1), V - 1)
                draft[:, c] = q1[ta].astype(np.float32)
        res = orc.tree_accept(draft, tokens, np.tile(par, (CHUNK, 1)), 1.0, seed=5,
                              offset=chunk, logits=logits)
        alen, acc, nxt = res["accept_len"], res["accepted_nodes"], res["next_token"]
        first = np.where(alen >= 1, tokens[np.arange(CHUNK), np.maximum(acc[:, 0], 0)], nxt)
        second = np.empty(CHUNK, np.int64)
        two = alen >= 2
        second[two] = tokens[np.arange(CHUNK)[two], acc[two, 1]]
        one = alen == 1
        second[one] = nxt[one]
        zero = alen == 0
        cdf = np.cumsum(p1[first[zero]], axis=1)
        second[zero] = np.minimum((cdf < rng.random(zero.sum())[:, None]).sum(axis=1), V - 1)
        np.add.at(counts, (first, second), 1)
    joint = p0[:, None] * p1
    assert _chi2_pvalue(counts.ravel(), joint.ravel()) > 0.01


@pytest.mark.slow
def test_single_candidate_acceptance_closed_form(orc):
    rng = np.random.default_rng(303)
    V = 10
    lrow = rng.standard_normal(V)
    p = _softmax(lrow)
    q = _softmax(rng.standard_normal(V) * 2.0)
    n_acc = 0
    for chunk in range(TRIALS // CHUNK):
        tokens = np.zeros((CHUNK, 2), np.int32)
        tokens[:, 1] = rng.choice(V, size=CHUNK, p=q)
        draft = np.zeros((CHUNK, 2, V), np.float32)
        draft[:, 1] = q.astype(np.float32)
        logits = np.zeros((CHUNK, 2, V))
        logits[:, 0] = lrow
        res = orc.tree_accept(draft, tokens, np.tile([-1, 0], (CHUNK, 1)), 1.0, seed=9,
                              offset=chunk, logits=logits)
        n_acc += int((res["accept_len"] == 1).sum())
    P = np.minimum(p, q.astype(np.float32).astype(np.float64)).sum()
    sigma = np.sqrt(TRIALS * P * (1 - P))
    assert abs(n_acc - TRIALS * P) < 5 * sigma


def test_draft_equal_to_target_accepts_everything(orc):
    # dyadic target: p = (1/2, 1/4, ..., 1/128, 1/128) is exact in float32
    V = 8
    p = np.array([2.0 ** -(i + 1) for i in range(V - 1)] + [2.0 ** -(V - 1)])
    rng = np.random.default_rng(4)
    B, n_draft = 20_000, 4
    N = n_draft + 1
    tokens = np.zeros((B, N), np.int32)
    tokens[:, 1:] = rng.choice(V, size=(B, n_draft), p=p)
    draft = np.zeros((B, N, V), np.float32)
    draft[:, 1:] = p.astype(np.float32)
    logits = np.tile(np.log(p), (B, N, 1))
    res = orc.tree_accept(draft, tokens, np.tile(wl.chain_parents(n_draft), (B, 1)), 1.0,
                          seed=1, logits=logits)
    assert (res["accept_len"] == n_draft).all()
    np.testing.assert_array_equal(res["accepted_nodes"][:, :n_draft],
                                  np.tile(np.arange(1, N), (B, 1)))
    # the bonus token after a full chain follows p
    counts = np.bincount(res["next_token"], minlength=V)
    assert _chi2_pvalue(counts, p) > 0.01


def test_impossible_candidates_all_rejected_next_follows_target(orc):
    rng = np.random.default_rng(6)
    V, k, B = 7, 3, 200_000
    lrow = rng.standard_normal(V)
    lrow[4] = -1000.0  # p(4) == 0 in float64
    p = _softmax(lrow)
    assert p[4] == 0.0
    N = k + 1
    tokens = np.zeros((B, N), np.int32)
    tokens[:, 1:] = 4
    draft = np.zeros((B, N, V), np.float32)
    draft[:, 1:, 4] = 1.0
    logits = np.zeros((B, N, V))
    logits[:, 0] = lrow
    counts = np.zeros(V, np.int64)
    for chunk in range(B // CHUNK):
        s = slice(chunk * CHUNK, (chunk + 1) * CHUNK)
        res = orc.tree_accept(draft[s], tokens[s], np.tile([-1] + [0] * k, (CHUNK, 1)), 1.0,
                              seed=3, offset=chunk, logits=logits[s])
        assert (res["accept_len"] == 0).all()
        counts += np.bincount(res["next_token"], minlength=V)
    assert _chi2_pvalue(counts, p) > 0.01


def _brute_force_greedy(parents, tokens, logits):
    """Deepest node whose every drafted ancestor (itself included) carries the argmax
    token of its parent's logits row; with distinct sibling tokens it is unique."""
    N = len(parents)
    am = logits.argmax(axis=-1)
    best, best_depth = 0, 0
    for node in range(1, N):
        path, a = [], node
        while a > 0:
            path.append(a)
            a = parents[a]
        if all(tokens[c] == am[parents[c]] for c in path) and len(path) > best_depth:
            best, best_depth = node, len(path)
    path, a = [], best
    while a > 0:
        path.append(a)
        a = parents[a]
    return path[::-1], int(am[best])


@pytest.mark.parametrize("seed", range(6))
def test_greedy_equals_brute_force_argmax_matching(orc, seed):
    rng = np.random.default_rng(seed)
    B, N, V = 64, 24, 12
    par = np.stack([wl.random_parents(rng, N, 5) for _ in range(B)])
    logits = rng.standard_normal((B, N, V)).astype(np.float32)
    tokens = np.zeros((B, N), np.int32)
    for b in range(B):
        ch = wl.children_lists(par[b])
        for u in range(N):
            if not ch[u]:
                continue
            # distinct sibling tokens; the argmax token is among them 60% of the time
            am = int(logits[b, u].argmax())
            cand = list(rng.permutation([t for t in range(V) if t != am])[:len(ch[u])])
            if rng.random() < 0.6:
                cand[rng.integers(0, len(cand))] = am
            for c, t in zip(ch[u], cand):
                tokens[b, c] = t
    draft = np.full((B, N, V), 1.0 / V, np.float32)
    res = orc.tree_accept(draft, tokens, par, 0.0, logits=logits)
    for b in range(B):
        path, nxt = _brute_force_greedy(par[b], tokens[b], logits[b])
        assert res["accept_len"][b] == len(path)
        assert list(res["accepted_nodes"][b, :len(path)]) == path
        assert (res["accepted_nodes"][b, len(path):] == -1).all()
        assert res["next_token"][b] == nxt


def test_greedy_chain_is_longest_matching_prefix(orc):
    rng = np.random.default_rng(12)
    B, n, V = 500, 7, 5
    logits = rng.standard_normal((B, n + 1, V))
    am = logits.argmax(-1)
    tokens = np.zeros((B, n + 1), np.int32)
    match = rng.random((B, n)) < 0.7
    tokens[:, 1:] = np.where(match, am[:, :-1], (am[:, :-1] + 1) % V)
    res = orc.tree_accept(np.zeros((B, n + 1, V), np.float32), tokens,
                          np.tile(wl.chain_parents(n), (B, 1)), 0.0, logits=logits)
    expect = np.argmin(np.concatenate([match, np.zeros((B, 1), bool)], 1), axis=1)
    np.testing.assert_array_equal(res["accept_len"], expect)
    np.testing.assert_array_equal(res["next_token"], am[np.arange(B), expect])


def test_greedy_ties_take_lowest_token(orc):
    logits = np.array([[[1.0, 3.0, 3.0, 0.0], [0, 0, 0, 0]]], np.float32)
    tokens = np.array([[0, 2]], np.int32)  # token 2 ties with 1 but 1 is the argmax
    res = orc.tree_accept(np.zeros((1, 2, 4), np.float32), tokens, [[-1, 0]], 0.0, logits=logits)
    assert res["accept_len"][0] == 0 and res["next_token"][0] == 1
    assert res["near"][0] == 1  # a tie is inside the margin


def test_invalid_tree_sentinels(orc):
    V = 4
    draft = np.full((3, 3, V), 0.25, np.float32)
    logits = np.zeros((3, 3, V), np.float32)
    tokens = np.array([[0, 1, 2], [0, 1, 9], [0, 1, 2]], np.int32)  # token 9 out of range
    par = np.array([[-1, 0, 2], [-1, 0, 0], [-1, 0, 1]], np.int32)  # row 0: forward parent
    res = orc.tree_accept(draft, tokens, par, 1.0, logits=logits)
    assert list(res["accept_len"][:2]) == [-1, -1] and list(res["next_token"][:2]) == [-1, -1]
    assert (res["accepted_nodes"][:2] == -1).all()
    assert res["accept_len"][2] >= 0


def test_lazy_rows_match_given_logits(orc):
    """The on-demand row mode (hidden x W) walks exactly like precomputed fp64 logits."""
    w = wl.scaled(wl.WORKLOADS["vicuna7b_static"], hidden=64, vocab=300, prefix_len=8)
    inp = wl.generate(w, 1.0, seed=77)
    logits = orc.lm_head(inp["hidden"], inp["w_lm"]).reshape(1, w.num_nodes, -1)
    a = orc.tree_accept(inp["draft_probs"], inp["tokens"], inp["parents"], 1.0, logits=logits)
    b = orc.tree_accept(inp["draft_probs"], inp["tokens"], inp["parents"], 1.0,
                        hidden=inp["hidden"], w_lm=inp["w_lm"])
    for key in ("accepted_nodes", "accept_len", "next_token"):
        np.testing.assert_array_equal(a[key], b[key])
