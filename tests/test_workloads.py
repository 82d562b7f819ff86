"""The seeded generator: shapes, tree validity, determinism and bf16 rounding."""
import numpy as np
import pytest

import workloads as wl


def test_node_counts():
    n = {k: w.num_nodes for k, w in wl.WORKLOADS.items()}
    assert n == dict(tiny_chain=6, vicuna7b_static=45, llama70b_dyn=60, batched7b=60, llama3_8b=64)


def test_static_tree_shape():
    par = wl.static_parents((4, 2, 2, 1))
    assert len(par) == 45 and par[0] == -1
    depth = np.zeros(45, int)
    for i in range(1, 45):
        assert 0 <= par[i] < i
        depth[i] = depth[par[i]] + 1
    assert list(np.bincount(depth)) == [1, 4, 8, 16, 16]


@pytest.mark.parametrize("max_depth", [1, 3, 6])
def test_random_tree_depth_bound(max_depth):
    rng = np.random.default_rng(0)
    par = wl.random_parents(rng, 64, max_depth)
    depth = np.zeros(64, int)
    for i in range(1, 64):
        assert 0 <= par[i] < i
        depth[i] = depth[par[i]] + 1
    assert depth.max() <= max_depth


def test_bf16_rounding_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 2 ** -9 + 2 ** -20], np.float32)
    got = wl.bf16_bits_to_f32(wl.round_to_bf16_bits(x))
    # 1+2^-8 is a tie -> even (1.0); 1+3*2^-8 is a tie -> even (1+2^-6)
    np.testing.assert_array_equal(got, np.array([1.0, 1.0, 1.0 + 2 ** -6, -2.5, 1.0], np.float32))


def test_generate_small_is_deterministic_and_consistent():
    w = wl.scaled(wl.WORKLOADS["batched7b"], batch=3, prefix_len=40, prefix_min=5, hidden=32, vocab=50)
    a = wl.generate(w, 1.0)
    b = wl.generate(w, 1.0)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k])
    B, N, V = 3, w.num_nodes, 50
    assert a["q"].shape == (B, N, 32, 128) and a["q"].dtype == np.uint16
    assert a["k_prefix"].shape == (B, 32, 40, 128)
    assert a["draft_probs"].shape == (B, N, V)
    assert ((a["prefix_lens"] >= 5) & (a["prefix_lens"] <= 40)).all()
    for bb in range(B):
        par = a["parents"][bb]
        for c in range(1, N):
            np.testing.assert_allclose(a["draft_probs"][bb, c].sum(), 1.0, rtol=1e-5)
            # siblings share their parent's row
            sib = [s for s in range(1, N) if par[s] == par[c]]
            np.testing.assert_array_equal(a["draft_probs"][bb, sib[0]], a["draft_probs"][bb, c])
    assert ((a["tokens"] >= 0) & (a["tokens"] < V)).all()


def test_greedy_children_are_top_k_of_parent_row():
    w = wl.scaled(wl.WORKLOADS["vicuna7b_static"], hidden=32, vocab=64, prefix_len=4)
    a = wl.generate(w, 0.0)
    par, tok, dp = a["parents"][0], a["tokens"][0], a["draft_probs"][0]
    ch = wl.children_lists(par)
    for u, kids in enumerate(ch):
        if kids:
            order = np.argsort(-dp[kids[0]].astype(np.float64), kind="stable")
            assert list(tok[kids]) == list(order[:len(kids)])
