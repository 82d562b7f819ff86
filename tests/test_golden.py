"""Hand-derived worked examples (tests/golden/*.json) checked against the oracle.

The pages print no numeric worked example; each fixture states the rule it
applies (with its passage) and the hand derivation of the expected values."""
import json
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


@pytest.mark.parametrize("name", ["walk_greedy_small.json", "walk_residual_small.json"])
def test_walk_fixture(orc, name):
    g = load(name)
    V, N = g["vocab"], len(g["parents"])
    logits = np.asarray(g["logits"], np.float32)[None]
    draft = np.asarray(g.get("draft_probs", np.zeros((N, V))), np.float32)[None]
    for seed, off in [(0, 0), (1, 5), (12345, 99)]:
        res = orc.tree_accept(draft, np.asarray([g["tokens"]], np.int32),
                              np.asarray([g["parents"]], np.int32), g["temperature"],
                              seed=seed, offset=off, logits=logits)
        assert list(res["accepted_nodes"][0]) == g["expect_accepted_nodes"]
        assert res["accept_len"][0] == g["expect_accept_len"]
        assert res["next_token"][0] == g["expect_next_token"]


def test_attention_fixture(orc):
    g = load("attention_equal_scores.json")
    N = len(g["parents"])
    f = lambda x: np.asarray(x, np.float32)
    out = orc.tree_attention(
        q=np.zeros((1, N, 1, 2), np.float32),
        k_prefix=f(g["prefix_keys"])[None, None], v_prefix=f(g["prefix_values"])[None, None],
        prefix_lens=[2], k_tree=f(g["tree_keys"])[None, :, None],
        v_tree=f(g["tree_values"])[None, :, None], parents=[g["parents"]])
    np.testing.assert_allclose(out[0, :, 0], g["expect_out"], rtol=1e-15)
