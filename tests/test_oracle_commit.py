"""Pins for oracle O4 (post-accept commit) against routines other than itself.

The commit (EAGLE summary, section 3 "Drafting and verification": the accepted tokens
extend the target's context and their features feed the next drafting round) appends
the root and the accepted nodes, root first, to the prefix K/V cache and gathers their
hidden rows.  Independent checks:
  * after the commit, each committed node's tree attention (oracle O1, itself pinned to
    torch SDPA) equals plain causal attention of that node's query over the first
    L_b + t + 1 positions of the updated cache, run through torch's SDPA in float64 --
    a wrong position, order, kv head, row or a K/V swap fails it;
  * logits of the gathered feature rows (numpy float64 matmul) equal oracle O2's logits
    of the committed nodes' hidden rows;
  * the walk's own output (oracle O3) commits cleanly: its accepted nodes form a chain;
  * the degenerate cases: an invalid tree (accept_len = -1), only the root (0 accepted),
    overflow of Lmax, a path that is not a chain, a bad prefix length; nothing outside
    the committed rows and positions changes.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import workloads as wl


def _problem(rng, B, N, Hq, Hkv, D, Lmax, lens, dtype, H=24, max_depth=4):
    def mk(shape):
        x = rng.standard_normal(shape).astype(np.float32)
        return wl.round_to_bf16_bits(x) if dtype == "bf16" else x
    parents = np.stack([wl.random_parents(rng, N, max_depth) for _ in range(B)]).astype(np.int32)
    return dict(q=mk((B, N, Hq, D)), k_prefix=mk((B, Hkv, Lmax, D)), v_prefix=mk((B, Hkv, Lmax, D)),
                k_tree=mk((B, N, Hkv, D)), v_tree=mk((B, N, Hkv, D)), hidden=mk((B, N, H)),
                prefix_lens=np.asarray(lens, np.int32), parents=parents)


def _random_path(rng, parents):
    """A random root-to-node chain: the accepted nodes of some walk (root excluded)."""
    N = len(parents)
    end = int(rng.integers(0, N))
    path = []
    a = end
    while a > 0:
        path.append(a)
        a = int(parents[a])
    return path[::-1]


def _accepts(rng, parents):
    B, N = parents.shape
    acc = np.full((B, N), -1, np.int32)
    alen = np.zeros(B, np.int32)
    for b in range(B):
        p = _random_path(rng, parents[b])
        acc[b, :len(p)] = p
        alen[b] = len(p)
    return acc, alen


def _f64(a, dtype):
    return torch.from_numpy(wl.as_f32(a, dtype).astype(np.float64))


def _check_attention_invariant(orc, inp, kp, vp, acc, alen, dtype, Hq, Hkv):
    G = Hq // Hkv
    rows = []
    for b in range(len(alen)):
        path = [0] + [int(c) for c in acc[b, :alen[b]]]
        for t, node in enumerate(path):
            for h in range(Hq):
                rows.append((b, t, node, h))
    sel = np.array([(b, node, h) for b, _, node, h in rows], np.int32)
    tree = orc.tree_attention(inp["q"], inp["k_prefix"], inp["v_prefix"], inp["prefix_lens"],
                              inp["k_tree"], inp["v_tree"], inp["parents"], rows=sel)
    K, Vv, Q = _f64(kp, dtype), _f64(vp, dtype), _f64(inp["q"], dtype)
    for r, (b, t, node, h) in enumerate(rows):
        n_keys = int(inp["prefix_lens"][b]) + t + 1
        k = K[b, h // G, :n_keys]
        v = Vv[b, h // G, :n_keys]
        ref = F.scaled_dot_product_attention(Q[b, node, h][None, None, None], k[None, None],
                                             v[None, None])[0, 0, 0].numpy()
        np.testing.assert_allclose(tree[r], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2)])
def test_committed_cache_reproduces_tree_attention(orc, dtype, Hq, Hkv):
    rng = np.random.default_rng(11 + Hq)
    B, N, D, Lmax = 3, 12, 16, 40
    lens = [7, 21, 28]
    inp = _problem(rng, B, N, Hq, Hkv, D, Lmax, lens, dtype)
    acc, alen = _accepts(rng, inp["parents"])
    kp, vp, new, feat = orc.commit(inp["k_prefix"], inp["v_prefix"], inp["prefix_lens"],
                                   inp["k_tree"], inp["v_tree"], inp["hidden"], inp["parents"],
                                   acc, alen)
    np.testing.assert_array_equal(new, np.asarray(lens) + alen + 1)
    _check_attention_invariant(orc, inp, kp, vp, acc, alen, dtype, Hq, Hkv)


def test_gathered_features_give_the_committed_logits(orc):
    rng = np.random.default_rng(5)
    B, N, H, V = 2, 10, 24, 37
    inp = _problem(rng, B, N, 2, 2, 8, 30, [4, 9], "f32", H=H)
    acc, alen = _accepts(rng, inp["parents"])
    w = (rng.standard_normal((V, H)) / np.sqrt(H)).astype(np.float32)
    _, _, new, feat = orc.commit(inp["k_prefix"], inp["v_prefix"], inp["prefix_lens"], inp["k_tree"],
                                 inp["v_tree"], inp["hidden"], inp["parents"], acc, alen)
    for b in range(B):
        path = [0] + [int(c) for c in acc[b, :alen[b]]]
        rows = np.array([b * N + node for node in path], np.int32)
        ref = orc.lm_head(inp["hidden"].reshape(B * N, H), w, rows=rows)
        got = feat[b, :len(path)].astype(np.float64) @ w.astype(np.float64).T
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("T", [0.0, 1.0])
def test_walk_output_commits(orc, T):
    """The oracle walk's accepted nodes form a root path, so the commit takes them."""
    w = wl.scaled(wl.WORKLOADS["batched7b"], batch=3, prefix_len=200, prefix_min=20, vocab=600,
                  hidden=128, num_q_heads=4, num_kv_heads=2, head_dim=64)
    inp = wl.generate(w, T)
    res = orc.tree_accept(inp["draft_probs"], inp["tokens"], inp["parents"], T, seed=3, offset=1,
                          hidden=inp["hidden"], w_lm=inp["w_lm"])
    hid = inp["hidden"].reshape(w.batch, w.num_nodes, w.hidden)
    kp, vp, new, feat = orc.commit(inp["k_prefix"], inp["v_prefix"], inp["prefix_lens"],
                                   inp["k_tree"], inp["v_tree"], hid, inp["parents"],
                                   res["accepted_nodes"], res["accept_len"])
    np.testing.assert_array_equal(new, inp["prefix_lens"] + res["accept_len"] + 1)
    _check_attention_invariant(orc, inp, kp, vp, res["accepted_nodes"], res["accept_len"], w.dtype,
                               w.num_q_heads, w.num_kv_heads)


def test_degenerate_cases(orc):
    rng = np.random.default_rng(9)
    B, N, Hkv, D, Lmax, H = 6, 8, 2, 8, 16, 8
    inp = _problem(rng, B, N, 2, Hkv, D, Lmax, [5, 5, 13, 5, 5, 17], "f32", H=H)
    par = inp["parents"].copy()
    par[:] = np.array([-1, 0, 1, 2, 0, 4, 5, 1], np.int32)  # two chains under the root
    acc = np.full((B, N), -1, np.int32)
    alen = np.array([-1, 0, 3, 2, 2, 0], np.int32)
    acc[2, :3] = [1, 2, 3]   # L = 13: 13 + 4 > 16 overflows
    acc[3, :2] = [1, 2]      # a chain
    acc[4, :2] = [1, 5]      # 5's parent is 4, not 1: not a chain
    # sequence 5: prefix length 17 > Lmax
    feat0 = np.full((B, N, H), 7.0, np.float32)
    kp, vp, new, feat = orc.commit(inp["k_prefix"], inp["v_prefix"], inp["prefix_lens"],
                                   inp["k_tree"], inp["v_tree"], inp["hidden"], par, acc, alen,
                                   feat=feat0)
    np.testing.assert_array_equal(new, [5, 6, -1, 8, -1, -1])
    for b in (0, 2, 4, 5):  # nothing written
        np.testing.assert_array_equal(kp[b], inp["k_prefix"][b])
        np.testing.assert_array_equal(vp[b], inp["v_prefix"][b])
        np.testing.assert_array_equal(feat[b], feat0[b])
    # sequence 1: only the root, at position 5
    np.testing.assert_array_equal(kp[1, :, 5], inp["k_tree"][1, 0])
    np.testing.assert_array_equal(feat[1, 0], inp["hidden"][1, 0])
    # sequence 3: root, 1, 2 at positions 5, 6, 7; everything else untouched
    np.testing.assert_array_equal(vp[3, :, 5:8], inp["v_tree"][3, [0, 1, 2]].transpose(1, 0, 2))
    keep = np.ones(Lmax, bool)
    keep[5:8] = False
    np.testing.assert_array_equal(kp[3, :, keep], inp["k_prefix"][3, :, keep])
    np.testing.assert_array_equal(feat[3, 3:], feat0[3, 3:])
