"""Pins for oracle O1 (tree attention) against routines other than itself.

The definition (EAGLE summary, section 3 "Training and verification": the target
scores the whole draft tree in one pass with tree attention) is that node i sees
the prefix and its own root-to-node path.  Three independent checks:
  * a chain tree is ordinary causal decoding of the chain appended to the prefix --
    torch's scaled_dot_product_attention in float64 with a causal mask;
  * every node of a random tree equals causal attention of its query over
    prefix ++ path(i), built explicitly and run through torch SDPA;
  * a one-node tree is plain decode attention over the prefix plus the node.
GQA, varlen prefixes and both input types are covered, so a wrong kv-head mapping,
a dropped self key, a descendant instead of an ancestor or a read past L_b fails.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import workloads as wl


def _inputs(rng, B, N, Hq, Hkv, D, Lmax, lens, parents, dtype):
    def mk(shape):
        x = rng.standard_normal(shape).astype(np.float32)
        return wl.round_to_bf16_bits(x) if dtype == "bf16" else x
    return dict(q=mk((B, N, Hq, D)), k_prefix=mk((B, Hkv, Lmax, D)), v_prefix=mk((B, Hkv, Lmax, D)),
                k_tree=mk((B, N, Hkv, D)), v_tree=mk((B, N, Hkv, D)),
                prefix_lens=np.asarray(lens, dtype=np.int32), parents=np.asarray(parents, np.int32))


def _f64(a, dtype):
    return torch.from_numpy(wl.as_f32(a, dtype).astype(np.float64))


def _sdpa_path(inp, dtype, b, i, h, Hq, Hkv):
    """SDPA of query (b,i,h) over prefix ++ path(i) (root first), all keys visible."""
    G = Hq // Hkv
    g = h // G
    L = int(inp["prefix_lens"][b])
    path = []
    a = i
    while a >= 0:
        path.append(a)
        a = int(inp["parents"][b, a])
    path = path[::-1]
    k = torch.cat([_f64(inp["k_prefix"], dtype)[b, g, :L], _f64(inp["k_tree"], dtype)[b, path, g]])
    v = torch.cat([_f64(inp["v_prefix"], dtype)[b, g, :L], _f64(inp["v_tree"], dtype)[b, path, g]])
    q = _f64(inp["q"], dtype)[b, i, h]
    return F.scaled_dot_product_attention(q[None, None, None], k[None, None], v[None, None])[0, 0, 0]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2)])
def test_chain_equals_causal_decode(orc, dtype, Hq, Hkv):
    rng = np.random.default_rng(7)
    B, n_draft, D, L = 2, 6, 16, 23
    N = n_draft + 1
    par = np.tile(wl.chain_parents(n_draft), (B, 1))
    inp = _inputs(rng, B, N, Hq, Hkv, D, L, [L, L], par, dtype)
    got = orc.tree_attention(**inp)
    G = Hq // Hkv
    for b in range(B):
        k = torch.cat([_f64(inp["k_prefix"], dtype)[b], _f64(inp["k_tree"], dtype)[b].permute(1, 0, 2)], 1)
        v = torch.cat([_f64(inp["v_prefix"], dtype)[b], _f64(inp["v_tree"], dtype)[b].permute(1, 0, 2)], 1)
        k = k.repeat_interleave(G, 0)
        v = v.repeat_interleave(G, 0)
        q = _f64(inp["q"], dtype)[b].permute(1, 0, 2)  # [Hq, N, D]
        # query n sits at sequence position L + n and sees every position <= L + n
        mask = torch.arange(L + N)[None, :] <= (L + torch.arange(N))[:, None]
        ref = F.scaled_dot_product_attention(q[None], k[None], v[None], attn_mask=mask)[0]
        np.testing.assert_allclose(got[b], ref.permute(1, 0, 2).numpy(), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_random_tree_equals_path_attention(orc, dtype):
    rng = np.random.default_rng(11)
    B, N, Hq, Hkv, D, Lmax = 3, 17, 6, 3, 8, 40
    lens = [40, 0, 13]
    par = np.stack([wl.random_parents(rng, N, 5) for _ in range(B)])
    inp = _inputs(rng, B, N, Hq, Hkv, D, Lmax, lens, par, dtype)
    got = orc.tree_attention(**inp)
    for b in range(B):
        for i in range(N):
            for h in range(Hq):
                ref = _sdpa_path(inp, dtype, b, i, h, Hq, Hkv).numpy()
                np.testing.assert_allclose(got[b, i, h], ref, rtol=1e-11, atol=1e-12)


def test_row_subset_matches_full(orc):
    rng = np.random.default_rng(5)
    B, N, Hq, Hkv, D, Lmax = 2, 9, 4, 2, 16, 31
    par = np.stack([wl.random_parents(rng, N, 3) for _ in range(B)])
    inp = _inputs(rng, B, N, Hq, Hkv, D, Lmax, [31, 7], par, "bf16")
    full = orc.tree_attention(**inp)
    rows = np.array([[1, 8, 3], [0, 0, 0], [1, 4, 1]])
    sub = orc.tree_attention(**inp, rows=rows)
    for r, (b, i, h) in enumerate(rows):
        np.testing.assert_array_equal(sub[r], full[b, i, h])


def test_single_node_tree_is_decode(orc):
    rng = np.random.default_rng(3)
    B, Hq, Hkv, D, L = 1, 2, 1, 32, 50
    inp = _inputs(rng, B, 1, Hq, Hkv, D, L, [L], [[-1]], "f32")
    got = orc.tree_attention(**inp)
    for h in range(Hq):
        k = np.concatenate([inp["k_prefix"][0, 0], inp["k_tree"][0, :, 0]]).astype(np.float64)
        v = np.concatenate([inp["v_prefix"][0, 0], inp["v_tree"][0, :, 0]]).astype(np.float64)
        s = k @ inp["q"][0, 0, h].astype(np.float64) / np.sqrt(D)
        w = np.exp(s - s.max())
        np.testing.assert_allclose(got[0, 0, h], (w / w.sum()) @ v, rtol=1e-12, atol=1e-13)


def test_custom_scale(orc):
    rng = np.random.default_rng(9)
    inp = _inputs(rng, 1, 3, 2, 2, 8, 5, [5], [[-1, 0, 1]], "f32")
    a = orc.tree_attention(**inp, scale=0.25)
    b_ = orc.tree_attention(**inp)  # default 1/sqrt(8)
    assert not np.allclose(a, b_)
    q = inp["q"][0, 2, 1].astype(np.float64)
    k = np.concatenate([inp["k_prefix"][0, 1], inp["k_tree"][0, :, 1]]).astype(np.float64)
    v = np.concatenate([inp["v_prefix"][0, 1], inp["v_tree"][0, :, 1]]).astype(np.float64)
    s = 0.25 * (k @ q)
    w = np.exp(s - s.max())
    np.testing.assert_allclose(a[0, 2, 1], (w / w.sum()) @ v, rtol=1e-12)


def test_invalid_tree_rejected(orc):
    rng = np.random.default_rng(1)
    inp = _inputs(rng, 1, 3, 1, 1, 4, 2, [2], [[-1, 2, 0]], "f32")  # forward parent
    with pytest.raises(ValueError):
        orc.tree_attention(**inp)
