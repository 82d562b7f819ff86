"""Seeded synthetic inputs for draft-tree verification (EAGLE / EAGLE-2).

This module only *makes inputs*: shapes, value distributions, tree shapes,
drafted tokens and draft distributions.  It is shared by the CPU oracle's
tests and by the CUDA path's tests and benchmark, and it holds none of the
verification arithmetic (no tree attention, no accept/resample walk).

The one place it multiplies hidden states by the LM-head weight is to build
the *draft* distributions of the workload recipe ("softmax(target logits +
noise)"): it stands in for the EAGLE draft model, which the pages describe as
reusing the target LLM's frozen LM head (EAGLE paper, section 3 "Draft
model").  Its float32 numpy product is data synthesis only: neither the oracle
nor the kernels read it back as their own logits.

Workload recipes (the five verify-step shapes; the pages print no model
dimensions, so these are the stated synthetic stand-ins for the Vicuna-7B,
LLaMA2-70B and LLaMA3-8B families the pages evaluate on):

  tiny_chain      B1  Hq=Hkv=4   D64  fp32 L64            chain of 5 drafted (N=6)   H256  V512     T=1
  vicuna7b_static B1  32/32      D128 bf16 L1024          static tree (4,2,2,1) N=45 H4096 V32000   T=0,1
  llama70b_dyn    B1  64/8       D128 bf16 L4096          60-node random, parents at depth<=5   H8192 V32000 T=1
  batched7b       B16 32/32      D128 bf16 L_b~U[512,4096] 60-node random per sequence, depth<=6 H4096 V32000 T=1
  llama3_8b       B8  32/8       D128 bf16 L8192          64-node random, depth<=7 H4096 V128256  T=0,1

Value distributions: Q, K, V, hidden ~ N(0, 1); W ~ N(0, 1/H) (the second
argument of N(., .) is a variance); bf16 tensors are rounded from float32 to
nearest-even.  Draft rows: one per parent node u, shared by u's children;
tiny_chain uses softmax(N(0, 2) logits), the bf16 workloads use
softmax(target_logits[u] / T' + noise) with T' = max(T, 1) and noise variance
1 (1.5 for llama3_8b).  Drafted tokens: at T > 0 each child's token is drawn
i.i.d. from its parent's draft row; at T == 0 the children of u take the
top-k tokens of u's row in index order (EAGLE paper, appendix A.1 "Tree
Structure": greedy children are the top-k tokens, non-greedy children are k
samples).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

F32 = "f32"
BF16 = "bf16"


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    dtype: str
    prefix_len: int            # fixed prefix length, or the upper bound when varlen
    prefix_min: Optional[int]  # lower bound of U[prefix_min, prefix_len] per sequence; None = fixed
    tree: str                  # "chain", "static", "random"
    tree_arg: tuple            # chain: (drafted,), static: branching, random: (nodes, max_depth)
    hidden: int
    vocab: int
    temperatures: tuple
    draft_noise_var: float     # variance of the noise added to target logits (bf16 workloads)
    seed_id: int

    @property
    def num_nodes(self) -> int:
        if self.tree == "chain":
            return self.tree_arg[0] + 1
        if self.tree == "static":
            total, width = 1, 1
            for k in self.tree_arg:
                width *= k
                total += width
            return total
        return self.tree_arg[0]


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny_chain", 1, 4, 4, 64, F32, 64, None, "chain", (5,), 256, 512,
                 (1.0,), 0.0, 1),
        Workload("vicuna7b_static", 1, 32, 32, 128, BF16, 1024, None, "static", (4, 2, 2, 1),
                 4096, 32000, (0.0, 1.0), 1.0, 2),
        Workload("llama70b_dyn", 1, 64, 8, 128, BF16, 4096, None, "random", (60, 6),
                 8192, 32000, (1.0,), 1.0, 3),
        Workload("batched7b", 16, 32, 32, 128, BF16, 4096, 512, "random", (60, 6),
                 4096, 32000, (1.0,), 1.0, 4),
        Workload("llama3_8b", 8, 32, 8, 128, BF16, 8192, None, "random", (64, 7),
                 4096, 128256, (0.0, 1.0), 1.5, 5),
    ]
}


def scaled(base: Workload, **kw) -> Workload:
    """A smaller copy of a workload (same recipe, other sizes) for fast parity cases."""
    return dataclasses.replace(base, **kw)


# --------------------------------------------------------------------------- dtype helpers

def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest, ties to even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    flat = x.reshape(-1).view(np.uint32)
    out = np.empty(flat.shape, dtype=np.uint16)
    step = 1 << 24
    for s in range(0, flat.size, step):
        u = flat[s:s + step]
        # finite inputs stay below 2**32 after the bias, so uint32 arithmetic is exact
        out[s:s + step] = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
                           >> np.uint32(16)).astype(np.uint16)
    return out.reshape(x.shape)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> the exactly equal float32 values."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _normal(rng: np.random.Generator, shape, var: float = 1.0) -> np.ndarray:
    out = rng.standard_normal(size=shape, dtype=np.float32)
    if var != 1.0:
        out *= np.float32(np.sqrt(var))
    return out


def _softmax_rows(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.float64)
    z = z - z.max(axis=-1, keepdims=True)
    e = np.exp(z)
    return (e / e.sum(axis=-1, keepdims=True)).astype(np.float32)


# --------------------------------------------------------------------------- trees

def chain_parents(n_drafted: int) -> np.ndarray:
    return np.arange(-1, n_drafted, dtype=np.int32)


def static_parents(branching) -> np.ndarray:
    """Breadth-first full tree: every node of depth d has branching[d] children."""
    parents = [-1]
    level = [0]
    for k in branching:
        nxt = []
        for u in level:
            for _ in range(k):
                parents.append(u)
                nxt.append(len(parents) - 1)
        level = nxt
    return np.asarray(parents, dtype=np.int32)


def random_parents(rng: np.random.Generator, n_nodes: int, max_depth: int) -> np.ndarray:
    """Node i's parent is uniform over the earlier nodes whose depth is < max_depth."""
    parents = np.full(n_nodes, -1, dtype=np.int32)
    depth = np.zeros(n_nodes, dtype=np.int64)
    for i in range(1, n_nodes):
        cand = np.nonzero(depth[:i] < max_depth)[0]
        p = int(cand[rng.integers(0, len(cand))])
        parents[i] = p
        depth[i] = depth[p] + 1
    return parents


def children_lists(parents: np.ndarray):
    ch = [[] for _ in range(len(parents))]
    for i in range(1, len(parents)):
        ch[int(parents[i])].append(i)
    return ch


# --------------------------------------------------------------------------- generation

def _draw_tokens(rng, parents, draft_rows, temperature):
    """Fill tokens[c] for every drafted node c from its parent's draft row."""
    n = len(parents)
    tokens = np.zeros(n, dtype=np.int32)
    ch = children_lists(parents)
    for u in range(n):
        kids = ch[u]
        if not kids:
            continue
        row = draft_rows[u].astype(np.float64)
        if temperature == 0.0:
            order = np.argsort(-row, kind="stable")
            for rank, c in enumerate(kids):
                tokens[c] = order[rank]
        else:
            cdf = np.cumsum(row)
            cdf /= cdf[-1]
            draws = np.searchsorted(cdf, rng.random(len(kids)), side="right")
            tokens[kids] = np.minimum(draws, len(row) - 1)
    return tokens


def generate(w: Workload, temperature: float, seed: Optional[int] = None) -> dict:
    """All inputs of one verify step for workload ``w`` at ``temperature``.

    Returns numpy arrays.  bf16 tensors come as uint16 bit patterns under the
    key name and as exact float32 copies under ``<name>_f32`` only where the
    caller asks through :func:`as_f32`.  Layouts follow the library:
      q [B,N,Hq,D], k_prefix/v_prefix [B,Hkv,Lmax,D], prefix_lens [B],
      k_tree/v_tree [B,N,Hkv,D], parents [B,N], hidden [B*N,H], w_lm [V,H],
      draft_probs [B,N,V] (row c = distribution node c was drafted from;
      row 0 unused), tokens [B,N] (tokens[.,0] = committed root token).
    """
    rng = np.random.default_rng(1000 + w.seed_id if seed is None else seed)
    B, N, Hq, Hkv, D = w.batch, w.num_nodes, w.num_q_heads, w.num_kv_heads, w.head_dim
    H, V, Lmax = w.hidden, w.vocab, w.prefix_len

    if w.prefix_min is None:
        prefix_lens = np.full(B, Lmax, dtype=np.int32)
    else:
        prefix_lens = rng.integers(w.prefix_min, Lmax + 1, size=B).astype(np.int32)

    if w.tree == "chain":
        par1 = [chain_parents(w.tree_arg[0]) for _ in range(B)]
    elif w.tree == "static":
        par1 = [static_parents(w.tree_arg) for _ in range(B)]
    else:
        par1 = [random_parents(rng, w.tree_arg[0], w.tree_arg[1]) for _ in range(B)]
    parents = np.stack(par1).astype(np.int32)

    q = _normal(rng, (B, N, Hq, D))
    k_prefix = _normal(rng, (B, Hkv, Lmax, D))
    v_prefix = _normal(rng, (B, Hkv, Lmax, D))
    # Padding past each sequence's prefix holds large garbage so a read past L_b shows.
    for b in range(B):
        L = int(prefix_lens[b])
        if L < Lmax:
            k_prefix[b, :, L:, :] *= 100.0
            v_prefix[b, :, L:, :] *= 100.0
    k_tree = _normal(rng, (B, N, Hkv, D))
    v_tree = _normal(rng, (B, N, Hkv, D))
    hidden = _normal(rng, (B * N, H))
    w_lm = _normal(rng, (V, H), var=1.0 / H)

    out = dict(prefix_lens=prefix_lens, parents=parents)
    if w.dtype == BF16:
        for name, arr in dict(q=q, k_prefix=k_prefix, v_prefix=v_prefix, k_tree=k_tree,
                              v_tree=v_tree, hidden=hidden, w_lm=w_lm).items():
            out[name] = round_to_bf16_bits(arr)
    else:
        out.update(q=q, k_prefix=k_prefix, v_prefix=v_prefix, k_tree=k_tree, v_tree=v_tree,
                   hidden=hidden, w_lm=w_lm)
    del q, k_prefix, v_prefix, k_tree, v_tree

    # Draft rows (one per parent) and drafted tokens.
    draft = np.zeros((B, N, V), dtype=np.float32)
    tokens = np.zeros((B, N), dtype=np.int32)
    tokens[:, 0] = rng.integers(0, V, size=B)
    t_eff = max(temperature, 1.0)
    hid_f32 = as_f32(out["hidden"], w.dtype)
    w_f32 = as_f32(out["w_lm"], w.dtype) if w.dtype == BF16 else out["w_lm"]
    for b in range(B):
        par = parents[b]
        ch = children_lists(par)
        us = [u for u in range(N) if ch[u]]
        if w.dtype == F32:
            rows = _softmax_rows(_normal(rng, (len(us), V), var=2.0))
        else:
            tl = hid_f32[b * N + np.asarray(us)] @ w_f32.T
            rows = _softmax_rows(tl / np.float32(t_eff) + _normal(rng, tl.shape, w.draft_noise_var))
        row_of = {u: rows[j] for j, u in enumerate(us)}
        tok_rows = np.zeros((N, V), dtype=np.float32)
        for u in us:
            tok_rows[u] = row_of[u]
        tokens_b = _draw_tokens(rng, par, tok_rows, temperature)
        tokens[b, 1:] = tokens_b[1:]
        for c in range(1, N):
            draft[b, c] = row_of[int(par[c])]
    out.update(draft_probs=draft, tokens=tokens, temperature=np.float32(temperature))
    return out


def as_f32(arr: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float32 values of an input tensor (bf16 bit patterns widened)."""
    if dtype == BF16:
        return bf16_bits_to_f32(arr)
    return np.asarray(arr, dtype=np.float32)


def shape_of(w: Workload) -> dict:
    return dict(batch=w.batch, num_nodes=w.num_nodes, num_q_heads=w.num_q_heads,
                num_kv_heads=w.num_kv_heads, head_dim=w.head_dim, max_prefix_len=w.prefix_len,
                hidden=w.hidden, vocab=w.vocab, dtype=w.dtype)


def random_logits(rng: np.random.Generator, B: int, N: int, V: int, scale: float = 1.0):
    """Stand-alone fp32 logits for accept-only cases (no LM head involved)."""
    return (_normal(rng, (B, N, V)) * np.float32(scale)).astype(np.float32)
