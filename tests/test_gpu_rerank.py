"""eagle_tree_rerank on the GPU against oracle O5, bit for bit: random expanded candidate
trees of several sizes, deep chains (one tree level per round of the kernel), confidences
that are NaN, negative or above 1, ties, trees that are not topological, and more kept
nodes than candidates."""
import numpy as np
import pytest
import torch

import workloads as wl

pytestmark = pytest.mark.gpu


def _run(cuda_lib, orc, par, tok, conf, m):
    B, M = par.shape
    d = {n: torch.from_numpy(np.ascontiguousarray(a)).cuda() for n, a in
         (("par", par.astype(np.int32)), ("tok", tok.astype(np.int32)), ("conf", conf.astype(np.float32)))}
    sel = torch.full((B, m), 7, dtype=torch.int32, device="cuda")
    po, to = torch.full_like(sel, 7), torch.full_like(sel, 7)
    masks = torch.full((B, m), 7, dtype=torch.int64, device="cuda")
    nsel = torch.full((B,), 7, dtype=torch.int32, device="cuda")
    cuda_lib.tree_rerank(d["par"], d["tok"], d["conf"], m, sel, po, to, masks, nsel)
    torch.cuda.synchronize()
    ref = orc.tree_rerank(par, tok, conf, m)
    np.testing.assert_array_equal(nsel.cpu().numpy(), ref["num_selected"])
    np.testing.assert_array_equal(sel.cpu().numpy(), ref["sel"])
    np.testing.assert_array_equal(po.cpu().numpy(), ref["parents"])
    np.testing.assert_array_equal(to.cpu().numpy(), ref["tokens"])
    np.testing.assert_array_equal(masks.cpu().numpy().view(np.uint64), ref["masks"])
    return ref


@pytest.mark.parametrize("B,M,m,depth", [(4, 60, 45, 6), (16, 200, 64, 8), (3, 1024, 64, 12),
                                         (5, 33, 1, 4), (2, 10, 64, 3)])
def test_rerank_random_trees(cuda_lib, orc, B, M, m, depth):
    rng = np.random.default_rng(M * 131 + m)
    par = np.stack([wl.random_parents(rng, M, depth) for _ in range(B)])
    tok = rng.integers(0, 32000, (B, M))
    conf = rng.uniform(0.0, 1.0, (B, M)).astype(np.float32)
    conf[:, ::7] = np.round(conf[:, ::7], 1)  # repeated values: ties broken by index
    ref = _run(cuda_lib, orc, par, tok, conf, m)
    assert (ref["num_selected"] == min(m, M)).all()


def test_rerank_deep_chain_and_degenerate_confidences(cuda_lib, orc):
    rng = np.random.default_rng(9)
    M = 1024
    chain = wl.chain_parents(M - 1)
    star = np.array([-1] + [0] * (M - 1), np.int32)
    bad = chain.copy()
    bad[500] = 700  # not topological
    par = np.stack([chain, star, bad, star])
    tok = rng.integers(0, 1000, (4, M))
    conf = rng.uniform(0.9, 1.0, (4, M)).astype(np.float32)
    conf[1, 3::5] = np.nan
    conf[1, 4::5] = -1.0
    conf[3, :] = 1.5  # every value 1: the first indices
    _run(cuda_lib, orc, par, tok, conf, 64)
