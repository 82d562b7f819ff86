"""eagle_draft_select on the GPU against oracle O6: greedy children bit for bit (ties to
the lower index included), sampled children wherever the oracle's race is not a near tie
(margin 1e-4, as for the walk), confidences and row distributions within 1e-5 relative;
vocabularies with a ragged tail and the 128256-token vocabulary, k from 1 to 16, rows on
one CTA and rows split over a cluster."""
import numpy as np
import pytest
import torch

from tests.parity import MARGIN

pytestmark = pytest.mark.gpu


def _run(cuda_lib, logits, T, k, seed, offset, with_probs=True):
    B, F, V = logits.shape
    lg = torch.from_numpy(logits).cuda()
    tok = torch.full((B, F, k), 7, dtype=torch.int32, device="cuda")
    conf = torch.full((B, F, k), 7.0, dtype=torch.float32, device="cuda")
    probs = torch.full((B, F, V), 7.0, dtype=torch.float32, device="cuda") if with_probs else None
    cuda_lib.draft_select(lg, T, k, seed, offset, tok, conf, probs)
    torch.cuda.synchronize()
    assert cuda_lib.device_error(reset=True) == 0
    return tok.cpu().numpy(), conf.cpu().numpy(), None if probs is None else probs.cpu().numpy()


# rows of one CTA (small vocabularies, many rows) and rows split over clusters of 2 to 8 CTAs
# (large vocabularies, few rows), with ragged last slices (8195 = 7 * 1028 + 999)
CASES = [(2, 3, 1000, 4), (1, 8, 32000, 10), (3, 2, 1001, 16), (1, 2, 128256, 8), (4, 5, 777, 1),
         (1, 3, 8195, 5), (4, 8, 32000, 4), (2, 100, 4096, 3)]


@pytest.mark.parametrize("T", [0.0, 0.7, 1.0])
@pytest.mark.parametrize("B,F,V,k", CASES, ids=[f"B{c[0]}F{c[1]}V{c[2]}k{c[3]}" for c in CASES])
def test_draft_select_matches_oracle(cuda_lib, orc, B, F, V, k, T):
    rng = np.random.default_rng(V * 7 + k)
    logits = (rng.standard_normal((B, F, V)) * 2.0).astype(np.float32)
    logits[0, 0, 5:5 + k] = logits[0, 0].max() + 1.0  # a run of ties at the top
    tok, conf, probs = _run(cuda_lib, logits, T, k, seed=3, offset=11)
    ref = orc.draft_select(logits, T, k, seed=3, offset=11, margin=MARGIN, with_probs=True)
    p = ref["probs"]
    err = np.abs(probs - p).max(axis=-1) / p.max(axis=-1)
    assert err.max() <= 1e-5, err.max()
    exact = 0
    for b in range(B):
        for f in range(F):
            for j in range(k):
                t = int(tok[b, f, j])
                assert 0 <= t < V
                np.testing.assert_allclose(conf[b, f, j], p[b, f, t], rtol=1e-5)
                if ref["near"][b, f, j] == 0:
                    assert t == ref["tokens"][b, f, j], (b, f, j, t, ref["tokens"][b, f, j])
                    exact += 1
    # the deliberate run of ties at the top of row (0, 0) is a near decision by construction
    assert exact >= B * F * k - k - max(1, B * F * k // 20)
    if T == 0.0:
        np.testing.assert_array_equal(tok[0, 0], np.arange(5, 5 + k))


def test_draft_select_without_probs_and_all_nan_row(cuda_lib, orc):
    logits = np.random.default_rng(1).standard_normal((1, 2, 300)).astype(np.float32)
    logits[0, 1] = np.nan
    tok, conf, _ = _run(cuda_lib, logits, 0.0, 4, 0, 0, with_probs=False)
    ref = orc.draft_select(logits[:, :1], 0.0, 4)
    np.testing.assert_array_equal(tok[0, 0], ref["tokens"][0, 0])
    assert (tok[0, 1] == -1).all() and (conf[0, 1] == 0).all()


@pytest.mark.parametrize("T", [0.0, 0.7, 1.0])
@pytest.mark.parametrize("B,F,V,k", CASES, ids=[f"B{c[0]}F{c[1]}V{c[2]}k{c[3]}" for c in CASES])
def test_draft_distinct_matches_oracle(cuda_lib, orc, B, F, V, k, T):
    """Siblings drawn without replacement (oracle O7): distinct, bit-exact wherever the
    oracle's clocks are not a near tie, confidences and distributions within 1e-5."""
    rng = np.random.default_rng(V * 11 + k)
    logits = (rng.standard_normal((B, F, V)) * 2.0).astype(np.float32)
    lg = torch.from_numpy(logits).cuda()
    tok = torch.full((B, F, k), 7, dtype=torch.int32, device="cuda")
    conf = torch.full((B, F, k), 7.0, dtype=torch.float32, device="cuda")
    probs = torch.full((B, F, V), 7.0, dtype=torch.float32, device="cuda")
    cuda_lib.draft_select_distinct(lg, T, k, 5, 13, tok, conf, probs)
    torch.cuda.synchronize()
    assert cuda_lib.device_error(reset=True) == 0
    tok, conf, probs = tok.cpu().numpy(), conf.cpu().numpy(), probs.cpu().numpy()
    ref = orc.draft_select_distinct(logits, T, k, seed=5, offset=13, margin=MARGIN, with_probs=True)
    p = ref["probs"]
    assert (np.abs(probs - p).max(axis=-1) / p.max(axis=-1)).max() <= 1e-5
    exact = 0
    for b in range(B):
        for f in range(F):
            assert len(set(tok[b, f].tolist())) == k  # distinct siblings
            for j in range(k):
                t = int(tok[b, f, j])
                assert 0 <= t < V
                np.testing.assert_allclose(conf[b, f, j], p[b, f, t], rtol=1e-5)
                if ref["near"][b, f, j] == 0:
                    assert t == ref["tokens"][b, f, j], (b, f, j, t, ref["tokens"][b, f, j])
                    exact += 1
    # a near tie between two clocks flags both of their positions
    assert exact >= B * F * k - max(2, B * F * k // 10)


@pytest.mark.parametrize("B,F,V,k", [(2, 3, 1000, 4), (1, 10, 32000, 10), (1, 2, 128256, 16), (3, 1, 5, 5)])
def test_child_rows_match_oracle(cuda_lib, orc, B, F, V, k):
    """The row each sibling was drawn from (oracle O7) within 1e-5 of each row's maximum,
    exact zeros at the earlier siblings' tokens, and rows after a -1 token all zero."""
    rng = np.random.default_rng(V + k)
    probs = rng.dirichlet(np.full(V, 0.3), (B, F)).astype(np.float32)
    tokens = np.stack([np.stack([rng.permutation(V)[:k] for _ in range(F)]) for _ in range(B)]).astype(np.int32)
    if k > 2:
        tokens[0, 0, 2] = -1
    # siblings that carry most of the mass: the remaining mass is small and must not cancel
    probs[-1, -1] = 1e-6
    probs[-1, -1, tokens[-1, -1, :k - 1]] = 1.0
    probs[-1, -1] /= probs[-1, -1].sum()
    out = torch.full((B, F, k, V), 7.0, dtype=torch.float32, device="cuda")
    cuda_lib.draft_child_rows(torch.from_numpy(probs).cuda(), torch.from_numpy(tokens).cuda(), out)
    torch.cuda.synchronize()
    assert cuda_lib.device_error(reset=True) == 0
    got = out.cpu().numpy()
    ref = orc.draft_child_rows(probs.astype(np.float64), tokens)
    for b in range(B):
        for f in range(F):
            for j in range(k):
                gone = tokens[b, f, :j]
                if (gone < 0).any():
                    assert (got[b, f, j] == 0).all()
                else:
                    assert (got[b, f, j, gone] == 0).all()
    scale = np.maximum(ref.max(axis=-1, keepdims=True), 1e-30)
    assert (np.abs(got - ref) / scale).max() <= 1e-5


@pytest.mark.parametrize("conditioned", [True, False], ids=["child-rows", "shared-row"])
def test_without_replacement_chain_on_gpu(cuda_lib, conditioned):
    """The whole chain on the GPU: siblings drawn without replacement
    (eagle_draft_select_distinct), their rows (eagle_draft_child_rows), the walk
    (eagle_tree_accept).  Over 200,000 seeded trees the first emitted token follows the
    target p with the children's own rows, and does not with the parent's row shared."""
    from scipy import special, stats
    V, k, CH = 8, 3, 50000
    q_logits = np.array([2.0, 1.5, 1.0, 0.0, -0.5, -1.0, 0.5, 0.2], np.float32)
    p_logits = np.array([0.0, 0.3, 1.2, 0.8, 1.0, -0.4, 0.1, 0.6], np.float32)
    p = special.softmax(p_logits.astype(np.float64))
    N = k + 1
    shape = cuda_lib.make_shape(CH, N, 1, 1, 64, 1, 8, V, "f32")
    parents = torch.from_numpy(np.tile(np.array([-1] + [0] * k, np.int32), (CH, 1))).cuda()
    logits = torch.from_numpy(np.tile(p_logits, (CH, N, 1))).cuda()
    d_lg = torch.from_numpy(np.tile(q_logits, (CH, 1, 1))).cuda()
    tok = torch.empty((CH, 1, k), dtype=torch.int32, device="cuda")
    conf = torch.empty((CH, 1, k), dtype=torch.float32, device="cuda")
    probs = torch.empty((CH, 1, V), dtype=torch.float32, device="cuda")
    rows = torch.empty((CH, 1, k, V), dtype=torch.float32, device="cuda")
    acc = torch.empty((CH, N), dtype=torch.int32, device="cuda")
    alen = torch.empty((CH,), dtype=torch.int32, device="cuda")
    nxt = torch.empty((CH,), dtype=torch.int32, device="cuda")
    counts = np.zeros(V, np.int64)
    for off in range(4):
        cuda_lib.draft_select_distinct(d_lg, 1.0, k, 2, off, tok, conf, probs)
        draft = torch.zeros((CH, N, V), dtype=torch.float32, device="cuda")
        if conditioned:
            cuda_lib.draft_child_rows(probs, tok, rows)
            draft[:, 1:] = rows[:, 0]
        else:
            draft[:, 1:] = probs[:, 0][:, None, :]
        tokens = torch.zeros((CH, N), dtype=torch.int32, device="cuda")
        tokens[:, 1:] = tok[:, 0]
        cuda_lib.tree_accept(shape, logits, draft, tokens, parents, 1.0, 2, off, acc, alen, nxt)
        torch.cuda.synchronize()
        a, al, nx, tk = acc.cpu().numpy(), alen.cpu().numpy(), nxt.cpu().numpy(), tokens.cpu().numpy()
        first = np.where(al >= 1, tk[np.arange(CH), np.maximum(a[:, 0], 0)], nx)
        counts += np.bincount(first, minlength=V)
    assert cuda_lib.device_error(reset=True) == 0
    pv = stats.chisquare(counts, counts.sum() * p).pvalue
    if conditioned:
        assert pv > 0.01, (pv, counts / counts.sum(), p)
    else:
        assert pv < 1e-6, (pv, counts / counts.sum(), p)
