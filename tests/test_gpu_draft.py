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
