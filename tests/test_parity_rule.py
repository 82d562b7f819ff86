"""The margin rule the GPU walk is compared under (tests/parity.py) and the oracle
diagnostics it reads: a decision whose margin is within 1e-4 may go either way on the GPU,
every decision before it must not (EAGLE summary, section 2 "Preliminaries": each drafted
token is accepted with probability min(1, p/p_hat); the GPU decides in fp32, the oracle in
fp64, so only decisions with a margin are comparable bit for bit)."""
import numpy as np
import pytest

from tests.parity import MARGIN, compare_accept


def _ref(acc, alen, nxt, decisions, first_near=-1, exact_len=None, near_child=-1):
    N = len(acc)
    return dict(accepted_nodes=np.asarray([acc], np.int32), accept_len=np.asarray([alen], np.int32),
                next_token=np.asarray([nxt], np.int32), near=np.asarray([int(first_near >= 0)], np.int32),
                decisions=np.asarray([decisions], np.int32), first_near=np.asarray([first_near], np.int32),
                exact_len=np.asarray([alen if exact_len is None else exact_len], np.int32),
                near_child=np.asarray([near_child], np.int32))


def _gpu(acc, alen, nxt):
    return dict(accepted_nodes=np.asarray([acc], np.int32), accept_len=np.asarray([alen], np.int32),
                next_token=np.asarray([nxt], np.int32))


# root 0 with children 1, 2, 3; node 1 has children 4, 5
PAR = np.asarray([[-1, 0, 0, 0, 1, 1]], np.int32)


def test_no_near_decision_compares_everything():
    ref = _ref([1, 4, -1, -1, -1, -1], 2, 7, decisions=3)
    st = compare_accept(_gpu([1, 4, -1, -1, -1, -1], 2, 7), ref, PAR)
    assert (st.whole, st.compared, st.excluded) == (1, 3, 0)
    with pytest.raises(AssertionError):
        compare_accept(_gpu([1, 4, -1, -1, -1, -1], 2, 8), ref, PAR)  # another extra token
    with pytest.raises(AssertionError):
        compare_accept(_gpu([1, 5, -1, -1, -1, -1], 2, 7), ref, PAR)  # another child


def test_near_candidate_allows_either_outcome_for_it_only():
    # the oracle rejected candidate 1 outside the margin, then met candidate 2 inside it
    ref = _ref([2, -1, -1, -1, -1, -1], 1, 9, decisions=3, first_near=1, exact_len=0, near_child=2)
    for acc, n in (([2, -1, -1, -1, -1, -1], 1), ([3, -1, -1, -1, -1, -1], 1), ([-1] * 6, 0)):
        st = compare_accept(_gpu(acc, n, 5), ref, PAR)
        assert (st.whole, st.compared, st.excluded) == (0, 1, 2)
    # accepting candidate 1 contradicts a decision taken outside the margin
    with pytest.raises(AssertionError):
        compare_accept(_gpu([1, -1, -1, -1, -1, -1], 1, 5), ref, PAR)
    # not a root path
    with pytest.raises(AssertionError):
        compare_accept(_gpu([4, -1, -1, -1, -1, -1], 1, 5), ref, PAR)


def test_near_decision_deeper_fixes_the_prefix():
    ref = _ref([1, 5, -1, -1, -1, -1], 2, 3, decisions=4, first_near=2, exact_len=1, near_child=5)
    compare_accept(_gpu([1, -1, -1, -1, -1, -1], 1, 0), ref, PAR)
    compare_accept(_gpu([1, 5, -1, -1, -1, -1], 2, 0), ref, PAR)
    with pytest.raises(AssertionError):
        compare_accept(_gpu([2, -1, -1, -1, -1, -1], 1, 0), ref, PAR)   # prefix differs
    with pytest.raises(AssertionError):
        compare_accept(_gpu([1, 4, -1, -1, -1, -1], 2, 0), ref, PAR)    # 4 was rejected outside the margin


def test_near_final_race_fixes_the_whole_path():
    ref = _ref([1, -1, -1, -1, -1, -1], 1, 11, decisions=4, first_near=3, exact_len=1, near_child=-1)
    st = compare_accept(_gpu([1, -1, -1, -1, -1, -1], 1, 12), ref, PAR)
    assert (st.compared, st.excluded) == (3, 1)
    with pytest.raises(AssertionError):
        compare_accept(_gpu([1, 4, -1, -1, -1, -1], 2, 12), ref, PAR)


def test_near_greedy_argmax_allows_another_match():
    ref = _ref([1, -1, -1, -1, -1, -1], 1, 11, decisions=2, first_near=0, exact_len=0, near_child=-2)
    compare_accept(_gpu([3, -1, -1, -1, -1, -1], 1, 2), ref, PAR)
    compare_accept(_gpu([-1] * 6, 0, 2), ref, PAR)


def test_oracle_locates_its_first_near_decision(orc):
    """A walk built so that the accept test of the root's second candidate sits on its
    threshold: the oracle reports that decision as the first near one, with the first
    candidate's rejection (far from its threshold) before it."""
    V, N, T, seed, offset = 16, 3, 1.0, 5, 9
    rng = np.random.default_rng(3)
    logits = rng.standard_normal((1, N, V)).astype(np.float32)
    tokens = np.asarray([[0, 3, 6]], np.int32)
    par = np.asarray([[-1, 0, 0]], np.int32)
    p = np.exp(logits[0, 0].astype(np.float64) / T)
    p /= p.sum()
    draft = np.zeros((1, N, V), np.float32)
    # candidate 1: p_hat one-hot on its token, so its ratio is p(3); the seed puts its
    # uniform well above that
    draft[0, 1, 3] = 1.0
    u1 = orc.uniform(seed, offset, 0, 1, 0, 0)
    assert abs(u1 - p[3]) > 10 * MARGIN and u1 > p[3]  # rejected outside the margin
    # after the rejection p becomes p without token 3, renormalised
    r = p.copy()
    r[3] = 0.0
    r /= r.sum()
    u2 = orc.uniform(seed, offset, 0, 2, 0, 0)
    # candidate 2: p_hat(6) chosen so that p(6) / p_hat(6) equals u2 (to float32 rounding)
    q6 = np.float32(r[6] / u2)
    assert 0 < q6 < 1
    draft[0, 2, 6] = q6
    draft[0, 2, 0] = 1.0 - q6
    ref = orc.tree_accept(draft, tokens, par, T, seed=seed, offset=offset, logits=logits, margin=MARGIN)
    assert ref["first_near"][0] == 1
    assert ref["exact_len"][0] == 0
    assert ref["near_child"][0] == 2
    assert ref["near"][0] >= 1
    # with a margin of zero nothing is near and exact_len is the whole path
    ref0 = orc.tree_accept(draft, tokens, par, T, seed=seed, offset=offset, logits=logits, margin=0.0)
    assert ref0["first_near"][0] == -1 and ref0["near_child"][0] == -1
    assert ref0["exact_len"][0] == ref0["accept_len"][0]
