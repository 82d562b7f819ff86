"""Comparison helpers shared by the GPU parity tests."""
import numpy as np

# Tolerances (stated for this verification step): fp32 paths 1e-5 relative, bf16 paths
# 2e-2 after normalisation; both measured per output row as max|gpu - ref| / max|ref|.
TOL = {"f32": 1e-5, "bf16": 2e-2}
MARGIN = 1e-4


def row_rel_err(gpu: np.ndarray, ref: np.ndarray) -> np.ndarray:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    num = np.abs(gpu - ref).max(axis=-1)
    den = np.abs(ref).max(axis=-1)
    return num / np.maximum(den, 1e-30)


def is_root_path(parents, accepted, n):
    """accepted[0:n] is a chain root -> ... with each node the child of the previous."""
    prev = 0
    for k in range(n):
        c = int(accepted[k])
        if c <= 0 or parents[c] != prev:
            return False
        prev = c
    return True


class AcceptStats(dict):
    """What a walk comparison covered: ``whole`` sequences compared in full (path, length
    and extra token), ``compared`` decisions compared bit for bit out of ``decisions``
    taken by the oracle, ``excluded`` decisions past a sequence's first near decision."""

    def __init__(self, B):
        super().__init__(whole=0, compared=0, decisions=0, excluded=0, per_seq=[0] * B)

    def __getattr__(self, k):
        return self[k]


def compare_accept(gpu: dict, ref: dict, parents: np.ndarray, exact_all: bool = False):
    """Decision-by-decision comparison of the walk under the margin rule (a decision whose
    margin is within MARGIN may go either way; see the oracle's near/first_near outputs).

    Per sequence, every decision the oracle took before its first near decision must come
    out the same on the GPU:
      * no near decision (or ``exact_all``): the accepted path, its length and the extra
        token are equal;
      * otherwise the first ``exact_len`` accepted nodes are equal, and what follows
        depends on the near decision:
          - it tested candidate c: its earlier siblings were rejected outside the margin,
            so the GPU either stops there or accepts c or a later sibling;
          - it is the final race (-1): the whole path is fixed, only the token may differ;
          - it is a greedy argmax (-2): the GPU may match another child or stop;
        and the rest of the GPU's walk must be a valid root path.
    Returns an AcceptStats."""
    B, N = parents.shape
    st = AcceptStats(B)
    for b in range(B):
        g_len = int(gpu["accept_len"][b])
        g_acc = np.asarray(gpu["accepted_nodes"][b])
        r_len = int(ref["accept_len"][b])
        n_dec = int(ref["decisions"][b])
        first = int(ref["first_near"][b])
        st["decisions"] += n_dec
        if exact_all or first < 0:
            assert g_len == r_len, (b, g_len, r_len)
            np.testing.assert_array_equal(g_acc, ref["accepted_nodes"][b])
            assert gpu["next_token"][b] == ref["next_token"][b], (b, gpu["next_token"][b], ref["next_token"][b])
            st["whole"] += 1
            st["compared"] += n_dec
            st["per_seq"][b] = n_dec
            continue
        k = int(ref["exact_len"][b])
        nc = int(ref["near_child"][b])
        assert 0 <= g_len < N and is_root_path(parents[b], g_acc, g_len), (b, g_len, g_acc)
        assert (g_acc[g_len:] == -1).all(), (b, g_acc)
        assert g_len >= k, (b, g_len, k)
        np.testing.assert_array_equal(g_acc[:k], ref["accepted_nodes"][b][:k])
        if nc >= 0:
            # siblings tested before candidate nc were rejected outside the margin
            assert g_len == k or int(g_acc[k]) >= nc, (b, g_acc[k], nc)
        elif nc == -1:
            # every candidate at the last node was rejected outside the margin
            assert g_len == k, (b, g_len, k)
        st["compared"] += first
        st["excluded"] += n_dec - first
        st["per_seq"][b] = first
    return st
